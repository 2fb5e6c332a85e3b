// forecast.cu -- cross-layer expert correlation and the popularity forecast.
//
// PopFetcher, section 4.1 (Fig. 6): a token's expert choices at two consecutive
// MoE layers form a correlated pair (x, x'), and the next layer's hot experts
// follow from the previous layer's choices.  Section 4.2 (Eq. 2-3, lost in
// extraction): the conditional probability of the next-layer expert given the
// previous-layer one, and a popularity forecast built from it.  Reading taken:
//   C[i][h]  += tokens that chose i at layer j and h at layer j+1
//   P(h|i)    = C[i][h] / n_i,  n_i = (sum_h C[i][h]) / k_next
//   pred[h]   = sum_i pop_prev[i] * P(h|i) / k_prev
//
// moe_correlation_update: one thread per token adds its k_prev x k_next pairs;
// for E <= 128 into a per-CTA shared-memory histogram flushed with one global
// atomicAdd per non-zero bin, else straight into global memory.  Integer sums
// commute, so the result does not depend on the order.
// moe_popularity_forecast: one CTA of 1024 threads.  Row sums S_i (a warp per
// row), then q_i = (pop_i * k_next) / (S_i * k_prev) and, with C streamed
// through shared memory in row chunks, pred[h] = sum_i q_i * C[i][h] in
// IEEE double with every operation rounded separately (no fused multiply-add),
// i ascending, rounded once to fp32: bit-identical to the same sequence of
// operations done anywhere else.  Hot experts: rank by (pred desc, index asc).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kCorrThreads = 256;
constexpr int kCorrSmemMaxE = 128;

template <bool SMEM>
__global__ void __launch_bounds__(kCorrThreads)
correlation_kernel(const int32_t* __restrict__ ids_prev, int k_prev,
                   const int32_t* __restrict__ ids_next, int k_next, int T, int E,
                   int32_t* __restrict__ C, int32_t* err) {
    extern __shared__ int32_t s_c[];  // [E][E] when SMEM
    pdl_wait();
    pdl_trigger();
    if (SMEM) {
        for (int i = threadIdx.x; i < E * E; i += kCorrThreads) s_c[i] = 0;
        __syncthreads();
    }
    for (int t = blockIdx.x * kCorrThreads + threadIdx.x; t < T;
         t += gridDim.x * kCorrThreads) {
        for (int a = 0; a < k_prev; ++a) {
            const int i = ids_prev[(size_t)t * k_prev + a];
            if (i < 0 || i >= E) {
                flag_error(err, MOE_DEVERR_EXPERT_INDEX);
                continue;
            }
            for (int b = 0; b < k_next; ++b) {
                const int h = ids_next[(size_t)t * k_next + b];
                if (h < 0 || h >= E) {
                    flag_error(err, MOE_DEVERR_EXPERT_INDEX);
                    continue;
                }
                if (SMEM) atomicAdd(&s_c[i * E + h], 1);
                else atomicAdd(&C[(size_t)i * E + h], 1);
            }
        }
    }
    if (SMEM) {
        __syncthreads();
        for (int i = threadIdx.x; i < E * E; i += kCorrThreads)
            if (s_c[i]) atomicAdd(&C[i], s_c[i]);
    }
}

constexpr int kForecastThreads = 1024;
constexpr int kForecastStage = 8192;  // int32 counters staged per pass (32 KB)

__global__ void __launch_bounds__(kForecastThreads)
forecast_kernel(const float* __restrict__ pop_prev, const int32_t* __restrict__ C, int E,
                int k_prev, int k_next, float* __restrict__ pred, int P, int32_t* __restrict__ hot) {
    __shared__ double s_q[kMaxExperts];
    __shared__ float s_pred[kMaxExperts];
    __shared__ int32_t s_c[kForecastStage];
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = kForecastThreads / 32;
    for (int i = warp; i < E; i += kWarps) {
        long long s = 0;
        for (int h = lane; h < E; h += 32) s += C[(size_t)i * E + h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
            const double num = __dmul_rn((double)pop_prev[i], (double)k_next);
            const double den = __dmul_rn((double)s, (double)k_prev);
            s_q[i] = s == 0 ? 0.0 : __ddiv_rn(num, den);
        }
    }
    // pred[h] = sum over i ascending of q_i * C[i][h]; rows of C pass through
    // shared memory in chunks, each thread owning columns h = tid, tid + 1024
    const int rows_per_pass = kForecastStage / E;
    double acc = 0.0;  // thread's column h = tid (E <= 1024)
    for (int i0 = 0; i0 < E; i0 += rows_per_pass) {
        const int i1 = min(E, i0 + rows_per_pass);
        __syncthreads();  // s_q ready (first pass) / previous chunk consumed
        for (int idx = tid; idx < (i1 - i0) * E; idx += kForecastThreads)
            s_c[idx] = C[(size_t)i0 * E + idx];
        __syncthreads();
        if (tid < E)
            for (int i = i0; i < i1; ++i)
                acc = __dadd_rn(acc, __dmul_rn(s_q[i], (double)s_c[(i - i0) * E + tid]));
    }
    if (tid < E) {
        const float f = __double2float_rn(acc);
        pred[tid] = f;
        s_pred[tid] = f;
    }
    __syncthreads();
    for (int h = tid; h < E; h += kForecastThreads) {
        const float mine = s_pred[h];
        int rank = 0;
        for (int o = 0; o < E; ++o) {
            const float v = s_pred[o];
            rank += (v > mine) || (v == mine && o < h);
        }
        if (rank < P) hot[rank] = h;
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_correlation_update(const int32_t* ids_prev, int k_prev,
                                              const int32_t* ids_next, int k_next, int T, int E,
                                              int32_t* C, moe_stream_t stream) {
    if (T < 0 || E < 1 || E > kMaxExperts || k_prev < 1 || k_prev > E || k_next < 1 ||
        k_next > E)
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * k_prev >= INT32_MAX || (int64_t)T * k_next >= INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (!C || (T > 0 && (!ids_prev || !ids_next))) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int grid = (T + kCorrThreads - 1) / kCorrThreads;
    const int cap = num_sms() * 2;
    if (grid > cap) grid = cap;
    if (E <= kCorrSmemMaxE) {
        const int smem = E * E * 4;
        if (ensure_smem<correlation_kernel<true>>(smem) != MOE_OK) return MOE_ERR_CUDA;
        return launch_pdl(correlation_kernel<true>, grid, kCorrThreads, smem, st, ids_prev,
                          k_prev, ids_next, k_next, T, E, C, device_error_word());
    }
    return launch_pdl(correlation_kernel<false>, grid, kCorrThreads, 0, st, ids_prev, k_prev,
                      ids_next, k_next, T, E, C, device_error_word());
}

extern "C" MOE_API int moe_popularity_forecast(const float* pop_prev, const int32_t* C, int E,
                                               int k_prev, int k_next, float* pred, int P,
                                               int32_t* hot, moe_stream_t stream) {
    if (E < 1 || E > kMaxExperts || k_prev < 1 || k_next < 1 || P < 0 || P > E)
        return MOE_ERR_INVALID_ARG;
    if (!pop_prev || !C || !pred || (P > 0 && !hot)) return MOE_ERR_INVALID_ARG;
    return launch_pdl(forecast_kernel, 1, kForecastThreads, 0,
                      reinterpret_cast<cudaStream_t>(stream), pop_prev, C, E, k_prev, k_next, pred,
                      P, hot);
}
