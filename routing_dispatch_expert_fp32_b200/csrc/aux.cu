// aux.cu -- moe_aux_loss: GShard's load-balancing loss for the router.
//
// PopFetcher, section 2.3.1, names GShard's load-balancing loss (it evens out
// the workload across workers) without the formula.  Reading taken (the
// GShard / Switch form):
//   f_e  = counts[e] / (T k)              routed fraction of expert e
//   P_e  = mean over tokens of softmax(z)_e,  z = logits + bias
//   loss = E * sum_e f_e P_e
//
// K1 aux_partial: one CTA per chunk of 256 tokens; a group of L lanes holds one
//    token's keys (as in the router), takes the max and the softmax denominator
//    by butterfly reductions, and each lane accumulates its experts'
//    probabilities over the warp's tokens in a fixed order; groups, then warps,
//    are combined in a fixed order into one fp32 partial per (chunk, expert).
// K2 aux_final: one CTA sums the chunk partials in double (chunks ascending),
//    forms P_e, f_e and the loss (fixed-order block reduction).
// Deterministic: no atomics, every sum in a fixed order.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kAuxChunk = 256;

template <int VPL>
constexpr int aux_threads() { return VPL >= 16 ? 256 : 1024; }

template <int L, int VPL>
__global__ void __launch_bounds__(aux_threads<VPL>())
aux_partial_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E,
                   float* __restrict__ partial) {
    constexpr int kThreads = aux_threads<VPL>();
    constexpr int kWarps = kThreads / 32;
    constexpr int G = 32 / L;
    constexpr int kPerWarp = kAuxChunk / kWarps;
    constexpr int kIters = kPerWarp / G;
    constexpr int kEMax = L * VPL;  // experts this instantiation handles
    __shared__ float s_part[kWarps][kEMax];
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane / L, gl = lane % L;
    float b[VPL], acc[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = gl + i * L;
        b[i] = (bias != nullptr && e < E) ? bias[e] : 0.0f;
        acc[i] = 0.0f;
    }
    const int t_warp = blockIdx.x * kAuxChunk + warp * kPerWarp;
#pragma unroll 1
    for (int it = 0; it < kIters; ++it) {
        const int t = t_warp + it * G + g;
        const bool active = t < T;
        const float* row = logits + (size_t)(active ? t : T - 1) * E;
        float z[VPL];
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = gl + i * L;
            z[i] = (e < E) ? __fadd_rn(__ldg(row + e), b[i]) : -INFINITY;
            m = fmaxf(m, z[i]);
        }
#pragma unroll
        for (int off = L / 2; off > 0; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off, L));
        float ex[VPL], s = 0.0f;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            ex[i] = (gl + i * L < E) ? expf(__fsub_rn(z[i], m)) : 0.0f;
            s = __fadd_rn(s, ex[i]);
        }
#pragma unroll
        for (int off = L / 2; off > 0; off >>= 1)
            s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off, L));
        if (active) {
#pragma unroll
            for (int i = 0; i < VPL; ++i) acc[i] = __fadd_rn(acc[i], __fdiv_rn(ex[i], s));
        }
    }
    // groups of the warp hold the same experts: fold them (fixed order)
#pragma unroll
    for (int off = L; off < 32; off <<= 1)
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            acc[i] = __fadd_rn(acc[i], __shfl_xor_sync(0xffffffffu, acc[i], off));
    if (g == 0) {
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = gl + i * L;
            if (e < E) s_part[warp][e] = acc[i];
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads) {
        float v = 0.0f;
        for (int wv = 0; wv < kWarps; ++wv) v = __fadd_rn(v, s_part[wv][e]);
        partial[(size_t)blockIdx.x * E + e] = v;
    }
}

__global__ void __launch_bounds__(1024)
aux_final_kernel(const float* __restrict__ partial, int nchunks, int T, int E, int k,
                 const int32_t* __restrict__ counts, float* __restrict__ loss,
                 float* __restrict__ prob_mean) {
    __shared__ double s_red[1024];
    pdl_wait();
    pdl_trigger();
    double mine = 0.0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        double S = 0.0;
        for (int c = 0; c < nchunks; ++c) S += (double)partial[(size_t)c * E + e];
        const double Pe = T > 0 ? S / (double)T : 0.0;
        const double fe = T > 0 ? (double)counts[e] / ((double)T * (double)k) : 0.0;
        mine += fe * Pe;
        if (prob_mean) prob_mean[e] = (float)Pe;
    }
    s_red[threadIdx.x] = mine;
    __syncthreads();
    for (int half = blockDim.x / 2; half > 0; half >>= 1) {
        if ((int)threadIdx.x < half) s_red[threadIdx.x] += s_red[threadIdx.x + half];
        __syncthreads();
    }
    if (threadIdx.x == 0) loss[0] = (float)((double)E * s_red[0]);
}

template <int L, int VPL>
int launch_partial(int nchunks, cudaStream_t st, const float* logits, const float* bias, int T,
                   int E, float* partial) {
    return launch_pdl(aux_partial_kernel<L, VPL>, nchunks, aux_threads<VPL>(), 0, st, logits,
                      bias, T, E, partial);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_aux_loss(const float* logits, const float* bias, int T, int E, int k,
                                    const int32_t* counts, float* loss, float* prob_mean,
                                    void* workspace, size_t workspace_bytes,
                                    moe_stream_t stream) {
    if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
    if (!counts || !loss || (T > 0 && !logits)) return MOE_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < moe_route_workspace_size(T, E, k)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int nchunks = (T + kAuxChunk - 1) / kAuxChunk;
    float* partial = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(workspace) + 255u) &
                                              ~uintptr_t(255u));
    if (T > 0) {
        int rc;
        if (E <= 8) rc = launch_partial<8, 1>(nchunks, st, logits, bias, T, E, partial);
        else if (E <= 16) rc = launch_partial<16, 1>(nchunks, st, logits, bias, T, E, partial);
        else if (E <= 32) rc = launch_partial<32, 1>(nchunks, st, logits, bias, T, E, partial);
        else if (E <= 64) rc = launch_partial<32, 2>(nchunks, st, logits, bias, T, E, partial);
        else if (E <= 128) rc = launch_partial<32, 4>(nchunks, st, logits, bias, T, E, partial);
        else if (E <= 256) rc = launch_partial<32, 8>(nchunks, st, logits, bias, T, E, partial);
        else if (E <= 512) rc = launch_partial<32, 16>(nchunks, st, logits, bias, T, E, partial);
        else rc = launch_partial<32, 32>(nchunks, st, logits, bias, T, E, partial);
        if (rc != MOE_OK) return MOE_ERR_CUDA;
    }
    return launch_pdl(aux_final_kernel, 1, 1024, 0, st, (const float*)partial, nchunks, T, E, k,
                      counts, loss, prob_mean);
}
