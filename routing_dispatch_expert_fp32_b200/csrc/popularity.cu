// popularity.cu -- moe_popularity_update: per-expert popularity over a
// sliding window of steps.
//
// PopFetcher, section 3.1: the routing information collector counts the tokens
// routed to each expert (the expert's popularity).  Section 4.2, Eq. 1 (lost in
// extraction): popularity is averaged over a window of recent iterations.
// Reading taken: mean of the last n = min(step + 1, W) count vectors; hot
// experts ranked by window sum (desc), equal sums to the lower index.
//
// One CTA: thread e writes this step's count into ring row step % W, sums its
// column over the n live rows (int64) and writes the correctly rounded mean;
// then one warp per expert counts the experts ranked above it (32 sums per
// lane pass, a warp sum), and the expert of rank r < P is hot[r].
#include "common.cuh"

namespace moe {

// The step comes from `step_ptr` when it is not null (and is advanced by one at
// the end), else from `step_arg`.
__global__ void __launch_bounds__(1024)
popularity_kernel(const int32_t* __restrict__ counts, int E, int32_t* __restrict__ hist, int W,
                  long long step_arg, long long* step_ptr, float* __restrict__ mean, int P,
                  int32_t* __restrict__ hot) {
    __shared__ long long s_sum[kMaxExperts];
    pdl_wait();
    pdl_trigger();
    const long long step = step_ptr ? *step_ptr : step_arg;
    if (step < 0) return;
    const int slot = (int)(step % W);
    const long long n = step + 1 < W ? step + 1 : W;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int32_t c = counts[e];
        hist[(size_t)slot * E + e] = c;
        long long sum = c;
        // rows of the n - 1 earlier live steps: slot - 1, slot - 2, ... wrapped
        // into [0, W) (no 64-bit division per row)
#pragma unroll 4
        for (int i = 1; i < (int)n; ++i) {
            const int s = slot - i < 0 ? slot - i + W : slot - i;
            sum += hist[(size_t)s * E + e];
        }
        s_sum[e] = sum;
        mean[e] = __fdiv_rn(__ll2float_rn(sum), __ll2float_rn(n));
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    for (int e = threadIdx.x >> 5; e < E; e += nwarps) {
        const long long mine = s_sum[e];
        int above = 0;
        for (int o = lane; o < E; o += 32) {
            const long long v = s_sum[o];
            above += (v > mine) || (v == mine && o < e);
        }
        const int rank = __reduce_add_sync(0xffffffffu, above);
        if (lane == 0 && rank < P) hot[rank] = e;
    }
    if (step_ptr) {
        __syncthreads();  // every thread has read the step
        if (threadIdx.x == 0) *step_ptr = step + 1;
    }
}

// A thread per expert for the window sums and a warp per expert (up to 32
// warps) for the ranks.
static int popularity_threads(int E) {
    const int t = ((E + 31) / 32) * 32;
    return t < 1024 ? (E < 32 ? 32 : (t * 4 < 1024 ? t * 4 : 1024)) : 1024;
}

}  // namespace moe

extern "C" MOE_API int moe_popularity_update(const int32_t* counts, int E, int32_t* hist, int W,
                                     int64_t step, float* mean, int P, int32_t* hot,
                                     moe_stream_t stream) {
    using namespace moe;
    if (E < 1 || E > kMaxExperts || W < 1 || step < 0 || P < 0 || P > E) return MOE_ERR_INVALID_ARG;
    if (!counts || !hist || !mean || (P > 0 && !hot)) return MOE_ERR_INVALID_ARG;
    return launch_pdl(popularity_kernel, 1, popularity_threads(E), 0,
                      reinterpret_cast<cudaStream_t>(stream), counts, E, hist, W, (long long)step,
                      (long long*)nullptr, mean, P, hot);
}

extern "C" MOE_API int moe_popularity_update_dev(const int32_t* counts, int E, int32_t* hist, int W,
                                         int64_t* step, float* mean, int P, int32_t* hot,
                                         moe_stream_t stream) {
    using namespace moe;
    if (E < 1 || E > kMaxExperts || W < 1 || P < 0 || P > E) return MOE_ERR_INVALID_ARG;
    if (!counts || !hist || !mean || !step || (P > 0 && !hot)) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(step) & 7u) != 0) return MOE_ERR_UNSUPPORTED;
    return launch_pdl(popularity_kernel, 1, popularity_threads(E), 0,
                      reinterpret_cast<cudaStream_t>(stream), counts, E, hist, W, 0LL,
                      reinterpret_cast<long long*>(step), mean, P, hot);
}
