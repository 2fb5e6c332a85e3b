// route.cu -- moe_route: top-k softmax gate with GShard expert capacity.
//
// "A Survey on Mixture of Experts", section 5 (gate routing; tokens dispatched
// under an expert-capacity limit) and PopFetcher, section 2.1.2 (top-k gate).
//
// Three launches, no inter-CTA waiting:
//   K1 route_topk    one CTA of 32 warps (8 for E > 256) per chunk of 256 tokens (8 per warp;
//                    the next token's logits are loaded while the current one
//                    is ranked).  A group of L lanes
//                    (L = 8, 16 or 32) scores one token: each lane holds E/L
//                    of the fp32 keys z = logit + bias (coalesced loads), k
//                    rounds of a butterfly argmax under the total order
//                    (z desc, index asc) pick the experts, lane j keeps slot j
//                    and computes w_j = exp(z_j - z_0) / sum_i exp(z_i - z_0).
//                    Per-chunk expert histogram in shared memory (atomicAdd
//                    on counts commutes, so the result is order-free).
//   K2 route_scan    one CTA: per expert, exclusive prefix of the chunk
//                    histograms (two-level: segments of chunks, then chunks),
//                    counts, kept = min(counts, capacity), offsets = exclusive
//                    scan of kept, n_dropped.
//   K3 route_assign  one CTA per chunk again (a token per thread); a slot's position inside its
//                    expert = chunk base + slots of earlier warps of the chunk
//                    + earlier lanes of its warp, all from per-warp lane masks
//                    (atomicOr commutes; popc of the lower-lane bits gives the
//                    token-order rank).  Position < capacity -> row, else -1.
#include <climits>

#include "common.cuh"

namespace moe {

constexpr int kChunk = 256;        // tokens per chunk (= per CTA in K1 and K3)
// K1 threads: 32 warps (kChunk / 32 tokens each); 8 warps when a lane holds
// 16 or more keys, so the keys of two tokens stay in registers.
template <int VPL>
constexpr int topk_threads() { return VPL >= 16 ? 256 : 1024; }
constexpr int kThreads = kChunk;   // K3: one token per thread
constexpr int kWarps = kThreads / 32;
constexpr int kScanThreads = 1024;

__device__ __forceinline__ bool key_better(float av, int ai, float bv, int bi) {
    return av > bv || (av == bv && ai < bi);
}

// Order-preserving map of a finite fp32 to uint32 (larger float -> larger
// key); -0.0 is folded onto +0.0 first so that the two still tie.
__device__ __forceinline__ uint32_t order_key(float z) {
    const uint32_t u = __float_as_uint(z == 0.0f ? 0.0f : z);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// ------------------------------------------------------------------- K1 ----
template <int L, int VPL>
__global__ void __launch_bounds__(topk_threads<VPL>())
route_topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E,
                  int k, int32_t* __restrict__ ids, float* __restrict__ w,
                  int32_t* __restrict__ chunk_hist) {
    __shared__ int s_hist[kMaxExperts];
    constexpr int kTopkThreads = topk_threads<VPL>();
    for (int e = threadIdx.x; e < E; e += kTopkThreads) s_hist[e] = 0;
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    constexpr int G = 32 / L;                          // tokens per warp per iteration
    constexpr int kPerWarp = kChunk / (kTopkThreads / 32);
    constexpr int kIters = kPerWarp / G;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane / L, gl = lane % L;

    // this lane's experts are gl, gl + L, gl + 2L, ...
    float b[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = gl + i * L;
        b[i] = (bias != nullptr && e < E) ? bias[e] : 0.0f;
    }

    const int t_warp = blockIdx.x * kChunk + warp * kPerWarp;
    float zn[VPL];  // logits of the next token of this group, in flight
    {
        const int t = min(t_warp + g, T - 1);
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = gl + i * L;
            zn[i] = (e < E) ? __ldg(logits + (size_t)t * E + e) : 0.0f;
        }
    }
#pragma unroll 1
    for (int it = 0; it < kIters; ++it) {
        const int t = t_warp + it * G + g;
        const bool active = t < T;
        float z[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = gl + i * L;
            z[i] = (e < E) ? __fadd_rn(zn[i], b[i]) : -INFINITY;
        }
        if (it + 1 < kIters) {
            const int tn = min(t + G, T - 1);
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int e = gl + i * L;
                zn[i] = (e < E) ? __ldg(logits + (size_t)tn * E + e) : 0.0f;
            }
        }

        uint32_t taken = 0;
        float my_z = 0.0f;
        int my_e = 0;
        if constexpr (L == 32) {
            // One token per warp: per round, the largest order key by a warp
            // reduction, then the lowest expert index among the lanes holding
            // it (each lane's candidate is its own lowest-index maximum).
            uint32_t key[VPL];
#pragma unroll
            for (int i = 0; i < VPL; ++i) key[i] = (gl + i * L < E) ? order_key(z[i]) : 0u;
            for (int r = 0; r < k; ++r) {
                uint32_t bk = 0u;
                int bi = INT_MAX;
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    if (!((taken >> i) & 1u) && key[i] > bk) {
                        bk = key[i];
                        bi = gl + i * L;
                    }
                }
                const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
                const int win = (int)__reduce_min_sync(0xffffffffu, bk == m ? (uint32_t)bi : 0xffffffffu);
                if (win % L == gl) taken |= 1u << (win / L);
                if (gl == r) {
                    my_z = key_value(m);
                    my_e = win;
                }
            }
        } else {
            for (int r = 0; r < k; ++r) {
                float bv = -INFINITY;
                int bi = INT_MAX;
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int e = gl + i * L;
                    if (e < E && !((taken >> i) & 1u) && key_better(z[i], e, bv, bi)) {
                        bv = z[i];
                        bi = e;
                    }
                }
#pragma unroll
                for (int off = L / 2; off > 0; off >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, off, L);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, off, L);
                    if (key_better(ov, oi, bv, bi)) {
                        bv = ov;
                        bi = oi;
                    }
                }
                // every lane of the group now holds the same winner
                if (bi % L == gl) taken |= 1u << (bi / L);
                if (gl == r) {
                    my_z = bv;
                    my_e = bi;
                }
            }
        }

        const float z0 = __shfl_sync(0xffffffffu, my_z, 0, L);
        const float ex = (gl < k) ? expf(__fsub_rn(my_z, z0)) : 0.0f;
        float s = 0.0f;
        for (int i = 0; i < k; ++i) s = __fadd_rn(s, __shfl_sync(0xffffffffu, ex, i, L));
        if (active && gl < k) {
            ids[(size_t)t * k + gl] = my_e;
            w[(size_t)t * k + gl] = __fdiv_rn(ex, s);
            atomicAdd(&s_hist[my_e], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kTopkThreads)
        chunk_hist[(size_t)blockIdx.x * E + e] = s_hist[e];
}

// ------------------------------------------------------------------- K2 ----
__global__ void __launch_bounds__(kScanThreads)
route_scan_kernel(const int32_t* __restrict__ chunk_hist, int nchunks, int T, int E, int k,
                  int capacity, int32_t* __restrict__ chunk_base, int32_t* __restrict__ counts,
                  int32_t* __restrict__ kept, int32_t* __restrict__ offsets,
                  int32_t* __restrict__ n_dropped) {
    __shared__ int32_t s_seg[kScanThreads];  // [segment][expert]
    __shared__ int32_t s_warp[kScanThreads / 32];
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x;
    const int S = kScanThreads / E;              // segments (E <= 1024 so S >= 1)
    const int cps = (nchunks + S - 1) / S;       // chunks per segment
    const int e = tid % E, seg = tid / E;
    const bool worker = seg < S;
    const int c0 = seg * cps, c1 = min(nchunks, c0 + cps);

    // phase 1: per (segment, expert) totals
    int32_t part = 0;
    if (worker) {
#pragma unroll 8
        for (int c = c0; c < c1; ++c) part += chunk_hist[(size_t)c * E + e];
    }
    if (worker) s_seg[seg * E + e] = part;
    __syncthreads();

    // phase 2: per expert, exclusive over segments; totals are the counts
    int32_t my_kept = 0;
    if (tid < E) {
        int32_t run = 0;
        for (int s = 0; s < S; ++s) {
            const int32_t v = s_seg[s * E + tid];
            s_seg[s * E + tid] = run;
            run += v;
        }
        counts[tid] = run;
        my_kept = (capacity > 0 && run > capacity) ? capacity : run;
        kept[tid] = my_kept;
    }
    __syncthreads();

    // phase 3: per chunk bases
    if (worker) {
        int32_t run = s_seg[seg * E + e];
#pragma unroll 8
        for (int c = c0; c < c1; ++c) {
            const int32_t v = chunk_hist[(size_t)c * E + e];
            chunk_base[(size_t)c * E + e] = run;
            run += v;
        }
    }

    // exclusive scan of kept over experts (block scan; tid >= E contributes 0)
    const int lane = tid & 31, wid = tid >> 5;
    int32_t incl = my_kept;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int32_t v = s_warp[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int32_t o = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += o;
        }
        s_warp[lane] = v;  // inclusive over warps
    }
    __syncthreads();
    const int32_t before = (wid > 0 ? s_warp[wid - 1] : 0) + incl - my_kept;
    if (tid < E) offsets[tid] = before;
    if (tid == 0) {
        const int32_t total = s_warp[31];
        offsets[E] = total;
        n_dropped[0] = (int32_t)((int64_t)T * k - total);
    }
}

// ------------------------------------------------------------------- K3 ----
__global__ void __launch_bounds__(kThreads)
route_assign_kernel(const int32_t* __restrict__ ids, int T, int E, int k, int capacity,
                    const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ offsets,
                    int32_t* __restrict__ slot_row, int32_t* __restrict__ row_slot) {
    __shared__ uint32_t s_mask[kWarps][kMaxExperts];
    __shared__ int32_t s_base[kMaxExperts];
    __shared__ int32_t s_off[kMaxExperts];
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < E; e += kThreads) {
        s_base[e] = chunk_base[(size_t)blockIdx.x * E + e];
        s_off[e] = offsets[e];
#pragma unroll
        for (int wv = 0; wv < kWarps; ++wv) s_mask[wv][e] = 0u;
    }
    __syncthreads();

    const int t = blockIdx.x * kChunk + warp * 32 + lane;
    const bool active = t < T;
    const int32_t* my_ids = ids + (size_t)t * k;
    if (active)
        for (int j = 0; j < k; ++j) atomicOr(&s_mask[warp][my_ids[j]], 1u << lane);
    __syncthreads();

    if (active) {
        const uint32_t lower = (1u << lane) - 1u;
        for (int j = 0; j < k; ++j) {
            const int e = my_ids[j];
            int32_t p = s_base[e] + __popc(s_mask[warp][e] & lower);
            for (int wv = 0; wv < warp; ++wv) p += __popc(s_mask[wv][e]);
            const int32_t s = t * k + j;
            if (capacity <= 0 || p < capacity) {
                const int32_t r = s_off[e] + p;
                slot_row[s] = r;
                row_slot[r] = s;
            } else {
                slot_row[s] = -1;
            }
        }
    }
}

static size_t align256(size_t v) { return (v + 255u) & ~size_t(255u); }

template <int L, int VPL>
static int launch_topk(int nchunks, cudaStream_t st, const float* logits, const float* bias,
                       int T, int E, int k, int32_t* ids, float* w, int32_t* hist) {
    return launch_pdl(route_topk_kernel<L, VPL>, nchunks, topk_threads<VPL>(), 0, st, logits, bias,
                      T, E, k, ids, w, hist);
}

// The three launches of one routing call; `scratch` is 256-byte aligned and
// holds at least route_scratch_bytes(T, E).
static size_t route_scratch_bytes(int T, int E) {
    const size_t nchunks = ((size_t)T + kChunk - 1) / kChunk;
    return 2 * align256(nchunks * (size_t)E * sizeof(int32_t));
}

static int launch_route(const float* logits, const float* bias, int T, int E, int k, int capacity,
                        int32_t* ids, float* w, int32_t* counts, int32_t* kept, int32_t* offsets,
                        int32_t* slot_row, int32_t* row_slot, int32_t* n_dropped, char* scratch,
                        cudaStream_t st) {
    const int nchunks = (T + kChunk - 1) / kChunk;
    int32_t* hist = reinterpret_cast<int32_t*>(scratch);
    int32_t* base = reinterpret_cast<int32_t*>(scratch + align256((size_t)nchunks * E * 4));
    if (T > 0) {
        int rc;
        if (E <= 8) rc = launch_topk<8, 1>(nchunks, st, logits, bias, T, E, k, ids, w, hist);
        else if (E <= 16) rc = launch_topk<16, 1>(nchunks, st, logits, bias, T, E, k, ids, w, hist);
        else if (E <= 32) rc = launch_topk<32, 1>(nchunks, st, logits, bias, T, E, k, ids, w, hist);
        else if (E <= 64) rc = launch_topk<32, 2>(nchunks, st, logits, bias, T, E, k, ids, w, hist);
        else if (E <= 128) rc = launch_topk<32, 4>(nchunks, st, logits, bias, T, E, k, ids, w, hist);
        else if (E <= 256) rc = launch_topk<32, 8>(nchunks, st, logits, bias, T, E, k, ids, w, hist);
        else if (E <= 512) rc = launch_topk<32, 16>(nchunks, st, logits, bias, T, E, k, ids, w, hist);
        else rc = launch_topk<32, 32>(nchunks, st, logits, bias, T, E, k, ids, w, hist);
        if (rc != MOE_OK) return MOE_ERR_CUDA;
    }
    if (launch_pdl(route_scan_kernel, 1, kScanThreads, 0, st, (const int32_t*)hist, nchunks, T, E,
                   k, capacity, base, counts, kept, offsets, n_dropped) != MOE_OK)
        return MOE_ERR_CUDA;
    if (T > 0) {
        if (launch_pdl(route_assign_kernel, nchunks, kThreads, 0, st, (const int32_t*)ids, T, E, k,
                       capacity, (const int32_t*)base, (const int32_t*)offsets, slot_row,
                       row_slot) != MOE_OK)
            return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

static int check_route_args(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                            int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* slot_row,
                            int32_t* row_slot, int32_t* n_dropped) {
    if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > E || k > kMaxTopK)
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * k >= INT32_MAX) return MOE_ERR_INVALID_ARG;
    if (!counts || !kept || !offsets || !n_dropped) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !ids || !w || !slot_row || !row_slot)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_route_workspace_size(int T, int E, int k) {
    (void)k;
    if (T < 0 || E <= 0) return 0;
    return route_scratch_bytes(T, E) + 256;  // + slack to align the caller's pointer
}

extern "C" MOE_API int moe_route(const float* logits, const float* bias, int T, int E, int k, int capacity,
                         int32_t* ids, float* w, int32_t* counts, int32_t* kept, int32_t* offsets,
                         int32_t* slot_row, int32_t* row_slot, int32_t* n_dropped, void* workspace,
                         size_t workspace_bytes, moe_stream_t stream) {
    const int rc = check_route_args(logits, T, E, k, ids, w, counts, kept, offsets, slot_row,
                                    row_slot, n_dropped);
    if (rc != MOE_OK) return rc;
    const size_t need = moe_route_workspace_size(T, E, k);
    if (!workspace || workspace_bytes < need) return MOE_ERR_WORKSPACE;
    char* ws = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(workspace) + 255u) &
                                       ~uintptr_t(255u));
    return launch_route(logits, bias, T, E, k, capacity, ids, w, counts, kept, offsets, slot_row,
                        row_slot, n_dropped, ws, reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------------
// moe_route_noalloc: moe_route for callers that cannot allocate device memory.
//
// Some callers are not allowed to allocate on the path that runs the layer:
// serving loops with a fixed memory plan, plugins inside a host framework that
// owns every device allocation, code that must not risk the implicit device
// synchronisation cudaMalloc/cudaFree can cause.  For them the router's scratch
// (per-chunk histograms and bases) lives in a fixed device array compiled into
// this library, so the call needs nothing beyond its inputs and outputs.
//
// The array below is a host-side placeholder symbol in host code, not a device
// address.  Its device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, the first time the entry
// point runs there; that first call should therefore happen before any stream
// capture.  Every call shares the one array: two calls whose kernels overlap on
// the device (different streams, or different host threads) race on it and
// must be serialised by the caller.  The router's kernels overwrite every
// scratch word they read, so nothing has to be cleared between calls.
namespace moe {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB on every device
static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

static void* noalloc_scratch_ptr() {
    constexpr int kMaxDevices = 64;
    static void* cache[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) return nullptr;
        cache[dev] = p;
    }
    return cache[dev];
}

}  // namespace moe

extern "C" MOE_API int moe_route_noalloc(const float* logits, const float* bias, int T, int E, int k,
                                 int capacity, int32_t* ids, float* w, int32_t* counts,
                                 int32_t* kept, int32_t* offsets, int32_t* slot_row,
                                 int32_t* row_slot, int32_t* n_dropped, moe_stream_t stream) {
    const int rc = check_route_args(logits, T, E, k, ids, w, counts, kept, offsets, slot_row,
                                    row_slot, n_dropped);
    if (rc != MOE_OK) return rc;
    // The fixed scratch bounds the problem size.
    if (moe_route_workspace_size(T, E, k) > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
    void* scratch = noalloc_scratch_ptr();
    if (!scratch) return MOE_ERR_CUDA;
    return launch_route(logits, bias, T, E, k, capacity, ids, w, counts, kept, offsets, slot_row,
                        row_slot, n_dropped, static_cast<char*>(scratch),
                        reinterpret_cast<cudaStream_t>(stream));
}
