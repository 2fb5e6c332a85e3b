// route.cu -- moe_route: top-k softmax gate with GShard expert capacity.
//
// "A Survey on Mixture of Experts", section 5 (gate routing; tokens dispatched
// under an expert-capacity limit) and PopFetcher, section 2.1.2 (top-k gate).
//
// Ranking: z = logit + bias (one fp32 add) is mapped to a 32-bit key whose
// unsigned order is the order (z desc): -0.0 is folded onto +0.0 (they tie),
// and every NaN gets the largest key (a NaN ranks above every number, as in
// torch.topk), so each of the k rounds picks an expert in [0, E) whatever the
// input.  Equal keys go to the lower expert index.
//
// Three launches, no inter-CTA waiting (chunks of 128 tokens, or 64 / 32 when
// that gives too few chunks to fill the GPU):
//   K1 route_topk    one CTA per chunk.  E <= 32: one token per thread; the
//                    row's keys sit in registers (16-byte loads when E % 4 == 0)
//                    and k passes of an unrolled max pick the experts.  E > 32:
//                    one token per warp, lane l holding experts
//                    (i / V) * 32V + l * V + i % V (V-wide vector loads), with
//                    the next tokens' logits loaded while the current ones are
//                    ranked; a lane sorts its candidates once (up to 8 of them),
//                    then per round the largest head key by a warp reduction,
//                    the lowest index among the lanes holding it, and the owner
//                    pops its head.  Weights
//                    w_j = exp(z_j - z_0) / sum_i exp(z_i - z_0), the sum in rank
//                    order.  Per-chunk expert histogram in shared memory
//                    (atomicAdd on counts commutes: the result is order-free).
//   K2 route_scan    one CTA per 32 experts: per expert, the exclusive prefix of
//                    the chunk histograms over chunks (32 warps each sum a
//                    segment of chunks, then the segments are scanned), counts,
//                    kept = min(counts, capacity).
//   K3 route_assign  one CTA per chunk (a token per thread); offsets = exclusive
//                    scan of kept (every CTA scans the E values itself; CTA 0
//                    writes offsets and n_dropped); a slot's position inside its
//                    expert = chunk base + slots of earlier warps of the chunk
//                    + earlier lanes of its warp, all from per-warp lane masks
//                    (atomicOr commutes; popc of the lower-lane bits gives the
//                    token-order rank).  Position < capacity -> row, else -1.
#include <climits>

#include "common.cuh"

namespace moe {

constexpr int kMaxChunk = 128;        // tokens per chunk at most (= per CTA in K1 and K3)
constexpr int kMaxWarps = kMaxChunk / 32;
constexpr int kChunkTarget = 296;     // chunks wanted: two per SM of a 148-SM B200

// Tokens per chunk: 128, or 64 / 32 when 128 would leave fewer than
// kChunkTarget chunks, so that smaller batches still spread over the GPU.  A
// function of T alone (the workspace size depends on it).
static int chunk_tokens(int T) {
    if ((T + 127) / 128 >= kChunkTarget) return 128;
    if ((T + 63) / 64 >= kChunkTarget) return 64;
    return 32;
}
constexpr int kScanThreads = 1024;

// K1 threads for E > 32: 8 warps of 16 tokens; 4 warps of 32 tokens when a
// lane holds 16 or more keys (register budget).
template <int VPL>
constexpr int warp_topk_threads() { return VPL >= 16 ? 128 : 256; }
// CTAs per SM the register budget is held to (four: every chunk of the
// largest batches resident in one wave).
template <int VPL>
constexpr int warp_topk_min_blocks() { return VPL <= 4 ? 4 : (VPL <= 8 ? 3 : 1); }

// Order key of z: larger z -> larger key; -0.0 ties with +0.0; NaN above all.
// Keys of numbers are >= 0x007FFFFF (that of -inf), so 0 is free as "none".
__device__ __forceinline__ uint32_t route_key(float z) {
    if (z != z) return 0xFFFFFFFFu;
    const uint32_t u = __float_as_uint(z == 0.0f ? 0.0f : z);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// ------------------------------------------------------------------- K1 ----
// E <= EMAX <= 32: one token per thread.  KMAX >= k bounds the unrolled
// rounds; vw (1, 2 or 4) is the load width (the host checks E % vw == 0 and the
// alignment of `logits`).
template <int EMAX, int KMAX>
__global__ void __launch_bounds__(kMaxChunk)
route_topk_lane_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T,
                       int E, int k, int vw, int ch, int32_t* __restrict__ ids,
                       float* __restrict__ w, int32_t* __restrict__ chunk_hist, int32_t* err) {
    __shared__ int s_hist[EMAX];
    __shared__ float s_bias[EMAX];
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x < EMAX) {
        s_hist[threadIdx.x] = 0;
        s_bias[threadIdx.x] =
            (bias != nullptr && (int)threadIdx.x < E) ? bias[threadIdx.x] : 0.0f;
    }
    __syncthreads();
    const int t = blockIdx.x * ch + threadIdx.x;  // blockDim.x == ch
    if (t < T) {
        const float* row = logits + (size_t)t * E;
        float z[EMAX];
        if (vw == 4) {
#pragma unroll
            for (int q = 0; q < EMAX / 4; ++q) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (4 * q < E) v = __ldg(reinterpret_cast<const float4*>(row) + q);
                z[4 * q] = v.x; z[4 * q + 1] = v.y; z[4 * q + 2] = v.z; z[4 * q + 3] = v.w;
            }
        } else if (vw == 2) {
#pragma unroll
            for (int q = 0; q < EMAX / 2; ++q) {
                float2 v = make_float2(0.f, 0.f);
                if (2 * q < E) v = __ldg(reinterpret_cast<const float2*>(row) + q);
                z[2 * q] = v.x; z[2 * q + 1] = v.y;
            }
        } else {
#pragma unroll
            for (int e = 0; e < EMAX; ++e) z[e] = (e < E) ? __ldg(row + e) : 0.0f;
        }
        uint32_t key[EMAX];
#pragma unroll
        for (int e = 0; e < EMAX; ++e) key[e] = (e < E) ? route_key(__fadd_rn(z[e], s_bias[e])) : 0u;

        int si[KMAX];
        float ex[KMAX];
        float z0 = 0.0f, s = 0.0f;
#pragma unroll
        for (int r = 0; r < KMAX; ++r) {
            si[r] = 0;
            ex[r] = 0.0f;
            if (r < k) {
                // strict '>' scanning upward: equal keys keep the lower index
                uint32_t bk = 0u;
                int bi = 0;
#pragma unroll
                for (int e = 0; e < EMAX; ++e)
                    if (key[e] > bk) {
                        bk = key[e];
                        bi = e;
                    }
#pragma unroll
                for (int e = 0; e < EMAX; ++e)
                    if (e == bi) key[e] = 0u;
                const float zr = key_value(bk);
                if (r == 0) z0 = zr;
                si[r] = bi;
                ex[r] = expf(__fsub_rn(zr, z0));
                s = __fadd_rn(s, ex[r]);
            }
        }
#pragma unroll
        for (int r = 0; r < KMAX; ++r) {
            if (r < k) {
                ids[(size_t)t * k + r] = si[r];
                w[(size_t)t * k + r] = __fdiv_rn(ex[r], s);
                if (si[r] < E) atomicAdd(&s_hist[si[r]], 1);
                else flag_error(err, MOE_DEVERR_EXPERT_INDEX);
            }
        }
    }
    __syncthreads();
    if ((int)threadIdx.x < E) chunk_hist[(size_t)blockIdx.x * E + threadIdx.x] = s_hist[threadIdx.x];
}

// E > 32: one token per warp; each lane holds VPL keys, loaded VW floats at a
// time: slot i of lane l is expert (i / VW) * 32 * VW + l * VW + i % VW, which
// grows with i, so a lane's strict '>' scan keeps the lowest index of a tie.
// Sorts VPL (key, expert) pairs into (key desc, expert asc) order with a
// fixed comparator network (Batcher's for 8, the optimal one for 4).
__device__ __forceinline__ void cas_desc(uint32_t& ka, int& ea, uint32_t& kb, int& eb) {
    const bool sw = kb > ka || (kb == ka && eb < ea);
    const uint32_t k0 = sw ? kb : ka, k1 = sw ? ka : kb;
    const int e0 = sw ? eb : ea, e1 = sw ? ea : eb;
    ka = k0; kb = k1; ea = e0; eb = e1;
}
template <int VPL>
__device__ __forceinline__ void sort_desc(uint32_t (&k)[VPL], int (&e)[VPL]) {
    if constexpr (VPL == 2) {
        cas_desc(k[0], e[0], k[1], e[1]);
    } else if constexpr (VPL == 4) {
        constexpr int net[5][2] = {{0, 1}, {2, 3}, {0, 2}, {1, 3}, {1, 2}};
#pragma unroll
        for (int c = 0; c < 5; ++c) cas_desc(k[net[c][0]], e[net[c][0]], k[net[c][1]], e[net[c][1]]);
    } else if constexpr (VPL == 8) {
        constexpr int net[19][2] = {{0, 1}, {2, 3}, {4, 5}, {6, 7}, {0, 2}, {1, 3}, {4, 6},
                                    {5, 7}, {1, 2}, {5, 6}, {0, 4}, {1, 5}, {2, 6}, {3, 7},
                                    {2, 4}, {3, 5}, {1, 2}, {3, 4}, {5, 6}};
#pragma unroll
        for (int c = 0; c < 19; ++c) cas_desc(k[net[c][0]], e[net[c][0]], k[net[c][1]], e[net[c][1]]);
    }
}

template <int VPL, int VW>
__device__ __forceinline__ void load_lane(const float* __restrict__ row, int lane_vw, int E,
                                          float (&v)[VPL]) {
#pragma unroll
    for (int g = 0; g < VPL / VW; ++g) {
        const int e = g * 32 * VW + lane_vw;
        if constexpr (VW == 4) {
            float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
            if (e < E) q = __ldg(reinterpret_cast<const float4*>(row + e));
            v[4 * g] = q.x; v[4 * g + 1] = q.y; v[4 * g + 2] = q.z; v[4 * g + 3] = q.w;
        } else if constexpr (VW == 2) {
            float2 q = make_float2(0.f, 0.f);
            if (e < E) q = __ldg(reinterpret_cast<const float2*>(row + e));
            v[2 * g] = q.x; v[2 * g + 1] = q.y;
        } else {
            v[g] = (e < E) ? __ldg(row + e) : 0.0f;
        }
    }
}

template <int VPL, int VW>
__global__ void __launch_bounds__(warp_topk_threads<VPL>(), warp_topk_min_blocks<VPL>())
route_topk_warp_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T,
                       int E, int k, int ch, int32_t* __restrict__ ids, float* __restrict__ w,
                       int32_t* __restrict__ chunk_hist, int32_t* err) {
    constexpr int kT = warp_topk_threads<VPL>();
    const int per_warp = ch / (kT / 32);                   // tokens per warp (>= 4)
    constexpr int D = VPL <= 4 ? 4 : (VPL <= 8 ? 2 : 1);  // tokens in flight per warp
    static_assert(32 / (warp_topk_threads<VPL>() / 32) % D == 0, "token groups");
    constexpr int kMaxPerWarp = kMaxChunk / (kT / 32);
    __shared__ int s_hist[kMaxExperts];
    // per warp, per token of the warp: the k selected keys' values and experts
    // (written in the selection rounds, read back one token per lane; rows of
    // kp = k | 1 words, so the lanes' reads fall in distinct banks)
    __shared__ float s_z[kT / 32][kMaxPerWarp * (kMaxTopK + 1)];
    __shared__ int32_t s_id[kT / 32][kMaxPerWarp * (kMaxTopK + 1)];
    const int kp = k | 1;
    pdl_wait();
    pdl_trigger();
    for (int e = threadIdx.x; e < E; e += kT) s_hist[e] = 0;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int lane_vw = lane * VW;
    float b[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = (i / VW) * 32 * VW + lane_vw + i % VW;
        b[i] = (bias != nullptr && e < E) ? __ldg(bias + e) : 0.0f;
    }
    __syncthreads();

    const int t_warp = blockIdx.x * ch + warp * per_warp;
    float cur[D][VPL], nxt[D][VPL];
#pragma unroll
    for (int u = 0; u < D; ++u) {
        const int t = t_warp + u;
        if (t < T) load_lane<VPL, VW>(logits + (size_t)t * E, lane_vw, E, cur[u]);
    }
#pragma unroll 1
    for (int g = 0; g < per_warp / D; ++g) {
        if (g + 1 < per_warp / D) {
#pragma unroll
            for (int u = 0; u < D; ++u) {
                const int t = t_warp + (g + 1) * D + u;
                if (t < T) load_lane<VPL, VW>(logits + (size_t)t * E, lane_vw, E, nxt[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < D; ++u) {
            const int t = t_warp + g * D + u;
            if (t < T) {  // warp-uniform
                uint32_t key[VPL];
                int ex_i[VPL];  // expert of each slot
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int e = (i / VW) * 32 * VW + lane_vw + i % VW;
                    ex_i[i] = e;
                    key[i] = (e < E) ? route_key(__fadd_rn(cur[u][i], b[i])) : 0u;
                }
                const int tw = g * D + u;  // token index within the warp
                float* zrow = s_z[warp] + tw * kp;
                int32_t* idrow = s_id[warp] + tw * kp;
                if constexpr (VPL <= 8) {
                    // the lane's candidates sorted once, (key desc, expert asc); a
                    // round takes the best head of the warp and its owner pops it
                    sort_desc<VPL>(key, ex_i);
                    for (int r = 0; r < k; ++r) {
                        // k <= E, so some lane still holds an untaken expert: m > 0
                        const uint32_t m = __reduce_max_sync(0xffffffffu, key[0]);
                        const int win = (int)__reduce_min_sync(
                            0xffffffffu, key[0] == m ? (uint32_t)ex_i[0] : 0xffffffffu);
                        if (ex_i[0] == win) {
#pragma unroll
                            for (int i = 0; i + 1 < VPL; ++i) {
                                key[i] = key[i + 1];
                                ex_i[i] = ex_i[i + 1];
                            }
                            key[VPL - 1] = 0u;
                            ex_i[VPL - 1] = INT_MAX;
                        }
                        if (lane == 0) {
                            zrow[r] = key_value(m);
                            idrow[r] = win;
                        }
                    }
                } else {
                    for (int r = 0; r < k; ++r) {
                        uint32_t bk = 0u;
                        int bi = INT_MAX;
#pragma unroll
                        for (int i = 0; i < VPL; ++i)
                            if (key[i] > bk) {
                                bk = key[i];
                                bi = ex_i[i];
                            }
                        const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
                        const int win = (int)__reduce_min_sync(
                            0xffffffffu, bk == m ? (uint32_t)bi : 0xffffffffu);
#pragma unroll
                        for (int i = 0; i < VPL; ++i)
                            if (ex_i[i] == win) key[i] = 0u;
                        if (lane == 0) {
                            zrow[r] = key_value(m);
                            idrow[r] = win;
                        }
                    }
                }
            }
        }
        if (g + 1 < per_warp / D) {
#pragma unroll
            for (int u = 0; u < D; ++u)
#pragma unroll
                for (int i = 0; i < VPL; ++i) cur[u][i] = nxt[u][i];
        }
    }
    __syncwarp();
    // lane j finishes the warp's token j: w_j = exp(z_j - z_0) / sum_i exp(z_i - z_0)
    // (sum in rank order), the k ids and weights stored contiguously
    {
        const int t = t_warp + lane;
        if (lane < per_warp && t < T) {
            const float* zrow = s_z[warp] + lane * kp;
            const int32_t* idrow = s_id[warp] + lane * kp;
            const float z0 = zrow[0];
            float sum = 0.0f;
            for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, expf(__fsub_rn(zrow[j], z0)));
            for (int j = 0; j < k; ++j) {
                const int e = idrow[j];
                ids[(size_t)t * k + j] = e;
                w[(size_t)t * k + j] = __fdiv_rn(expf(__fsub_rn(zrow[j], z0)), sum);
                if ((unsigned)e < (unsigned)E) atomicAdd(&s_hist[e], 1);
                else flag_error(err, MOE_DEVERR_EXPERT_INDEX);
            }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kT)
        chunk_hist[(size_t)blockIdx.x * E + e] = s_hist[e];
}

// ------------------------------------------------------------------- K2 ----
// One CTA per 32 experts (lane = expert); warp s sums chunks
// [s * cps, (s + 1) * cps), the 32 segment totals are scanned per expert, and
// each warp rescans its segment to write the chunk bases.
__global__ void __launch_bounds__(kScanThreads)
route_scan_kernel(const int32_t* __restrict__ chunk_hist, int nchunks, int E, int capacity,
                  int32_t* __restrict__ chunk_base, int32_t* __restrict__ counts,
                  int32_t* __restrict__ kept) {
    __shared__ int32_t s_seg[32][33];
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int e = blockIdx.x * 32 + lane;
    const bool ok = e < E;
    const int cps = (nchunks + 31) / 32;
    const int c0 = wid * cps, c1 = min(nchunks, c0 + cps);
    int32_t part = 0;
    if (ok) {
#pragma unroll 4
        for (int c = c0; c < c1; ++c) part += chunk_hist[(size_t)c * E + e];
    }
    s_seg[wid][lane] = part;
    __syncthreads();
    if (wid == 0) {
        int32_t run = 0;
        for (int s = 0; s < 32; ++s) {
            const int32_t v = s_seg[s][lane];
            s_seg[s][lane] = run;
            run += v;
        }
        if (ok) {
            counts[e] = run;
            kept[e] = (capacity > 0 && run > capacity) ? capacity : run;
        }
    }
    __syncthreads();
    if (ok) {
        int32_t run = s_seg[wid][lane];
#pragma unroll 4
        for (int c = c0; c < c1; ++c) {
            const int32_t v = chunk_hist[(size_t)c * E + e];
            chunk_base[(size_t)c * E + e] = run;
            run += v;
        }
    }
}

// ------------------------------------------------------------------- K3 ----
__global__ void __launch_bounds__(kMaxChunk)
route_assign_kernel(const int32_t* __restrict__ ids, int T, int E, int k, int capacity,
                    int ch, int nchunks, const int32_t* __restrict__ chunk_base,
                    const int32_t* __restrict__ kept, int32_t* __restrict__ offsets,
                    int32_t* __restrict__ n_dropped, int32_t* __restrict__ slot_row,
                    int32_t* __restrict__ row_slot, int32_t* err) {
    __shared__ uint32_t s_mask[kMaxWarps][kMaxExperts];
    __shared__ int32_t s_base[kMaxExperts];
    __shared__ int32_t s_off[kMaxExperts + 1];
    __shared__ int32_t s_warp[kMaxWarps];
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthr = blockDim.x, nwarps = nthr >> 5;  // blockDim.x == ch

    // offsets: exclusive scan of kept over the experts, per = experts a thread holds
    const int per = (E + nthr - 1) / nthr;
    const int e0 = tid * per;
    int32_t loc = 0;
    for (int i = 0; i < per; ++i)
        if (e0 + i < E) loc += kept[e0 + i];
    int32_t incl = loc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp[warp] = incl;
    for (int e = tid; e < E; e += nthr) {
        s_base[e] = blockIdx.x < nchunks ? chunk_base[(size_t)blockIdx.x * E + e] : 0;
#pragma unroll
        for (int wv = 0; wv < kMaxWarps; ++wv) s_mask[wv][e] = 0u;
    }
    __syncthreads();
    int32_t run = incl - loc;
    int32_t total = 0;
    for (int wv = 0; wv < nwarps; ++wv) {
        if (wv < warp) run += s_warp[wv];
        total += s_warp[wv];
    }
    for (int i = 0; i < per; ++i)
        if (e0 + i < E) {
            s_off[e0 + i] = run;
            run += kept[e0 + i];
        }
    if (tid == 0) s_off[E] = total;
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int e = tid; e <= E; e += nthr) offsets[e] = s_off[e];
        if (tid == 0) n_dropped[0] = (int32_t)((int64_t)T * k - total);
    }

    const int t = blockIdx.x * ch + tid;
    const bool active = t < T;
    const int32_t* my_ids = ids + (size_t)t * k;
    if (active)
        for (int j = 0; j < k; ++j) {
            const int e = my_ids[j];
            if ((unsigned)e < (unsigned)E) atomicOr(&s_mask[warp][e], 1u << lane);
        }
    __syncthreads();

    if (active) {
        const uint32_t lower = (1u << lane) - 1u;
        for (int j = 0; j < k; ++j) {
            const int e = my_ids[j];
            const int32_t s = t * k + j;
            if ((unsigned)e >= (unsigned)E) {
                flag_error(err, MOE_DEVERR_EXPERT_INDEX);
                slot_row[s] = -1;
                continue;
            }
            int32_t p = s_base[e] + __popc(s_mask[warp][e] & lower);
            for (int wv = 0; wv < warp; ++wv) p += __popc(s_mask[wv][e]);
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

template <int EMAX, int KMAX>
static int launch_lane(int nchunks, int ch, cudaStream_t st, const float* logits,
                       const float* bias, int T, int E, int k, int vw, int32_t* ids, float* w,
                       int32_t* hist) {
    return launch_pdl(route_topk_lane_kernel<EMAX, KMAX>, nchunks, ch, 0, st, logits, bias, T, E,
                      k, vw, ch, ids, w, hist, device_error_word());
}
template <int EMAX>
static int launch_lane_k(int nchunks, int ch, cudaStream_t st, const float* logits,
                         const float* bias, int T, int E, int k, int vw, int32_t* ids, float* w,
                         int32_t* hist) {
    if (k <= 2)
        return launch_lane<EMAX, 2>(nchunks, ch, st, logits, bias, T, E, k, vw, ids, w, hist);
    if (k <= 8)
        return launch_lane<EMAX, 8>(nchunks, ch, st, logits, bias, T, E, k, vw, ids, w, hist);
    return launch_lane<EMAX, EMAX>(nchunks, ch, st, logits, bias, T, E, k, vw, ids, w, hist);
}
template <int VPL>
static int launch_warp(int nchunks, int ch, cudaStream_t st, const float* logits,
                       const float* bias, int T, int E, int k, bool vec, int32_t* ids, float* w,
                       int32_t* hist) {
    constexpr int VW = VPL >= 4 ? 4 : VPL;
    if (vec)
        return launch_pdl(route_topk_warp_kernel<VPL, VW>, nchunks, warp_topk_threads<VPL>(), 0,
                          st, logits, bias, T, E, k, ch, ids, w, hist, device_error_word());
    return launch_pdl(route_topk_warp_kernel<VPL, 1>, nchunks, warp_topk_threads<VPL>(), 0, st,
                      logits, bias, T, E, k, ch, ids, w, hist, device_error_word());
}

// The three launches of one routing call in chunks of ch tokens; `scratch` is
// 256-byte aligned and holds at least route_scratch_bytes(T, E, ch).
static size_t route_scratch_bytes(int T, int E, int ch) {
    const size_t nchunks = ((size_t)T + ch - 1) / ch;
    return 2 * align256(nchunks * (size_t)E * sizeof(int32_t));
}

static int launch_route(const float* logits, const float* bias, int T, int E, int k, int capacity,
                        int32_t* ids, float* w, int32_t* counts, int32_t* kept, int32_t* offsets,
                        int32_t* slot_row, int32_t* row_slot, int32_t* n_dropped, char* scratch,
                        int ch, cudaStream_t st) {
    const int nchunks = (T + ch - 1) / ch;
    int32_t* hist = reinterpret_cast<int32_t*>(scratch);
    int32_t* base = reinterpret_cast<int32_t*>(scratch + align256((size_t)nchunks * E * 4));
    if (T > 0) {
        // widest load the row layout and the pointer's alignment allow
        const uintptr_t p = reinterpret_cast<uintptr_t>(logits);
        const int vw = (E % 4 == 0 && p % 16 == 0) ? 4 : (E % 2 == 0 && p % 8 == 0) ? 2 : 1;
        const int n = nchunks;
        int rc;
        if (E <= 8) rc = launch_lane_k<8>(n, ch, st, logits, bias, T, E, k, vw, ids, w, hist);
        else if (E <= 16) rc = launch_lane_k<16>(n, ch, st, logits, bias, T, E, k, vw, ids, w, hist);
        else if (E <= 32) rc = launch_lane_k<32>(n, ch, st, logits, bias, T, E, k, vw, ids, w, hist);
        else if (E <= 64) rc = launch_warp<2>(n, ch, st, logits, bias, T, E, k, vw >= 2, ids, w, hist);
        else if (E <= 128) rc = launch_warp<4>(n, ch, st, logits, bias, T, E, k, vw == 4, ids, w, hist);
        else if (E <= 256) rc = launch_warp<8>(n, ch, st, logits, bias, T, E, k, vw == 4, ids, w, hist);
        else if (E <= 512) rc = launch_warp<16>(n, ch, st, logits, bias, T, E, k, vw == 4, ids, w, hist);
        else rc = launch_warp<32>(n, ch, st, logits, bias, T, E, k, vw == 4, ids, w, hist);
        if (rc != MOE_OK) return MOE_ERR_CUDA;
    }
    if (launch_pdl(route_scan_kernel, (E + 31) / 32, kScanThreads, 0, st, (const int32_t*)hist,
                   nchunks, E, capacity, base, counts, kept) != MOE_OK)
        return MOE_ERR_CUDA;
    // at least one CTA: it writes offsets and n_dropped even when T = 0
    if (launch_pdl(route_assign_kernel, nchunks > 0 ? nchunks : 1, ch, 0, st, (const int32_t*)ids,
                   T, E, k, capacity, ch, nchunks, (const int32_t*)base, (const int32_t*)kept,
                   offsets, n_dropped, slot_row, row_slot, device_error_word()) != MOE_OK)
        return MOE_ERR_CUDA;
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
    return route_scratch_bytes(T, E, chunk_tokens(T)) + 256;  // + slack to align the pointer
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
                        row_slot, n_dropped, ws, chunk_tokens(T),
                        reinterpret_cast<cudaStream_t>(stream));
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

// Device address of the array on the current device, looked up once per device
// (host threads that race on the first lookup store the same address).
static void* noalloc_scratch_ptr() {
    static std::atomic<void*> cache[kMaxDevices] = {};
    const int dev = current_device();
    if (dev < 0) return nullptr;
    void* p = cache[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) return nullptr;
        cache[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace moe

extern "C" MOE_API int moe_route_noalloc(const float* logits, const float* bias, int T, int E, int k,
                                 int capacity, int32_t* ids, float* w, int32_t* counts,
                                 int32_t* kept, int32_t* offsets, int32_t* slot_row,
                                 int32_t* row_slot, int32_t* n_dropped, moe_stream_t stream) {
    const int rc = check_route_args(logits, T, E, k, ids, w, counts, kept, offsets, slot_row,
                                    row_slot, n_dropped);
    if (rc != MOE_OK) return rc;
    // The fixed scratch bounds the problem size (128-token chunks whatever T).
    if (route_scratch_bytes(T, E, kMaxChunk) + 256 > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
    void* scratch = noalloc_scratch_ptr();
    if (!scratch) return MOE_ERR_CUDA;
    return launch_route(logits, bias, T, E, k, capacity, ids, w, counts, kept, offsets, slot_row,
                        row_slot, n_dropped, static_cast<char*>(scratch), kMaxChunk,
                        reinterpret_cast<cudaStream_t>(stream));
}
