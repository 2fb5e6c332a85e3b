// bwd.cu -- backward pass of the MoE layer: output decode, expert computation,
// gate routing and gate projection (input encode's backward is in permute.cu).
//
// PopFetcher, section 5.2.1: every expert GEMM of the forward pass has two in
// the backward pass, one for the input and one for the weights; the other
// steps are the adjoints of the forward gathers, scatters and the softmax.
//
// moe_combine_backward: one warp per token, kept slots j ascending:
//   dw[t][j] = <dy[t], Yp[row]> (fp32 lanes, fixed butterfly), and
//   dYp[row] = w[t][j] * dy[t] (the product taken exactly in double and
//   rounded once to the row's type).  HBM-bound: dy is read once per slot
//   (k times, from L1/L2 after the first), Yp read and dYp written once.
// moe_route_backward: a lane per token; the renormalised softmax over the
//   token's selected experts gives dz_j = w_j (dw_j - sum_i w_i dw_i), taken
//   in double with every operation rounded separately and i ascending, then
//   rounded once to fp32; dlogits is dense [T][E] (zero off the selection).
//   dbias = column sums of dlogits: per 256-token chunk in double (fixed
//   slices of tokens, then the slices), then over chunks ascending --
//   deterministic.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdChunk = 256;  // tokens per CTA in the routing backward

template <int DT> struct Row;
template <> struct Row<MOE_DTYPE_BF16> {
    __device__ static float dot(const uint4& a, const uint4& b, float acc) {
        const uint32_t ua[4] = {a.x, a.y, a.z, a.w}, ub[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc = fmaf(bf16lo(ua[i]), bf16lo(ub[i]), acc);
            acc = fmaf(bf16hi(ua[i]), bf16hi(ub[i]), acc);
        }
        return acc;
    }
    __device__ static uint32_t scale2(uint32_t u, double w) {
        const __nv_bfloat16 lo = __double2bfloat16(__dmul_rn(w, (double)bf16lo(u)));
        const __nv_bfloat16 hi = __double2bfloat16(__dmul_rn(w, (double)bf16hi(u)));
        return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
    }
    __device__ static uint4 scale(const uint4& v, float w) {
        const double wd = (double)w;
        return make_uint4(scale2(v.x, wd), scale2(v.y, wd), scale2(v.z, wd), scale2(v.w, wd));
    }
};
template <> struct Row<MOE_DTYPE_F32> {
    __device__ static float dot(const uint4& a, const uint4& b, float acc) {
        acc = fmaf(__uint_as_float(a.x), __uint_as_float(b.x), acc);
        acc = fmaf(__uint_as_float(a.y), __uint_as_float(b.y), acc);
        acc = fmaf(__uint_as_float(a.z), __uint_as_float(b.z), acc);
        acc = fmaf(__uint_as_float(a.w), __uint_as_float(b.w), acc);
        return acc;
    }
    __device__ static uint4 scale(const uint4& v, float w) {  // fp32 product: one rounding
        return make_uint4(__float_as_uint(__fmul_rn(w, __uint_as_float(v.x))),
                          __float_as_uint(__fmul_rn(w, __uint_as_float(v.y))),
                          __float_as_uint(__fmul_rn(w, __uint_as_float(v.z))),
                          __float_as_uint(__fmul_rn(w, __uint_as_float(v.w))));
    }
};

template <int DT>
__global__ void __launch_bounds__(kBwdThreads)
combine_backward_kernel(const uint4* __restrict__ dy, const uint4* __restrict__ Yp, int T, int nvec,
                        int k, const int32_t* __restrict__ slot_row, const float* __restrict__ w,
                        float* __restrict__ dw, uint4* __restrict__ dYp, int R_max, int32_t* err) {
    using R = Row<DT>;
    constexpr int U = 4;  // vectors per lane in flight
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int wpb = kBwdThreads / 32;
    const int nwarps = gridDim.x * wpb;
    for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += nwarps) {
        int my_row = -1;
        float my_w = 0.0f;
        if (lane < k) {
            my_row = __ldg(slot_row + (size_t)t * k + lane);
            my_w = __ldg(w + (size_t)t * k + lane);
            if (my_row < -1 || my_row >= R_max) {
                flag_error(err, MOE_DEVERR_ROW_INDEX);
                my_row = -1;
            }
        }
        const uint4* g = dy + (size_t)t * nvec;
        for (int j = 0; j < k; ++j) {
            const int row = __shfl_sync(0xffffffffu, my_row, j);
            const float wj = __shfl_sync(0xffffffffu, my_w, j);
            float dot = 0.0f;
            if (row >= 0) {
                const uint4* y = Yp + (size_t)row * nvec;
                uint4* o = dYp + (size_t)row * nvec;
                for (int c0 = 0; c0 < nvec; c0 += 32 * U) {
                    uint4 gv[U], yv[U];
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int c = c0 + u * 32 + lane;
                        gv[u] = c < nvec ? __ldg(g + c) : make_uint4(0, 0, 0, 0);
                        yv[u] = c < nvec ? ldg_nc_v4(y + c) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int c = c0 + u * 32 + lane;
                        dot = R::dot(gv[u], yv[u], dot);
                        if (c < nvec) stg_v4(o + c, R::scale(gv[u], wj));
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    dot = __fadd_rn(dot, __shfl_xor_sync(0xffffffffu, dot, off));
            }
            if (lane == 0) dw[(size_t)t * k + j] = dot;  // dropped slot: 0
        }
    }
}

// k <= KMAX <= 4: one pass over the row's columns instead of one per slot.  Per
// block of 32*U vectors the token's dy block is loaded once and the blocks of
// all its kept rows of Yp are loaded before the first multiply-add (KMAX*U
// vectors per lane in flight); each slot keeps its own partial dot product,
// summed over the lanes at the end.
template <int DT, int KMAX, int U>
__global__ void __launch_bounds__(kBwdThreads)
combine_backward_wide_kernel(const uint4* __restrict__ dy, const uint4* __restrict__ Yp, int T,
                             int nvec, int k, const int32_t* __restrict__ slot_row,
                             const float* __restrict__ w, float* __restrict__ dw,
                             uint4* __restrict__ dYp, int R_max, int32_t* err) {
    using R = Row<DT>;
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int wpb = kBwdThreads / 32;
    const int nwarps = gridDim.x * wpb;
    for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += nwarps) {
        int my_row = -1;
        float my_w = 0.0f;
        if (lane < k) {
            my_row = __ldg(slot_row + (size_t)t * k + lane);
            my_w = __ldg(w + (size_t)t * k + lane);
            if (my_row < -1 || my_row >= R_max) {
                flag_error(err, MOE_DEVERR_ROW_INDEX);
                my_row = -1;
            }
        }
        int rows[KMAX];
        float wv[KMAX], dot[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {  // lanes >= k hold -1: slots past k are skipped
            rows[j] = __shfl_sync(0xffffffffu, my_row, j);
            wv[j] = __shfl_sync(0xffffffffu, my_w, j);
            dot[j] = 0.0f;
        }
        const uint4* g = dy + (size_t)t * nvec;
        for (int c0 = 0; c0 < nvec; c0 += 32 * U) {
            uint4 gv[U], yv[KMAX][U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                gv[u] = c < nvec ? __ldg(g + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + u * 32 + lane;
                    yv[j][u] = (rows[j] >= 0 && c < nvec)
                                   ? ldg_nc_v4(Yp + (size_t)rows[j] * nvec + c)
                                   : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (rows[j] < 0) continue;
                uint4* o = dYp + (size_t)rows[j] * nvec;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + u * 32 + lane;
                    dot[j] = R::dot(gv[u], yv[j][u], dot[j]);
                    if (c < nvec) stg_v4(o + c, R::scale(gv[u], wv[j]));
                }
            }
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                dot[j] = __fadd_rn(dot[j], __shfl_xor_sync(0xffffffffu, dot[j], off));
            if (lane == 0 && j < k) dw[(size_t)t * k + j] = rows[j] >= 0 ? dot[j] : 0.0f;
        }
    }
}

// dlogits rows of one chunk of 256 tokens, then (when dbias is wanted) the
// chunk's column sums in double.  Each warp takes 32 consecutive tokens at
// once, a lane per token (the loads of all 32 tokens are in flight together):
// the warp zeroes the 32 rows (one contiguous block of 32*E floats), then each
// lane writes its token's k entries.  Column sums: S = 256 / E slices of the
// chunk's tokens per expert (E <= 256), each summed by one thread in token
// order, then the slices in order -- a fixed order for a given E.
__global__ void __launch_bounds__(kBwdThreads)
route_backward_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w,
                      const float* __restrict__ dw, int T, int E, int k,
                      float* __restrict__ dlogits, double* __restrict__ partial, int32_t* err) {
    __shared__ double s_part[kBwdThreads];
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = blockIdx.x * kBwdChunk;
    const int t1 = min(T, t0 + kBwdChunk);
    const int tw = t0 + warp * 32;  // this warp's first token
    if (tw < t1) {
        const int nt = min(32, t1 - tw);
        // zero rows [tw, tw + nt): contiguous, 16-byte vectors where aligned
        float* blk = dlogits + (size_t)tw * E;
        const size_t n = (size_t)nt * E;
        if ((reinterpret_cast<uintptr_t>(blk) & 15u) == 0) {
            const size_t nv = n / 4;
            for (size_t i = lane; i < nv; i += 32)
                reinterpret_cast<float4*>(blk)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (size_t i = nv * 4 + lane; i < n; i += 32) blk[i] = 0.0f;
        } else {
            for (size_t i = lane; i < n; i += 32) blk[i] = 0.0f;
        }
        __syncwarp();
        const int t = tw + lane;
        if (lane < nt) {
            // s = sum_i w_i dw_i, i ascending, each product and sum rounded in double
            const float* wt = w + (size_t)t * k;
            const float* gt = dw + (size_t)t * k;
            double s = 0.0;
            for (int i = 0; i < k; ++i)
                s = __dadd_rn(s, __dmul_rn((double)__ldg(wt + i), (double)__ldg(gt + i)));
            float* row = dlogits + (size_t)t * E;
            for (int j = 0; j < k; ++j) {
                const int e = __ldg(ids + (size_t)t * k + j);
                if (e < 0 || e >= E) {
                    flag_error(err, MOE_DEVERR_EXPERT_INDEX);
                    continue;
                }
                const double wj = (double)__ldg(wt + j), gj = (double)__ldg(gt + j);
                row[e] = __double2float_rn(__dmul_rn(wj, __dsub_rn(gj, s)));
            }
        }
    }
    if (!partial) return;
    __syncthreads();  // the chunk's rows are written (block-scope visibility)
    const int n_tok = t1 - t0;
    if (E <= kBwdThreads) {
        const int S = kBwdThreads / E;            // slices per expert
        const int per = (kBwdChunk + S - 1) / S;  // tokens per slice
        const int e = threadIdx.x % E, sl = threadIdx.x / E;
        double acc = 0.0;
        if (sl < S) {
            const int a = sl * per, b = min(n_tok, a + per);
#pragma unroll 4
            for (int t = a; t < b; ++t)
                acc = __dadd_rn(acc, (double)dlogits[(size_t)(t0 + t) * E + e]);
        }
        s_part[threadIdx.x] = acc;
        __syncthreads();
        if (threadIdx.x < E) {
            double v = 0.0;
            for (int q = 0; q < S; ++q) v = __dadd_rn(v, s_part[q * E + threadIdx.x]);
            partial[(size_t)blockIdx.x * E + threadIdx.x] = v;
        }
    } else {
        for (int e = threadIdx.x; e < E; e += kBwdThreads) {
            double acc = 0.0;
#pragma unroll 4
            for (int t = 0; t < n_tok; ++t)
                acc = __dadd_rn(acc, (double)dlogits[(size_t)(t0 + t) * E + e]);
            partial[(size_t)blockIdx.x * E + e] = acc;
        }
    }
}

__global__ void __launch_bounds__(kBwdThreads)
bias_grad_kernel(const double* __restrict__ partial, int nchunks, int E, float* __restrict__ dbias) {
    pdl_wait();
    pdl_trigger();
    for (int e = blockIdx.x * kBwdThreads + threadIdx.x; e < E; e += gridDim.x * kBwdThreads) {
        double acc = 0.0;
        for (int c = 0; c < nchunks; ++c) acc = __dadd_rn(acc, partial[(size_t)c * E + e]);
        dbias[e] = __double2float_rn(acc);
    }
}

int warp_grid(int T) {
    const int wpb = kBwdThreads / 32;
    const int need = (T + wpb - 1) / wpb;
    const int cap = num_sms() * 8;
    return need < cap ? need : cap;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_combine_backward(const void* dy, const void* Yp, int dtype, int T, int d,
                                            int k, const int32_t* slot_row, const float* w,
                                            float* dw, void* dYp, int R_max, moe_stream_t stream) {
    if (!dtype_ok(dtype)) return MOE_ERR_UNSUPPORTED;
    if (T < 0 || d < 1 || k < 1 || k > kMaxTopK || R_max < 0) return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * k >= INT32_MAX) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!dy || !Yp || !slot_row || !w || !dw || !dYp) return MOE_ERR_INVALID_ARG;
    if (((size_t)d * dtype_bytes(dtype)) % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (!aligned16(dy) || !aligned16(Yp) || !aligned16(dYp)) return MOE_ERR_UNSUPPORTED;
    const int nvec = (int)((size_t)d * dtype_bytes(dtype) / 16);
    auto kern = dtype == MOE_DTYPE_BF16 ? combine_backward_kernel<MOE_DTYPE_BF16>
                                        : combine_backward_kernel<MOE_DTYPE_F32>;
    // k <= 4: one pass over the columns, the slots' loads in flight together
    // (measured on one B200: 65536 tokens, d = 7168, k = 4: 1.80 -> 1.36 ms); with
    // 8 slots the per-slot passes, which reuse the dy row from L1, were faster
    // (8192 tokens, d = 4096, k = 8: 0.23 against 0.30 ms)
    if (k <= 4) {
        const bool bf = dtype == MOE_DTYPE_BF16;
        if (k <= 2)
            kern = bf ? combine_backward_wide_kernel<MOE_DTYPE_BF16, 2, 4>
                      : combine_backward_wide_kernel<MOE_DTYPE_F32, 2, 4>;
        else
            kern = bf ? combine_backward_wide_kernel<MOE_DTYPE_BF16, 4, 2>
                      : combine_backward_wide_kernel<MOE_DTYPE_F32, 4, 2>;
    }
    return launch_pdl(kern, warp_grid(T), kBwdThreads, 0, reinterpret_cast<cudaStream_t>(stream),
                      static_cast<const uint4*>(dy), static_cast<const uint4*>(Yp), T, nvec, k,
                      slot_row, w, dw, static_cast<uint4*>(dYp), R_max, device_error_word());
}

extern "C" MOE_API int moe_expert_ffn_backward(const void* Xp, const void* H, const void* dYp,
                                               const void* W1, const void* W2, int dtype, int E,
                                               int d, int F, const int32_t* offsets, int R_max,
                                               void* dH, void* dXp, float* dW1, float* dW2,
                                               moe_stream_t stream) {
    if (!dtype_ok(dtype)) return MOE_ERR_UNSUPPORTED;
    if (E < 1 || E > kMaxExperts || d < 1 || F < 1 || R_max < 0) return MOE_ERR_INVALID_ARG;
    if ((int64_t)E * d >= INT32_MAX || (int64_t)E * F >= INT32_MAX) return MOE_ERR_INVALID_ARG;
    if (R_max > 0 && (!Xp || !H || !dYp || !W1 || !W2 || !offsets || !dH || !dXp))
        return MOE_ERR_INVALID_ARG;
    const size_t es = dtype_bytes(dtype);
    if ((d * es) % 16 != 0 || (F * es) % 16 != 0) return MOE_ERR_UNSUPPORTED;
    const void* ptrs[] = {Xp, H, dYp, W1, W2, dH, dXp, dW1, dW2};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (R_max == 0) {  // no rows: zero weight gradients, nothing else to do
        for (float* g : {dW1, dW2})
            if (g && cudaMemsetAsync(g, 0, sizeof(float) * (size_t)E * d * F, st) != cudaSuccess)
                return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (dtype == MOE_DTYPE_BF16)
        return launch_ffn_backward_bf16(Xp, H, dYp, W1, W2, E, d, F, offsets, R_max, dH, dXp, dW1,
                                        dW2, st);
    return launch_ffn_backward_f32(
        static_cast<const float*>(Xp), static_cast<const float*>(H), static_cast<const float*>(dYp),
        static_cast<const float*>(W1), static_cast<const float*>(W2), E, d, F, offsets, R_max,
        static_cast<float*>(dH), static_cast<float*>(dXp), dW1, dW2, st);
}

extern "C" MOE_API int moe_route_backward(const int32_t* ids, const float* w, const float* dw,
                                          int T, int E, int k, float* dlogits, float* dbias,
                                          void* workspace, size_t workspace_bytes,
                                          moe_stream_t stream) {
    if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > kMaxTopK || k > E)
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * E >= INT32_MAX || (int64_t)T * k >= INT32_MAX) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!ids || !w || !dw || !dlogits)) return MOE_ERR_INVALID_ARG;
    if (dbias && (!workspace || workspace_bytes < moe_route_workspace_size(T, E, k)))
        return MOE_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int nchunks = (T + kBwdChunk - 1) / kBwdChunk;
    double* partial = nullptr;
    if (dbias)
        partial = reinterpret_cast<double*>((reinterpret_cast<uintptr_t>(workspace) + 255u) &
                                            ~uintptr_t(255u));
    if (T > 0) {
        const int rc = launch_pdl(route_backward_kernel, nchunks, kBwdThreads, 0, st, ids, w, dw,
                                  T, E, k, dlogits, partial, device_error_word());
        if (rc != MOE_OK) return rc;
    }
    if (!dbias) return MOE_OK;
    return launch_pdl(bias_grad_kernel, (E + kBwdThreads - 1) / kBwdThreads, kBwdThreads, 0, st,
                      static_cast<const double*>(partial), nchunks, E, dbias);
}

extern "C" MOE_API size_t moe_gate_backward_workspace_size(int T, int d, int E, int dtype) {
    if (T < 0 || d < 1 || E < 1 || !dtype_ok(dtype)) return 0;
    if (T == 0) return 0;
    if (dtype == MOE_DTYPE_BF16 && gate_backward_tc_ok(d, E))
        return gate_backward_tc_workspace(T, d, E);
    const int ks = gate_backward_splits(T, d, E);
    return ks > 1 ? (size_t)ks * E * d * sizeof(float) + 256 : 0;
}

extern "C" MOE_API int moe_gate_backward(const void* x, const void* Wg, int dtype, int T, int d,
                                         int E, const float* dlogits, void* dx, float* dWg,
                                         void* workspace, size_t workspace_bytes,
                                         moe_stream_t stream) {
    if (!dtype_ok(dtype)) return MOE_ERR_UNSUPPORTED;
    if (T < 0 || d < 1 || E < 1 || E > kMaxExperts) return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * d >= INT32_MAX || (int64_t)T * E >= INT32_MAX) return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * 3 >= INT32_MAX) return MOE_ERR_INVALID_ARG;
    if (!Wg || (T > 0 && (!x || !dlogits || !dx))) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {  // no tokens: dWg = 0
        if (!dWg) return MOE_OK;
        return cudaMemsetAsync(dWg, 0, sizeof(float) * (size_t)E * d, st) == cudaSuccess
                   ? MOE_OK
                   : MOE_ERR_CUDA;
    }
    const size_t need = moe_gate_backward_workspace_size(T, d, E, dtype);
    if (dtype == MOE_DTYPE_BF16 && gate_backward_tc_ok(d, E)) {
        if (!workspace || workspace_bytes < need) return MOE_ERR_WORKSPACE;
        if (!aligned16(x) || !aligned16(Wg) || !aligned16(dx) || !aligned16(dWg))
            return MOE_ERR_UNSUPPORTED;
        return launch_gate_backward_bf16(x, Wg, T, d, E, dlogits, dx, dWg, workspace, st);
    }
    const size_t need_simt = dWg ? need : 0;
    if (need_simt && (!workspace || workspace_bytes < need_simt)) return MOE_ERR_WORKSPACE;
    float* part = need_simt ? reinterpret_cast<float*>(
                                  (reinterpret_cast<uintptr_t>(workspace) + 255u) & ~uintptr_t(255u))
                            : nullptr;
    return launch_gate_backward(x, Wg, dtype, T, d, E, dlogits, dx, dWg, part, st);
}
