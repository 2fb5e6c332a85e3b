// permute.cu -- moe_dispatch (input encode) and moe_combine (output decode).
//
// "A Survey on Mixture of Experts", section 5: input encode gathers the tokens
// of each expert into contiguous memory so the expert GEMM sees one dense
// block; output decode is the inverse, restoring token order by the gating
// indices (here with the gate weights applied, as the layer output is the
// gate-weighted sum of the selected experts' outputs).
//
// The backward of input encode (moe_dispatch_backward) is the same gather as
// output decode with unit weights: dx[t] = sum of the token's kept rows of dXp.
//
// Both are HBM-bound row copies.  Token-parallel: one warp owns one token row
// at a time (grid-stride over tokens), moves it in 16-byte vectors with
// U vectors per lane in flight, and
//   dispatch: reads x[t] once and writes it to each of its kept rows (a token
//             with no kept row is not read);
//   combine:  reads the token's kept rows of Yp, accumulates w_j * row in fp32
//             with j ascending, and writes y[t] once.  For k <= 8 the loads of
//             all k rows of a column block are issued before the first
//             multiply-add (one memory round trip per block instead of k).
// Algorithmic bytes: dispatch U*d*s + R*d*s (+ T*k*4 index; U = tokens with a
// kept row), combine R*d*s + T*d*s (+ T*k*8 index/weights), s = element size.
#include "common.cuh"

namespace moe {

constexpr int kPermThreads = 256;
constexpr int kU = 4;  // 16-byte vectors per lane in flight

__global__ void __launch_bounds__(kPermThreads)
dispatch_kernel(const uint4* __restrict__ x, int T, int nvec, int k,
                const int32_t* __restrict__ slot_row, uint4* __restrict__ Xp, int R_max,
                int32_t* err) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int wpb = kPermThreads / 32;
    const int nwarps = gridDim.x * wpb;
    for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += nwarps) {
        int my_row = -1;
        if (lane < k) {
            my_row = __ldg(slot_row + (size_t)t * k + lane);
            if (my_row < -1 || my_row >= R_max) {
                flag_error(err, MOE_DEVERR_ROW_INDEX);
                my_row = -1;
            }
        }
        // a token whose every slot was dropped is not read at all
        if (!__any_sync(0xffffffffu, my_row >= 0)) continue;
        const uint4* src = x + (size_t)t * nvec;
        for (int c0 = 0; c0 < nvec; c0 += 32 * kU) {
            uint4 v[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < nvec) v[u] = ldg_nc_v4(src + c);
            }
            for (int j = 0; j < k; ++j) {
                const int row = __shfl_sync(0xffffffffu, my_row, j);
                if (row < 0) continue;
                uint4* dst = Xp + (size_t)row * nvec;
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int c = c0 + u * 32 + lane;
                    if (c < nvec) stg_v4(dst + c, v[u]);
                }
            }
        }
    }
}

// Element access for the two storage types: 8 bf16 or 4 fp32 per vector.
template <int DT> struct Vec;
template <> struct Vec<MOE_DTYPE_BF16> {
    static constexpr int N = 8;
    __device__ static void fma(float* acc, float wj, const uint4& v) {
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[2 * i] = fmaf(wj, bf16lo(u[i]), acc[2 * i]);
            acc[2 * i + 1] = fmaf(wj, bf16hi(u[i]), acc[2 * i + 1]);
        }
    }
    __device__ static uint4 pack(const float* acc) {
        return make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                          pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    }
};
template <> struct Vec<MOE_DTYPE_F32> {
    static constexpr int N = 4;
    __device__ static void fma(float* acc, float wj, const uint4& v) {
        acc[0] = fmaf(wj, __uint_as_float(v.x), acc[0]);
        acc[1] = fmaf(wj, __uint_as_float(v.y), acc[1]);
        acc[2] = fmaf(wj, __uint_as_float(v.z), acc[2]);
        acc[3] = fmaf(wj, __uint_as_float(v.w), acc[3]);
    }
    __device__ static uint4 pack(const float* acc) {
        return make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]),
                          __float_as_uint(acc[2]), __float_as_uint(acc[3]));
    }
};

template <int DT>
__global__ void __launch_bounds__(kPermThreads)
combine_kernel(const uint4* __restrict__ Yp, int T, int nvec, int k,
               const int32_t* __restrict__ slot_row, const float* __restrict__ w,
               uint4* __restrict__ y, int R_max, int32_t* err) {
    using V = Vec<DT>;
    constexpr int CU = 2;  // vectors per lane per pass (accumulators: CU * V::N floats)
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int wpb = kPermThreads / 32;
    const int nwarps = gridDim.x * wpb;
    for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += nwarps) {
        int my_row = -1;
        float my_w = 0.0f;
        if (lane < k) {
            my_row = __ldg(slot_row + (size_t)t * k + lane);
            my_w = w ? __ldg(w + (size_t)t * k + lane) : 1.0f;
            if (my_row < -1 || my_row >= R_max) {
                flag_error(err, MOE_DEVERR_ROW_INDEX);
                my_row = -1;
            }
        }
        for (int c0 = 0; c0 < nvec; c0 += 32 * CU) {
            float acc[CU][V::N];
#pragma unroll
            for (int u = 0; u < CU; ++u)
#pragma unroll
                for (int i = 0; i < V::N; ++i) acc[u][i] = 0.0f;
            for (int j = 0; j < k; ++j) {
                const int row = __shfl_sync(0xffffffffu, my_row, j);
                const float wj = __shfl_sync(0xffffffffu, my_w, j);
                if (row < 0) continue;
                const uint4* src = Yp + (size_t)row * nvec;
                uint4 v[CU];
#pragma unroll
                for (int u = 0; u < CU; ++u) {
                    const int c = c0 + u * 32 + lane;
                    v[u] = (c < nvec) ? ldg_nc_v4(src + c) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < CU; ++u) V::fma(acc[u], wj, v[u]);
            }
            uint4* dst = y + (size_t)t * nvec;
#pragma unroll
            for (int u = 0; u < CU; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < nvec) stg_v4(dst + c, V::pack(acc[u]));
            }
        }
    }
}

// k <= KMAX: every kept row's CU vectors of a column block are in flight at
// once; the sum is the same j-ascending fp32 sequence as combine_kernel's.
template <int DT, int KMAX, int CU>
__global__ void __launch_bounds__(kPermThreads)
combine_wide_kernel(const uint4* __restrict__ Yp, int T, int nvec, int k,
                    const int32_t* __restrict__ slot_row, const float* __restrict__ w,
                    uint4* __restrict__ y, int R_max, int32_t* err) {
    using V = Vec<DT>;
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int wpb = kPermThreads / 32;
    const int nwarps = gridDim.x * wpb;
    for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += nwarps) {
        int my_row = -1;
        float my_w = 0.0f;
        if (lane < k) {
            my_row = __ldg(slot_row + (size_t)t * k + lane);
            my_w = w ? __ldg(w + (size_t)t * k + lane) : 1.0f;
            if (my_row < -1 || my_row >= R_max) {
                flag_error(err, MOE_DEVERR_ROW_INDEX);
                my_row = -1;
            }
        }
        int rows[KMAX];
        float ws[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            rows[j] = __shfl_sync(0xffffffffu, my_row, j);  // lanes >= k hold -1
            ws[j] = __shfl_sync(0xffffffffu, my_w, j);
        }
        uint4* dst = y + (size_t)t * nvec;
        for (int c0 = 0; c0 < nvec; c0 += 32 * CU) {
            uint4 v[KMAX][CU];
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
#pragma unroll
                for (int u = 0; u < CU; ++u) {
                    const int c = c0 + u * 32 + lane;
                    v[j][u] = (rows[j] >= 0 && c < nvec)
                                  ? ldg_nc_v4(Yp + (size_t)rows[j] * nvec + c)
                                  : make_uint4(0, 0, 0, 0);
                }
            float acc[CU][V::N];
#pragma unroll
            for (int u = 0; u < CU; ++u)
#pragma unroll
                for (int i = 0; i < V::N; ++i) acc[u][i] = 0.0f;
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                if (rows[j] >= 0) {
#pragma unroll
                    for (int u = 0; u < CU; ++u) V::fma(acc[u], ws[j], v[j][u]);
                }
#pragma unroll
            for (int u = 0; u < CU; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < nvec) stg_v4(dst + c, V::pack(acc[u]));
            }
        }
    }
}

// The combine (or dispatch-backward) launch for this k: the wide kernel up to
// k = 8, the one-row-at-a-time kernel beyond.
template <int DT>
static int launch_combine(cudaStream_t st, int grid, const uint4* Yp, int T, int nvec, int k,
                          const int32_t* slot_row, const float* w, uint4* y, int R_max) {
    if (k <= 2)
        return launch_pdl(combine_wide_kernel<DT, 2, 4>, grid, kPermThreads, 0, st, Yp, T, nvec,
                          k, slot_row, w, y, R_max, device_error_word());
    if (k <= 4)
        return launch_pdl(combine_wide_kernel<DT, 4, 2>, grid, kPermThreads, 0, st, Yp, T, nvec,
                          k, slot_row, w, y, R_max, device_error_word());
    if (k <= 8)
        return launch_pdl(combine_wide_kernel<DT, 8, 1>, grid, kPermThreads, 0, st, Yp, T, nvec,
                          k, slot_row, w, y, R_max, device_error_word());
    return launch_pdl(combine_kernel<DT>, grid, kPermThreads, 0, st, Yp, T, nvec, k, slot_row, w,
                      y, R_max, device_error_word());
}

static int perm_grid(int T) {
    const int wpb = kPermThreads / 32;
    const int need = (T + wpb - 1) / wpb;
    const int cap = num_sms() * 8;
    return need < cap ? need : cap;
}

static int check_rows(const void* a, const void* b, int dtype, int T, int d, int k) {
    if (!dtype_ok(dtype)) return MOE_ERR_UNSUPPORTED;
    if (T < 0 || d < 1 || k < 1 || k > kMaxTopK) return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * k >= INT32_MAX) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!a || !b)) return MOE_ERR_INVALID_ARG;
    if (((size_t)d * dtype_bytes(dtype)) % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (!aligned16(a) || !aligned16(b)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_dispatch(const void* x, int dtype, int T, int d, int k, const int32_t* slot_row,
                            void* Xp, int R_max, moe_stream_t stream) {
    const int rc = check_rows(x, Xp, dtype, T, d, k);
    if (rc != MOE_OK) return rc;
    if (T > 0 && (!slot_row || R_max < 0)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    const int nvec = (int)((size_t)d * dtype_bytes(dtype) / 16);
    return launch_pdl(dispatch_kernel, perm_grid(T), kPermThreads, 0,
                      reinterpret_cast<cudaStream_t>(stream), static_cast<const uint4*>(x), T,
                      nvec, k, slot_row, static_cast<uint4*>(Xp), R_max, device_error_word());
}

extern "C" MOE_API int moe_combine(const void* Yp, int dtype, int T, int d, int k, const int32_t* slot_row,
                           const float* w, void* y, int R_max, moe_stream_t stream) {
    const int rc = check_rows(Yp, y, dtype, T, d, k);
    if (rc != MOE_OK) return rc;
    if (T > 0 && (!slot_row || R_max < 0)) return MOE_ERR_INVALID_ARG;  // w NULL: unit weights
    if (T == 0) return MOE_OK;
    const int nvec = (int)((size_t)d * dtype_bytes(dtype) / 16);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint4* src = static_cast<const uint4*>(Yp);
    uint4* dst = static_cast<uint4*>(y);
    if (dtype == MOE_DTYPE_BF16)
        return launch_combine<MOE_DTYPE_BF16>(st, perm_grid(T), src, T, nvec, k, slot_row, w, dst,
                                              R_max);
    return launch_combine<MOE_DTYPE_F32>(st, perm_grid(T), src, T, nvec, k, slot_row, w, dst,
                                         R_max);
}

extern "C" MOE_API int moe_dispatch_backward(const void* dXp, int dtype, int T, int d, int k,
                                             const int32_t* slot_row, void* dx, int R_max,
                                             moe_stream_t stream) {
    const int rc = check_rows(dXp, dx, dtype, T, d, k);
    if (rc != MOE_OK) return rc;
    if (T > 0 && (!slot_row || R_max < 0)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    const int nvec = (int)((size_t)d * dtype_bytes(dtype) / 16);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint4* src = static_cast<const uint4*>(dXp);
    uint4* dst = static_cast<uint4*>(dx);
    if (dtype == MOE_DTYPE_BF16)
        return launch_combine<MOE_DTYPE_BF16>(st, perm_grid(T), src, T, nvec, k, slot_row,
                                              nullptr, dst, R_max);
    return launch_combine<MOE_DTYPE_F32>(st, perm_grid(T), src, T, nvec, k, slot_row, nullptr,
                                         dst, R_max);
}
