// gemm_simt.cu -- fp32 grouped GEMM on the CUDA cores (no TF32).
//
// Used for fp32 layers, where every operand and product stays fp32: the
// expert FFN (PopFetcher, section 5.1: FC -> ReLU -> FC) and the gate
// projection.  C[r][n] = act(sum_k A[r][k] * B_e[n][k]) for the rows r of
// group e; both operands K-major.  64 x 64 output tiles, 16-deep K slices
// staged in shared memory, 4 x 4 outputs per thread, persistent CTAs walking
// the device-side tile table.
#include "grouped.cuh"
#include "kernels.h"

namespace moe {

namespace {
constexpr int SBM = 64, SBN = 64, SBK = 16, SThreads = 256;
}

template <bool RELU>
__global__ void __launch_bounds__(SThreads)
gemm_simt_f32_kernel(const float* __restrict__ A, const float* __restrict__ B,
                     float* __restrict__ C, int N, int K, int E,
                     const int32_t* __restrict__ offsets, int single_M, int R_max, int32_t* err) {
    __shared__ int32_t s_prefix[kMaxExperts + 1];
    __shared__ int32_t s_warp[32];
    __shared__ float As[SBK][SBM + 4];
    __shared__ float Bs[SBK][SBN + 4];
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    pdl_wait();
    pdl_trigger();
    const int nt = (N + SBN - 1) / SBN;
    const int total =
        nt * build_tile_table(offsets, single_M, E, 1, SBM, R_max, s_prefix, s_warp, err);

    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const TileCoord tc = tile_coord(tile, s_prefix, E, offsets, single_M, SBM, SBN, nt);
        const float* Ab = A + (size_t)tc.row0 * K;
        const float* Bb = B + ((size_t)tc.e * N + tc.n0) * K;
        const int ncols = min(SBN, N - tc.n0);
        float acc[4][4] = {};
        for (int k0 = 0; k0 < K; k0 += SBK) {
            for (int i = tid; i < SBM * SBK; i += SThreads) {
                const int r = i / SBK, kk = i % SBK;
                As[kk][r] = (r < tc.rows && k0 + kk < K) ? Ab[(size_t)r * K + k0 + kk] : 0.0f;
                Bs[kk][r] = (r < ncols && k0 + kk < K) ? Bb[(size_t)r * K + k0 + kk] : 0.0f;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < SBK; ++kk) {
                float a[4], b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            }
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty * 4 + i;
            if (r >= tc.rows) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = tx * 4 + j;
                if (c >= ncols) continue;
                const float v = acc[i][j];
                C[(size_t)(tc.row0 + r) * N + tc.n0 + c] = RELU ? (v > 0.0f ? v : 0.0f) : v;
            }
        }
    }
}

int launch_gemm_simt_f32(const float* A, const float* B, float* C, int N, int K, int E,
                         const int32_t* offsets, int single_M, int R_max, bool relu,
                         cudaStream_t st) {
    const int nt = (N + SBN - 1) / SBN;
    const long long ub = ((long long)R_max / SBM + E) * nt;  // tile count upper bound
    const int grid = (int)(ub < (long long)num_sms() * 4 ? ub : (long long)num_sms() * 4);
    if (grid <= 0) return MOE_OK;
    int32_t* err = device_error_word();
    auto kern = relu ? gemm_simt_f32_kernel<true> : gemm_simt_f32_kernel<false>;
    return launch_pdl(kern, grid, SThreads, 0, st, A, B, C, N, K, E, offsets, single_M, R_max, err);
}


// ----------------------------------------------------------------------------
// Backward products on the CUDA cores, C = A . B with B N-major ([K][N] rows):
//   fixed K   (KVAR false): rows of group e (offsets, or one group of single_M
//             rows), A K-major [rows][lda], B = block e of [E*K_fix][ldb];
//   group K   (KVAR true):  output [M_fix][N] per group e contracted over the
//             group's rows [a, b): A M-major (row r holds A(., r)), B rows r;
//             C fp32 [E][M_fix][N], zero for a group without rows.  With
//             ksplit > 1 the rows of a group are cut into ksplit consecutive
//             slices and slice s writes its partial product to
//             C + s * E * M_fix * N (reduced afterwards in slice order).
// Epilogues: store, store where Hmask > 0 (the ReLU's gradient), or add to
// the values already in C.  Products and sums in fp32; A, B, C bf16 or fp32.
namespace {

__device__ __forceinline__ float ld_f(const float* p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_f(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_f(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

}  // namespace

template <typename TA, bool A_MN, typename TB, bool KVAR, int EPI, typename TC>
__global__ void __launch_bounds__(SThreads)
gemm_simt_bwd_kernel(const TA* __restrict__ A, int lda, const TB* __restrict__ B, int ldb,
                     TC* __restrict__ C, const TC* __restrict__ Hmask, int M_fix, int N,
                     int K_fix, int E, const int32_t* __restrict__ offsets, int single_M,
                     int R_max, int ksplit, int32_t* err) {
    __shared__ int32_t s_prefix[kMaxExperts + 1];
    __shared__ int32_t s_warp[32];
    __shared__ float As[SBK][SBM + 4];
    __shared__ float Bs[SBK][SBN + 4];
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    pdl_wait();
    pdl_trigger();
    const int nt = (N + SBN - 1) / SBN;
    const int mt = KVAR ? (M_fix + SBM - 1) / SBM : 1;
    int total;
    if (KVAR) {
        total = E * ksplit * mt * nt;
        if (blockIdx.x == 0 && tid == 0 && offsets)
            for (int e = 0; e < E; ++e) {
                const int a = offsets[e], b = offsets[e + 1];
                if (a < 0 || b < a || b > R_max) flag_error(err, MOE_DEVERR_OFFSETS);
            }
    } else {
        total = nt * build_tile_table(offsets, single_M, E, 1, SBM, R_max, s_prefix, s_warp, err);
    }

    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        int e, row0, rows, n0, ka, kr, sl = 0;
        if (KVAR) {
            e = tile / (ksplit * mt * nt);
            const int rem = tile - e * ksplit * mt * nt;
            sl = rem / (mt * nt);
            const int local = rem - sl * mt * nt;
            row0 = (local % mt) * SBM;
            rows = min(SBM, M_fix - row0);
            n0 = (local / mt) * SBN;
            const int ga = group_off(offsets, e, single_M);
            const int gb = group_off(offsets, e + 1, single_M);
            const int gr = (ga < 0 || gb < ga || gb > R_max) ? 0 : gb - ga;
            const int per = ((gr + ksplit - 1) / ksplit + SBK - 1) / SBK * SBK;
            ka = ga + sl * per;
            kr = max(0, min(gr - sl * per, per));
        } else {
            const TileCoord c = tile_coord(tile, s_prefix, E, offsets, single_M, SBM, SBN, nt);
            e = c.e;
            row0 = c.row0;
            rows = c.rows;
            n0 = c.n0;
            ka = 0;
            kr = K_fix;
        }
        const int ncols = min(SBN, N - n0);
        const TB* Bb = KVAR ? B + (size_t)ka * ldb + n0 : B + (size_t)e * K_fix * ldb + n0;
        float acc[4][4] = {};
        for (int k0 = 0; k0 < kr; k0 += SBK) {
            for (int i = tid; i < SBM * SBK; i += SThreads) {
                if (A_MN) {
                    const int kk = i / SBM, m = i % SBM;
                    As[kk][m] = (m < rows && k0 + kk < kr)
                                    ? ld_f(A + (size_t)(ka + k0 + kk) * lda + row0 + m)
                                    : 0.0f;
                } else {
                    const int m = i / SBK, kk = i % SBK;
                    As[kk][m] = (m < rows && k0 + kk < kr)
                                    ? ld_f(A + (size_t)(row0 + m) * lda + k0 + kk)
                                    : 0.0f;
                }
                const int kk = i / SBN, n = i % SBN;
                Bs[kk][n] = (n < ncols && k0 + kk < kr) ? ld_f(Bb + (size_t)(k0 + kk) * ldb + n)
                                                        : 0.0f;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < SBK; ++kk) {
                float a[4], b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            }
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty * 4 + i;
            if (r >= rows) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = tx * 4 + j;
                if (c >= ncols) continue;
                const float v = acc[i][j];
                if (KVAR) {
                    reinterpret_cast<float*>(C)[(((size_t)sl * E + e) * M_fix + row0 + r) * N +
                                                n0 + c] = v;
                } else {
                    const size_t o = (size_t)(row0 + r) * N + n0 + c;
                    if (EPI == SIMT_EPI_MASK) st_f(C + o, ld_f(Hmask + o) > 0.0f ? v : 0.0f);
                    else if (EPI == SIMT_EPI_ADD) st_f(C + o, ld_f(C + o) + v);
                    else st_f(C + o, v);
                }
            }
        }
    }
}

// out[i] = sum over s ascending of part[s * n + i]
__global__ void __launch_bounds__(SThreads)
split_reduce_kernel(const float* __restrict__ part, int ksplit, size_t n, float* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    for (size_t i = (size_t)blockIdx.x * SThreads + threadIdx.x; i < n;
         i += (size_t)gridDim.x * SThreads) {
        float v = part[i];
        for (int s = 1; s < ksplit; ++s) v = __fadd_rn(v, part[(size_t)s * n + i]);
        out[i] = v;
    }
}

int launch_split_reduce(const float* part, int ksplit, size_t n, float* out, cudaStream_t st) {
    long long grid = (long long)((n + SThreads - 1) / SThreads);
    if (grid > (long long)num_sms() * 8) grid = (long long)num_sms() * 8;
    if (grid <= 0) return MOE_OK;
    return launch_pdl(split_reduce_kernel, (int)grid, SThreads, 0, st, part, ksplit, n, out);
}

template <typename TA, bool A_MN, typename TB, bool KVAR, int EPI, typename TC>
int launch_simt_bwd(const TA* A, int lda, const TB* B, int ldb, TC* C, const TC* Hmask, int M_fix,
                    int N, int K_fix, int E, const int32_t* offsets, int single_M, int R_max,
                    cudaStream_t st, int ksplit = 1) {
    const int nt = (N + SBN - 1) / SBN;
    const long long ub = KVAR ? (long long)E * ksplit * ((M_fix + SBM - 1) / SBM) * nt
                              : ((long long)R_max / SBM + E) * nt;
    const int grid = (int)(ub < (long long)num_sms() * 4 ? ub : (long long)num_sms() * 4);
    if (grid <= 0) return MOE_OK;
    return launch_pdl(gemm_simt_bwd_kernel<TA, A_MN, TB, KVAR, EPI, TC>, grid, SThreads, 0, st, A,
                      lda, B, ldb, C, Hmask, M_fix, N, K_fix, E, offsets, single_M, R_max,
                      ksplit, device_error_word());
}

int launch_ffn_backward_f32(const float* Xp, const float* H, const float* dYp, const float* W1,
                            const float* W2, int E, int d, int F, const int32_t* offsets,
                            int R_max, float* dH, float* dXp, float* dW1, float* dW2,
                            cudaStream_t st) {
    int rc = launch_simt_bwd<float, false, float, false, SIMT_EPI_MASK, float>(
        dYp, d, W2, F, dH, H, 0, F, d, E, offsets, 0, R_max, st);
    if (rc != MOE_OK) return rc;
    rc = launch_simt_bwd<float, false, float, false, SIMT_EPI_STORE, float>(
        dH, F, W1, d, dXp, nullptr, 0, d, F, E, offsets, 0, R_max, st);
    if (rc != MOE_OK) return rc;
    if (dW2) {
        rc = launch_simt_bwd<float, true, float, true, SIMT_EPI_STORE, float>(
            dYp, d, H, F, dW2, nullptr, d, F, 0, E, offsets, 0, R_max, st);
        if (rc != MOE_OK) return rc;
    }
    if (dW1)
        rc = launch_simt_bwd<float, true, float, true, SIMT_EPI_STORE, float>(
            dH, F, Xp, d, dW1, nullptr, F, d, 0, E, offsets, 0, R_max, st);
    return rc;
}

// Token slices for dWg: enough (tile, slice) units to fill the GPU about
// seven times over 148 SMs, slices of at least 256 tokens.  A function of the
// shape only, so the result does not depend on the device.
int gate_backward_splits(int T, int d, int E) {
    const long long tiles = (long long)((E + SBM - 1) / SBM) * ((d + SBN - 1) / SBN);
    long long s = (1024 + tiles - 1) / tiles;
    const long long cap = ((long long)T + 255) / 256;
    if (s > cap) s = cap;
    return s < 1 ? 1 : (int)s;
}

template <typename TX>
static int gate_backward_t(const TX* x, const TX* Wg, int T, int d, int E, const float* dlogits,
                           TX* dx, float* dWg, float* part, cudaStream_t st) {
    // dx[t] += dlogits[t] . Wg  (one group of T rows, K = E, Wg rows are K)
    int rc = launch_simt_bwd<float, false, TX, false, SIMT_EPI_ADD, TX>(
        dlogits, E, Wg, d, dx, nullptr, 0, d, E, 1, nullptr, T, T, st);
    if (rc != MOE_OK || !dWg) return rc;
    // dWg = dlogits^T . x  (one group: contraction over all T tokens, in slices)
    const int ks = gate_backward_splits(T, d, E);
    if (ks == 1)
        return launch_simt_bwd<float, true, TX, true, SIMT_EPI_STORE, float>(
            dlogits, E, x, d, dWg, nullptr, E, d, 0, 1, nullptr, T, T, st);
    rc = launch_simt_bwd<float, true, TX, true, SIMT_EPI_STORE, float>(
        dlogits, E, x, d, part, nullptr, E, d, 0, 1, nullptr, T, T, st, ks);
    if (rc != MOE_OK) return rc;
    return launch_split_reduce(part, ks, (size_t)E * d, dWg, st);
}

int launch_gate_backward(const void* x, const void* Wg, int dtype, int T, int d, int E,
                         const float* dlogits, void* dx, float* dWg, float* part,
                         cudaStream_t st) {
    if (dtype == MOE_DTYPE_BF16)
        return gate_backward_t(static_cast<const __nv_bfloat16*>(x),
                               static_cast<const __nv_bfloat16*>(Wg), T, d, E, dlogits,
                               static_cast<__nv_bfloat16*>(dx), dWg, part, st);
    return gate_backward_t(static_cast<const float*>(x), static_cast<const float*>(Wg), T, d, E,
                           dlogits, static_cast<float*>(dx), dWg, part, st);
}

}  // namespace moe
