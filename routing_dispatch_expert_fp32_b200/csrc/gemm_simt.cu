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

}  // namespace moe
