// gate.cu -- router logits for layers with few experts (E <= 32).
//
// PopFetcher, section 2.1.2: the gate network scores every token against
// every expert, logits[t][e] = sum_c x[t][c] * Wg[e][c].  With E <= 32 the
// projection is a skinny product (a few flops per byte of x), so instead of
// 128-row tensor-core tiles (T/128 CTAs) it runs on the CUDA cores across the
// whole GPU: Wg is staged once per CTA in shared memory (zero-padded to EP
// rows), each warp takes TOK tokens at a time, every lane accumulates the EP x
// TOK partial dot products of its 16-byte slices of the rows in fp32, and warp
// reductions finish the sums.  HBM-bound on x: T*d*s bytes read, T*E*4 written.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kGateThreads = 256;
constexpr int kGateWarps = kGateThreads / 32;
constexpr int kGateSmemMax = 160 * 1024;

template <typename TIn> struct Elems;
template <> struct Elems<__nv_bfloat16> {
    static constexpr int N = 8;  // elements per 16-byte vector
    __device__ static void to_float(const uint4& v, float (&f)[8]) {
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = bf16lo(u[i]);
            f[2 * i + 1] = bf16hi(u[i]);
        }
    }
};
template <> struct Elems<float> {
    static constexpr int N = 4;
    __device__ static void to_float(const uint4& v, float (&f)[4]) {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
};

template <typename TIn, int EP, int TOK>
__global__ void __launch_bounds__(kGateThreads)
gate_small_kernel(const uint4* __restrict__ x, const uint4* __restrict__ Wg, int T, int nvec,
                  int E, float* __restrict__ logits) {
    using V = Elems<TIn>;
    extern __shared__ uint4 s_w[];  // [EP][nvec] vectors, rows >= E zero
    pdl_wait();
    pdl_trigger();
    for (int i = threadIdx.x; i < EP * nvec; i += kGateThreads) {
        const int e = i / nvec;
        s_w[i] = e < E ? Wg[i] : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int warp_global = blockIdx.x * kGateWarps + (threadIdx.x >> 5);
    const int nwarps = gridDim.x * kGateWarps;
    for (int t0 = warp_global * TOK; t0 < T; t0 += nwarps * TOK) {
        float acc[TOK][EP];
#pragma unroll
        for (int q = 0; q < TOK; ++q)
#pragma unroll
            for (int e = 0; e < EP; ++e) acc[q][e] = 0.0f;
        for (int c = lane; c < nvec; c += 32) {
            float xf[TOK][V::N];
#pragma unroll
            for (int q = 0; q < TOK; ++q) {
                const int t = min(t0 + q, T - 1);
                V::to_float(ldg_nc_v4(x + (size_t)t * nvec + c), xf[q]);
            }
#pragma unroll
            for (int e = 0; e < EP; ++e) {
                float wf[V::N];
                V::to_float(s_w[e * nvec + c], wf);
#pragma unroll
                for (int q = 0; q < TOK; ++q)
#pragma unroll
                    for (int j = 0; j < V::N; ++j) acc[q][e] = fmaf(xf[q][j], wf[j], acc[q][e]);
            }
        }
#pragma unroll
        for (int q = 0; q < TOK; ++q) {
            float mine = 0.0f;  // lane e keeps the total of expert e
#pragma unroll
            for (int e = 0; e < EP; ++e) {
                float v = acc[q][e];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == e) mine = v;
            }
            const int t = t0 + q;
            if (t < T && lane < E) logits[(size_t)t * E + lane] = mine;
        }
    }
}

template <typename TIn, int EP, int TOK>
int launch_small(const void* x, const void* Wg, int T, int nvec, int E, float* logits,
                 cudaStream_t st) {
    const int smem = EP * nvec * 16;
    if (ensure_smem<gate_small_kernel<TIn, EP, TOK>>(smem) != MOE_OK) return MOE_ERR_CUDA;
    const int per_cta = kGateWarps * TOK;
    int grid = (T + per_cta - 1) / per_cta;
    const int cap = num_sms() * 4;
    if (grid > cap) grid = cap;
    return launch_pdl(gate_small_kernel<TIn, EP, TOK>, grid, kGateThreads, smem, st,
                      static_cast<const uint4*>(x), static_cast<const uint4*>(Wg), T, nvec, E,
                      logits);
}

template <typename TIn>
int dispatch_small(const void* x, const void* Wg, int T, int nvec, int E, float* logits,
                   cudaStream_t st) {
    if (E <= 8) return launch_small<TIn, 8, 4>(x, Wg, T, nvec, E, logits, st);
    if (E <= 16) return launch_small<TIn, 16, 4>(x, Wg, T, nvec, E, logits, st);
    return launch_small<TIn, 32, 2>(x, Wg, T, nvec, E, logits, st);
}

}  // namespace

bool gate_small_fits(int E, int d, int dtype) {
    if (E > 32) return false;
    const int EP = E <= 8 ? 8 : (E <= 16 ? 16 : 32);
    return (size_t)EP * d * dtype_bytes(dtype) <= (size_t)kGateSmemMax;
}

int launch_gate_small(const void* x, const void* Wg, int dtype, int T, int d, int E,
                      float* logits, cudaStream_t st) {
    const int nvec = (int)((size_t)d * dtype_bytes(dtype) / 16);
    if (dtype == MOE_DTYPE_BF16)
        return dispatch_small<__nv_bfloat16>(x, Wg, T, nvec, E, logits, st);
    return dispatch_small<float>(x, Wg, T, nvec, E, logits, st);
}

}  // namespace moe
