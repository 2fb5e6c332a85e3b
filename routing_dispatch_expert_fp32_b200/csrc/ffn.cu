// ffn.cu -- moe_expert_ffn, moe_expert_ffn_gather and moe_gate entry points
// (argument checks, then the grouped GEMM launches).
//
// Expert computation, PopFetcher section 5.1: FC(d -> F), ReLU, FC(F -> d),
// run group by group over the contiguous per-expert row blocks of input
// encode.  bf16 layers run on the tcgen05 tensor cores; fp32 layers on the
// CUDA cores (fp32 products, no TF32).  The gate projection (PopFetcher,
// section 2.1.2) is the same GEMM with one group and fp32 output, or, for
// fp32 layers with E <= 32, the skinny CUDA-core kernel of gate.cu.
#include "common.cuh"
#include "kernels.h"

using namespace moe;

extern "C" MOE_API int moe_expert_ffn(const void* Xp, const void* W1, const void* W2, int dtype, int E,
                              int d, int F, const int32_t* offsets, int R_max, void* H, void* Yp,
                              moe_stream_t stream) {
    if (!dtype_ok(dtype)) return MOE_ERR_UNSUPPORTED;
    if (E < 1 || E > kMaxExperts || d < 1 || F < 1 || R_max < 0) return MOE_ERR_INVALID_ARG;
    if ((int64_t)E * d >= INT32_MAX || (int64_t)E * F >= INT32_MAX) return MOE_ERR_INVALID_ARG;
    if (!Xp || !W1 || !W2 || !offsets || !H || !Yp) return MOE_ERR_INVALID_ARG;
    const size_t es = dtype_bytes(dtype);
    if ((d * es) % 16 != 0 || (F * es) % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (!aligned16(Xp) || !aligned16(W1) || !aligned16(W2) || !aligned16(H) || !aligned16(Yp))
        return MOE_ERR_UNSUPPORTED;
    if (R_max == 0) return MOE_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int rc;
    if (dtype == MOE_DTYPE_BF16) {
        rc = launch_gemm_tc_bf16(Xp, W1, H, false, F, d, E, offsets, 0, R_max, true, st);
        if (rc != MOE_OK) return rc;
        return launch_gemm_tc_bf16(H, W2, Yp, false, d, F, E, offsets, 0, R_max, false, st);
    }
    rc = launch_gemm_simt_f32(static_cast<const float*>(Xp), static_cast<const float*>(W1),
                              static_cast<float*>(H), F, d, E, offsets, 0, R_max, true, st);
    if (rc != MOE_OK) return rc;
    return launch_gemm_simt_f32(static_cast<const float*>(H), static_cast<const float*>(W2),
                                static_cast<float*>(Yp), d, F, E, offsets, 0, R_max, false, st);
}

extern "C" MOE_API int moe_expert_ffn_gather(const void* x, int T, int k, const int32_t* row_slot,
                                             const float* w, const void* W1, const void* W2,
                                             int dtype, int E, int d, int F,
                                             const int32_t* offsets, int R_max, void* H, void* Yp,
                                             moe_stream_t stream) {
    if (!dtype_ok(dtype)) return MOE_ERR_UNSUPPORTED;
    if (dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;  // tensor-core path only
    if (T < 0 || k < 1 || k > kMaxTopK || E < 1 || E > kMaxExperts || d < 1 || F < 1 || R_max < 0)
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * k >= INT32_MAX || (int64_t)E * d >= INT32_MAX || (int64_t)E * F >= INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (R_max > 0 && (!x || !row_slot || !W1 || !W2 || !offsets || !H || !Yp))
        return MOE_ERR_INVALID_ARG;
    if ((d * 2) % 16 != 0 || (F * 2) % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(W1) || !aligned16(W2) || !aligned16(H) || !aligned16(Yp))
        return MOE_ERR_UNSUPPORTED;
    if (R_max == 0 || T == 0) return MOE_OK;
    return launch_ffn_gather_bf16(x, T, k, row_slot, w, W1, W2, E, d, F, offsets, R_max, H, Yp,
                                  reinterpret_cast<cudaStream_t>(stream));
}

extern "C" MOE_API int moe_gate(const void* x, const void* Wg, int dtype, int T, int d, int E,
                        float* logits, moe_stream_t stream) {
    if (!dtype_ok(dtype)) return MOE_ERR_UNSUPPORTED;
    if (T < 0 || d < 1 || E < 1 || E > kMaxExperts) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !Wg || !logits) return MOE_ERR_INVALID_ARG;
    if ((d * dtype_bytes(dtype)) % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(Wg) || !aligned16(logits)) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // fp32 layers with few experts: the CUDA-core kernel (measured faster than
    // the tiled SIMT GEMM there); bf16 stays on the tensor cores, which were
    // measured faster than that kernel (skewed_drops: 15.0 vs 16.2 us).
    if (dtype == MOE_DTYPE_F32 && gate_small_fits(E, d, dtype))
        return launch_gate_small(x, Wg, dtype, T, d, E, logits, st);
    if (dtype == MOE_DTYPE_BF16)
        return launch_gemm_tc_bf16(x, Wg, logits, true, E, d, 1, nullptr, T, T, false, st);
    return launch_gemm_simt_f32(static_cast<const float*>(x), static_cast<const float*>(Wg), logits,
                                E, d, 1, nullptr, T, T, false, st);
}
