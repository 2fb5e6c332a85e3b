// kernels.h -- launchers shared between the kernel files and the ABI entry points.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Expert FFN with the token rows gathered straight from x (no dispatched
// copy) and, when w is non-null, the gate weight applied to each output row
// (gemm_tc.cu, bf16, 1-CTA tiles).
int launch_ffn_gather_bf16(const void* x, int T, int k, const int32_t* row_slot, const float* w,
                           const void* W1, const void* W2, int E, int d, int F,
                           const int32_t* offsets, int R_max, void* H, void* Yp,
                           cudaStream_t st);

// fp32 grouped GEMM on the CUDA cores (gemm_simt.cu).
int launch_gemm_simt_f32(const float* A, const float* B, float* C, int N, int K, int E,
                         const int32_t* offsets, int single_M, int R_max, bool relu,
                         cudaStream_t st);

// bf16 grouped GEMM on tcgen05 tensor cores (gemm_tc.cu); C is bf16, or fp32
// when out_f32 (no ReLU then).
int launch_gemm_tc_bf16(const void* A, const void* B, void* C, bool out_f32, int N, int K, int E,
                        const int32_t* offsets, int single_M, int R_max, bool relu,
                        cudaStream_t st);

// Whether a grouped GEMM of N columns takes the 2-CTA pair tiles (the forward
// pass's rule: groups dense on average, or 128-row tiles filling fewer than
// three waves), and the pair GEMM with the weights read N-major ([E*K, N], rows
// e*K.. for group e), C bf16, zeroed where Hmask (when non-null, [R, N] bf16)
// is not positive (gemm_tc.cu; the expert backward's input gradients).
bool gemm_pair_tiles(int R_max, int E, int N);
int launch_gemm_pair_nmajor_bf16(const void* A, const void* B, void* C, int N, int K, int E,
                                 const int32_t* offsets, int R_max, const void* Hmask,
                                 cudaStream_t st);

// Router logits for E <= 32 on the CUDA cores (gate.cu); gate_small_fits says
// whether the gate weights fit the kernel's shared-memory stage.
bool gate_small_fits(int E, int d, int dtype);
int launch_gate_small(const void* x, const void* Wg, int dtype, int T, int d, int E,
                      float* logits, cudaStream_t st);

// Backward of the expert FFN over the grouped rows (gemm_bwd.cu for bf16 on
// tcgen05, gemm_simt.cu for fp32): dH = (dYp . W2_e) masked by H > 0,
// dXp = dH . W1_e, and (when non-null) dW2_e = dYp_e^T H_e, dW1_e = dH_e^T Xp_e
// in fp32.
int launch_ffn_backward_bf16(const void* Xp, const void* H, const void* dYp, const void* W1,
                             const void* W2, int E, int d, int F, const int32_t* offsets,
                             int R_max, void* dH, void* dXp, float* dW1, float* dW2,
                             cudaStream_t st);
int launch_ffn_backward_f32(const float* Xp, const float* H, const float* dYp, const float* W1,
                            const float* W2, int E, int d, int F, const int32_t* offsets,
                            int R_max, float* dH, float* dXp, float* dW1, float* dW2,
                            cudaStream_t st);

// Epilogues of the CUDA-core backward product (gemm_simt.cu).
enum { SIMT_EPI_STORE = 0, SIMT_EPI_MASK = 1, SIMT_EPI_ADD = 2 };

// Gate projection backward on the CUDA cores (gemm_simt.cu):
// dx += dlogits . Wg, and dWg = dlogits^T . x (fp32) when dWg is non-null,
// the tokens cut into gate_backward_splits(T, d, E) slices whose partial
// products go to `part` ([splits][E][d] fp32, unused with one slice).
int gate_backward_splits(int T, int d, int E);
int launch_gate_backward(const void* x, const void* Wg, int dtype, int T, int d, int E,
                         const float* dlogits, void* dx, float* dWg, float* part,
                         cudaStream_t st);

// out[i] = sum over s ascending of part[s * n + i] (gemm_simt.cu).
int launch_split_reduce(const float* part, int ksplit, size_t n, float* out, cudaStream_t st);

// Gate projection backward of bf16 layers on tcgen05 (gemm_bwd.cu): dlogits
// split exactly into three bf16 planes; dx += dlogits . Wg, dWg (fp32, when
// non-null) over token slices added in order.  Needs d and E multiples of 8
// (gate_backward_tc_ok) and gate_backward_tc_workspace(T, d, E) bytes.
bool gate_backward_tc_ok(int d, int E);
void gate_backward_tc_slices(int T, int d, int E, int* S, int* slice_rows);
size_t gate_backward_tc_workspace(int T, int d, int E);
int launch_gate_backward_bf16(const void* x, const void* Wg, int T, int d, int E,
                              const float* dlogits, void* dx, float* dWg, void* ws,
                              cudaStream_t st);

}  // namespace moe
