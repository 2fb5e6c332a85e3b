// kernels.h -- launchers shared between the kernel files and the ABI entry points.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// fp32 grouped GEMM on the CUDA cores (gemm_simt.cu).
int launch_gemm_simt_f32(const float* A, const float* B, float* C, int N, int K, int E,
                         const int32_t* offsets, int single_M, int R_max, bool relu,
                         cudaStream_t st);

// bf16 grouped GEMM on tcgen05 tensor cores (gemm_tc.cu); C is bf16, or fp32
// when out_f32 (no ReLU then).
int launch_gemm_tc_bf16(const void* A, const void* B, void* C, bool out_f32, int N, int K, int E,
                        const int32_t* offsets, int single_M, int R_max, bool relu,
                        cudaStream_t st);

// Router logits for E <= 32 on the CUDA cores (gate.cu); gate_small_fits says
// whether the gate weights fit the kernel's shared-memory stage.
bool gate_small_fits(int E, int d, int dtype);
int launch_gate_small(const void* x, const void* Wg, int dtype, int T, int d, int E,
                      float* logits, cudaStream_t st);

}  // namespace moe
