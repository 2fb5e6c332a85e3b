// common.cuh -- helpers shared by the MoE kernels (device side and host-side
// argument checks).  Nothing here is shared with the CPU oracle.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "../../include/moe.h"

namespace moe {

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;

// Per-device error word (defined in abi.cu): device-side checks OR bits into
// it instead of faulting; moe_device_error() reads and clears it.  Kernels in
// other translation units receive its address as an argument.
int32_t* device_error_word();  // nullptr if the symbol lookup failed

__device__ __forceinline__ void flag_error(int32_t* err, int32_t bits) {
    if (err) atomicOr(err, bits);
}

// ----------------------------------------------------------------- host ----
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t dtype_bytes(int dtype) { return dtype == MOE_DTYPE_BF16 ? 2u : 4u; }
inline bool dtype_ok(int dtype) { return dtype == MOE_DTYPE_F32 || dtype == MOE_DTYPE_BF16; }

// Launch-error check: returns MOE_ERR_CUDA if the last launch failed.
inline int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

constexpr int kMaxDevices = 64;

inline int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

// SM count of the current device (queried once per device; host threads that
// race on the first query store the same value).
inline int num_sms() {
    static std::atomic<int> cache[kMaxDevices] = {};
    const int dev = current_device();
    if (dev < 0) return 148;
    int n = cache[dev].load(std::memory_order_acquire);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev].store(n, std::memory_order_release);
    }
    return n;
}

#ifdef MOE_TEST_HOOKS
// Test builds only: a cap on the persistent GEMMs' CTA count (abi.cu), so that
// a small problem makes one CTA (or one pair) walk many tiles.
int test_max_ctas();
inline int test_cap(int grid) {
    const int c = test_max_ctas();
    return (c > 0 && grid > c) ? c : grid;
}
#else
inline int test_cap(int grid) { return grid; }
#endif

// Raises a kernel's dynamic shared-memory limit once per device (and again only
// if a larger size is needed), so launches inside a stream capture make no
// attribute calls.  One cache per kernel (the kernel is the template argument,
// so kernels that share a signature do not share a cache); raising the limit
// is serialised so that a smaller request never undoes a larger one.
template <auto kern>
inline int ensure_smem(int bytes) {
    static std::atomic<int> done[kMaxDevices] = {};
    static std::mutex mu;
    const int dev = current_device();
    if (dev < 0) return MOE_ERR_CUDA;
    if (done[dev].load(std::memory_order_acquire) >= bytes) return MOE_OK;
    std::lock_guard<std::mutex> lock(mu);
    if (done[dev].load(std::memory_order_relaxed) >= bytes) return MOE_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    done[dev].store(bytes, std::memory_order_release);
    return MOE_OK;
}

// Launches `kern` with programmatic stream serialization: the kernel may be
// scheduled while the previous kernel on the stream is still running, and it
// waits for that kernel (pdl_wait) before its first global-memory access.
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// --------------------------------------------------------------- device ----
// Programmatic dependent launch: wait until the previous kernel on the stream
// has completed and its writes are visible (returns at once when the kernel
// was launched without the attribute), and let the next kernel be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 16-byte global accesses.  Loads of read-only inputs bypass L1 allocation.
__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void stg_v4(void* p, const uint4& v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Two floats -> packed bf16x2 (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace moe
