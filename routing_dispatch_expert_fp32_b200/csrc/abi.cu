// abi.cu -- status strings, version and the per-device error word.
#include "common.cuh"

namespace moe {

__device__ int32_t g_device_error = 0;

// The symbol's device address, looked up once per device (host threads that
// race on the first lookup store the same address).
int32_t* device_error_word() {
    static std::atomic<int32_t*> cache[kMaxDevices] = {};
    const int dev = current_device();
    if (dev < 0) return nullptr;
    int32_t* p = cache[dev].load(std::memory_order_acquire);
    if (!p) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_device_error) != cudaSuccess) return nullptr;
        p = static_cast<int32_t*>(a);
        cache[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace moe

extern "C" MOE_API const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported dtype, size or alignment";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_DEVICE: return "device-side check failed";
        default: return "unknown status";
    }
}

extern "C" MOE_API int moe_version(void) { return 100; }

extern "C" MOE_API int moe_device_error(int32_t* bits, int clear) {
    if (!bits) return MOE_ERR_INVALID_ARG;
    int32_t v = 0;
    if (cudaMemcpyFromSymbol(&v, moe::g_device_error, sizeof v) != cudaSuccess) return MOE_ERR_CUDA;
    *bits = v;
    if (clear) {
        const int32_t zero = 0;
        if (cudaMemcpyToSymbol(moe::g_device_error, &zero, sizeof zero) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

#ifdef MOE_TEST_HOOKS
// Test builds only (-DMOE_TEST_HOOKS, built apart from the shipped library by
// the test suite): hooks that make the tcgen05 GEMMs' bounded waits run out
// with nothing in flight, and that cap their grid.
namespace moe {
static std::atomic<int> g_test_max_ctas{0};
int test_max_ctas() { return g_test_max_ctas.load(std::memory_order_relaxed); }
int test_stall_tc(int v);
int test_stall_bwd(int v);
}  // namespace moe

// stall != 0: the forward and backward GEMM producers issue no loads;
// max_ctas > 0: at most that many persistent GEMM CTAs (pairs: max_ctas / 2).
extern "C" MOE_API int moe_test_hooks(int stall, int max_ctas) {
    moe::g_test_max_ctas.store(max_ctas > 0 ? max_ctas : 0, std::memory_order_relaxed);
    if (moe::test_stall_tc(stall ? 1 : 0) != MOE_OK) return MOE_ERR_CUDA;
    if (moe::test_stall_bwd(stall ? 1 : 0) != MOE_OK) return MOE_ERR_CUDA;
    return MOE_OK;
}
#endif
