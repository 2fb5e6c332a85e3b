// abi.cu -- status strings, version and the per-device error word.
#include "common.cuh"

namespace moe {

__device__ int32_t g_device_error = 0;

int32_t* device_error_word() {
    static int32_t* cache[kMaxDevices] = {};
    const int dev = current_device();
    if (dev < 0) return nullptr;
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        cache[dev] = static_cast<int32_t*>(p);
    }
    return cache[dev];
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
