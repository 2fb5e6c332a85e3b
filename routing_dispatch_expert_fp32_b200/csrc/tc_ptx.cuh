// tc_ptx.cuh -- inline-PTX wrappers for the tcgen05 kernels: mbarriers with
// time-bounded waits, TMA tile loads, TMEM allocation, UMMA descriptors and
// issue, tcgen05.ld, and the epilogue's 32-column stores.  Shared by the
// forward (gemm_tc.cu) and backward (gemm_bwd.cu) grouped GEMMs.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;  // one 128-byte swizzle row of bf16
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
// Longest wait of one pipeline barrier before the kernel gives up: 2 s (a
// test build shortens it with -DMOE_WAIT_LIMIT_NS).
#ifndef MOE_WAIT_LIMIT_NS
#define MOE_WAIT_LIMIT_NS 2000000000ull
#endif
constexpr unsigned long long kTimeoutNs = MOE_WAIT_LIMIT_NS;

#ifdef MOE_TEST_HOOKS
// Test builds only (-DMOE_TEST_HOOKS; never the shipped library): a flag of
// this translation unit that makes the GEMM producers issue no loads at all,
// so that the MMA and epilogue waits run out with nothing in flight.
static __device__ int s_test_stall = 0;
__device__ __forceinline__ bool test_stall() {
    return *reinterpret_cast<volatile int*>(&s_test_stall) != 0;
}
static int set_test_stall(int v) {
    return cudaMemcpyToSymbol(s_test_stall, &v, sizeof v) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
#else
__device__ __forceinline__ bool test_stall() { return false; }
#endif

// ------------------------------------------------------------ PTX wrappers --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Waits for the phase of `bar` with the given parity.  Gives up (returns
// false) when another role has raised the abort flag, or after kTimeoutNs, in
// which case it raises the flag and records MOE_DEVERR_TIMEOUT.
static __device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                       int32_t* err, bool honour_abort = true) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait(a, parity)) return true;
        if ((spin & 63u) == 0) {
            if (honour_abort && *abort_flag) return false;
            if (globaltimer() - t0 > kTimeoutNs) {
                *abort_flag = 1;
                flag_error(err, MOE_DEVERR_TIMEOUT);
                return false;
            }
        }
    }
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}
// Tensor store from shared memory (bulk-group completion); the source must
// stay untouched until cp.async.bulk.wait_group.read says it has been read.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y,
                                             int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until at most N committed bulk groups of this thread still read
// shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read_allow() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
// Shared-memory matrix descriptor: K-major tile whose rows are 128 bytes with
// the 128-byte swizzle, 8-row core groups 1024 bytes apart (tile base must be
// 1024-byte aligned; +32 bytes steps one K=16 slice inside the swizzle row).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);  // start address
    d |= static_cast<uint64_t>(1) << 16;                  // leading byte offset (unused here)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;          // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                  // descriptor version
    d |= static_cast<uint64_t>(2) << 61;                  // 128-byte swizzle
    return d;
}
// MN-major operand descriptor, 128-byte swizzle: 64-element MN atoms (one
// 64 x 64 TMA box each) 8 KB apart, 8-row K groups 1 KB apart; +2 KB steps one
// K=16 slice.
constexpr int kMnAtomBytes = 64 * BK * 2;  // 8 KB
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);      // start address
    d |= static_cast<uint64_t>(kMnAtomBytes >> 4) << 16;       // leading byte offset
    d |= static_cast<uint64_t>(1024 >> 4) << 32;               // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                       // descriptor version
    d |= static_cast<uint64_t>(2) << 61;                       // 128-byte swizzle
    return d;
}
// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major (bit 15 / bit 16 mark an MN-major A / B).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------ epilogue
template <typename TOut, bool RELU>
struct Store32;
template <bool RELU>
struct Store32<__nv_bfloat16, RELU> {
    // 32 consecutive columns of one row; N % 8 == 0 is guaranteed by the host.
    __device__ static void run(__nv_bfloat16* dst, const uint32_t (&r)[32], int cols_left) {
        uint32_t p[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float lo = __uint_as_float(r[2 * i]), hi = __uint_as_float(r[2 * i + 1]);
            if (RELU) {
                lo = lo > 0.0f ? lo : 0.0f;
                hi = hi > 0.0f ? hi : 0.0f;
            }
            p[i] = pack_bf16x2(lo, hi);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (q * 8 < cols_left)
                stg_v4(dst + q * 8, make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]));
    }
};
template <bool RELU>
struct Store32<float, RELU> {
    __device__ static void run(float* dst, const uint32_t (&r)[32], int cols_left) {
        if (cols_left >= 32 && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint4 v = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
                if (RELU) {
                    v.x = __float_as_uint(fmaxf(__uint_as_float(v.x), 0.0f));
                    v.y = __float_as_uint(fmaxf(__uint_as_float(v.y), 0.0f));
                    v.z = __float_as_uint(fmaxf(__uint_as_float(v.z), 0.0f));
                    v.w = __float_as_uint(fmaxf(__uint_as_float(v.w), 0.0f));
                }
                stg_v4(dst + 4 * q, v);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (i < cols_left) {
                    const float v = __uint_as_float(r[i]);
                    dst[i] = RELU ? (v > 0.0f ? v : 0.0f) : v;
                }
            }
        }
    }
};


// ------------------------------------------------------------ tensor maps --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (thread-safe static
// initialisation; null if the driver does not provide it).
static EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return static_cast<EncodeTiledFn>(nullptr);
    }();
    return fn;
}

// 2-D bf16 tensor [outer, inner] (inner contiguous), 128-byte swizzle, box
// [box_outer, box_inner] with box_inner * 2 <= 128 bytes.
static int make_tmap(CUtensorMap* m, const void* base, int inner, int outer, int box_outer,
                     int box_inner = BK) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return MOE_ERR_CUDA;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner),
                               static_cast<cuuint32_t>(box_outer)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// 3-D fp32 tensor [outer2][outer1][inner] (inner contiguous), 128-byte
// swizzle, box [1][box_rows][32] (one 128-byte row per box row).
static int make_tmap_f32_3d(CUtensorMap* m, const void* base, int inner, int outer1, int outer2,
                            int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return MOE_ERR_CUDA;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer1),
                                static_cast<cuuint64_t>(outer2)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * 4,
                                   static_cast<cuuint64_t>(inner) * 4 * outer1};
    const cuuint32_t box[3] = {32, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace tc
}  // namespace moe
