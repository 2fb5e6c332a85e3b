// gemm_bwd.cu -- grouped bf16 GEMMs of the expert FFN's backward pass on the
// tcgen05 tensor cores.
//
// PopFetcher, section 5.2.1: each expert GEMM of the forward pass has two in
// the backward pass, one for the input and one for the weights.  With dYp the
// gradient of the expert outputs and H the stored hidden activation:
//   dH  = (dYp . W2_e) * [H > 0]   rows of group e; B = W2_e read as [K=d][N=F]
//   dXp = dH . W1_e                rows of group e; B = W1_e read as [K=F][N=d]
//   dW2_e = dYp_e^T . H_e          [d x F], contracting over the group's rows
//   dW1_e = dH_e^T  . Xp_e         [F x d], contracting over the group's rows
// The weights are read in their forward layout, so the B operand is N-major
// (N contiguous in memory); the weight gradients take both operands N- or
// M-major from the activation rows.  MN-major tiles are 64 K-rows by 64
// MN-elements per TMA box (128 bytes with the 128-byte swizzle); a 256-wide
// operand is four such boxes 8 KB apart (the descriptor's leading byte
// offset), 8-row K groups 1 KB apart (stride byte offset).
//
// Same pipeline as the forward kernel (gemm_tc.cu): persistent CTAs, TMA
// producer warp, one MMA-issuing thread, four epilogue warps draining two TMEM
// accumulators, every wait bounded in time.  For the weight gradients a
// group's last K block can run past the group's rows; the MMA thread zeroes
// those K-rows of the A tile in shared memory before issuing (so the products
// with whatever B holds there vanish).  A group with no rows gets zero weight
// gradients.
#include "grouped.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moe {
namespace tc {
namespace bwd {

constexpr int BN = 256;
constexpr int kStages = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB, either major
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int MN_BOX = 64;                    // MN elements per box (128 bytes)
constexpr int MN_BOX_BYTES = MN_BOX * BK * 2;  // 8 KB
constexpr int fixed_bytes() { return kStages * STAGE_BYTES + 256 + 128 + 1024; }

enum Epi { EPI_BF16 = 0, EPI_BF16_RELU_MASK = 1, EPI_F32 = 2 };

// MN-major operand descriptor, 128-byte swizzle: 64-element MN atoms 8 KB
// apart, 8-row K groups 1 KB apart; +2 KB steps one K=16 slice.
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);      // start address
    d |= static_cast<uint64_t>(MN_BOX_BYTES >> 4) << 16;       // leading byte offset
    d |= static_cast<uint64_t>(1024 >> 4) << 32;               // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                       // descriptor version
    d |= static_cast<uint64_t>(2) << 61;                       // 128-byte swizzle
    return d;
}

__device__ __forceinline__ float bf(uint32_t u, int hi) { return hi ? bf16hi(u) : bf16lo(u); }

template <bool A_MN, bool KVAR, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
gemm_bwd_kernel(const __grid_constant__ CUtensorMap tmap_a,
                const __grid_constant__ CUtensorMap tmap_b, void* __restrict__ Cv,
                const __nv_bfloat16* __restrict__ Hmask, int M_fix, int N, int K_fix, int E,
                const int32_t* __restrict__ offsets, int R_max, int32_t* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~static_cast<uintptr_t>(1023u));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * A_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kStages * B_BYTES);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* tfull = empty + kStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* s_warp = reinterpret_cast<int32_t*>(bars) + 64;
    int32_t* s_prefix = s_warp + 32;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, kEpiThreads);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    pdl_wait();
    pdl_trigger();
    const int nt = (N + BN - 1) / BN;
    int total;
    int mt_fix = 0;
    if (KVAR) {
        mt_fix = (M_fix + BM - 1) / BM;
        total = E * mt_fix * nt;
        if (threadIdx.x == 0) {  // validate the offsets the K loops will follow
            for (int e = 0; e < E; ++e) {
                const int a = offsets[e], b = offsets[e + 1];
                if (a < 0 || b < a || b > R_max) flag_error(err, MOE_DEVERR_OFFSETS);
            }
        }
    } else {
        total = nt * build_tile_table(offsets, 0, E, 1, BM, R_max, s_prefix, s_warp, err);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // Tile coordinates.  Fixed K: rows of one group.  Per-group K: the output
    // block (m0, n0) of group e, K = the group's rows [a, a + rows).
    auto coord = [&](int tile, int& e, int& m0, int& rows, int& n0, int& k0, int& nk,
                     int& kr) {
        if (KVAR) {
            e = tile / (mt_fix * nt);
            const int local = tile - e * mt_fix * nt;
            const int mb = local % mt_fix, nb = local / mt_fix;
            m0 = mb * BM;
            rows = min(BM, M_fix - m0);
            n0 = nb * BN;
            int a = offsets[e], b = offsets[e + 1];
            if (a < 0 || b < a || b > R_max) b = a = 0;  // flagged above
            k0 = a;
            kr = b - a;
            nk = (kr + BK - 1) / BK;
        } else {
            const TileCoord c = tile_coord(tile, s_prefix, E, offsets, 0, BM, BN, nt);
            e = c.e;
            m0 = c.row0;
            rows = c.rows;
            n0 = c.n0;
            k0 = 0;
            kr = K_fix;
            nk = (K_fix + BK - 1) / BK;
        }
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)));
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)));
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
                int e, m0, rows, n0, k0, nk, kr;
                coord(tile, e, m0, rows, n0, k0, nk, kr);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* a_st = sA + stage * A_BYTES;
                    uint8_t* b_st = sB + stage * B_BYTES;
                    mbar_arrive_expect_tx(full + stage, STAGE_BYTES);
                    if (A_MN) {
                        // A rows are activation rows (K); M runs along them
                        for (int j = 0; j < BM / MN_BOX; ++j)
                            tma_load_2d(a_st + j * MN_BOX_BYTES, &tmap_a, full + stage,
                                        m0 + j * MN_BOX, k0 + kb * BK);
                    } else {
                        tma_load_2d(a_st, &tmap_a, full + stage, kb * BK, m0);
                    }
                    // B: K rows of the weight (group e's block) or of the activations
                    const int b_row = KVAR ? k0 + kb * BK : e * K_fix + kb * BK;
                    for (int j = 0; j < BN / MN_BOX; ++j)
                        tma_load_2d(b_st + j * MN_BOX_BYTES, &tmap_b, full + stage,
                                    n0 + j * MN_BOX, b_row);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                const long long n = issued < kStages ? issued : kStages;
                for (long long i = issued - n; i < issued; ++i)
                    mbar_wait(full + (int)(i % kStages), (uint32_t)((i / kStages) & 1), abort_flag,
                              err, false);
            }
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        // Lane 0 waits and issues; the whole warp zeroes the K-rows past a
        // group's end (weight gradients), so that neither operand carries the
        // next group's rows, or unwritten memory, into the sum.
        const uint32_t idesc =
            idesc_bf16(BM, BN) | (A_MN ? (1u << 15) : 0u) | (1u << 16);  // B is N-major
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int it = 0;
        for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
            int e, m0, rows, n0, k0, nk, kr;
            coord(tile, e, m0, rows, n0, k0, nk, kr);
            const int acc = it & 1;
            int w_ok = 1;
            if (lane == 0) w_ok = mbar_wait(tempty + acc, ((it >> 1) & 1) ^ 1u, abort_flag, err);
            if (!__shfl_sync(0xffffffffu, w_ok, 0)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
            for (int kb = 0; kb < nk; ++kb) {
                if (lane == 0) w_ok = mbar_wait(full + stage, phase, abort_flag, err);
                if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint8_t* a_st = sA + stage * A_BYTES;
                uint8_t* b_st = sB + stage * B_BYTES;
                const int valid = kr - kb * BK;
                if (KVAR && valid < BK) {
                    // A K-row (or B K-row) is 128 bytes of one box whatever
                    // the swizzle inside it: zero rows [valid, BK) of every box
                    const int per_box = (BK - valid) * 8;  // 16-byte chunks
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    for (int i = lane; i < (BM / MN_BOX + BN / MN_BOX) * per_box; i += 32) {
                        const int box = i / per_box, q = i - box * per_box;
                        uint8_t* base = box < BM / MN_BOX
                                            ? a_st + box * MN_BOX_BYTES
                                            : b_st + (box - BM / MN_BOX) * MN_BOX_BYTES;
                        reinterpret_cast<uint4*>(base + valid * 128)[q] = z;
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                }
                if (lane == 0) {
                    const uint32_t a0 = smem_u32(a_st);
                    const uint32_t b0 = smem_u32(b_st);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t ad =
                            A_MN ? sw128_mn_desc(a0 + kk * 2048) : sw128_desc(a0 + kk * 32);
                        mma_bf16(d_tmem, ad, sw128_mn_desc(b0 + kk * 2048), idesc,
                                 (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(empty + stage);
                }
                __syncwarp();
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok && lane == 0) mma_commit(tfull + acc);  // also for nk == 0 (nothing issued)
        }
        if (lane == 0) {
            mma_commit(drain);
            mbar_wait(drain, 0, abort_flag, err, false);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        int it = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
            int e, m0, rows, n0, k0, nk, kr;
            coord(tile, e, m0, rows, n0, k0, nk, kr);
            const int acc = it & 1;
            if (!mbar_wait(tfull + acc, (it >> 1) & 1, abort_flag, err)) break;
            tc_fence_after();
            const bool row_ok = row < rows;
#pragma unroll 1
            for (int cc = 0; cc < BN; cc += 32) {
                uint32_t r[32];
                tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(acc * BN + cc), r);
                const int col = n0 + cc;
                if (!row_ok || col >= N) continue;
                if (EPI == EPI_F32) {
                    float* dst = static_cast<float*>(Cv) +
                                 (static_cast<size_t>(e) * M_fix + m0 + row) * N + col;
                    if (nk == 0) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = 0u;  // group without rows
                    }
                    Store32<float, false>::run(dst, r, N - col);
                } else {
                    __nv_bfloat16* dst =
                        static_cast<__nv_bfloat16*>(Cv) + static_cast<size_t>(m0 + row) * N + col;
                    if (EPI == EPI_BF16_RELU_MASK) {
                        // dH = (dYp . W2) where the forward activation was positive
                        const uint4* h = reinterpret_cast<const uint4*>(
                            Hmask + static_cast<size_t>(m0 + row) * N + col);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if (q * 8 >= N - col) break;
                            const uint4 hv = ldg_nc_v4(h + q);
                            const uint32_t hu[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                if (!(bf(hu[i >> 1], i & 1) > 0.0f)) r[q * 8 + i] = 0u;
                        }
                    }
                    Store32<__nv_bfloat16, false>::run(dst, r, N - col);
                }
            }
            tc_fence_before();
            mbar_arrive(tempty + acc);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <bool A_MN, bool KVAR, int EPI>
int launch_bwd(const CUtensorMap& ta, const CUtensorMap& tb, void* C, const __nv_bfloat16* Hm,
               int M_fix, int N, int K_fix, int E, const int32_t* offsets, int R_max, long long ub,
               cudaStream_t st) {
    const int smem = fixed_bytes() + 4 * (E + 1);
    if (ensure_smem<gemm_bwd_kernel<A_MN, KVAR, EPI>>(smem) != MOE_OK) return MOE_ERR_CUDA;
    const int grid = (int)(ub < num_sms() ? ub : num_sms());
    if (grid <= 0) return MOE_OK;
    return launch_pdl(gemm_bwd_kernel<A_MN, KVAR, EPI>, grid, kThreads, smem, st, ta, tb, C, Hm,
                      M_fix, N, K_fix, E, offsets, R_max, device_error_word());
}

}  // namespace bwd
}  // namespace tc

// dH = (dYp . W2_e) * [H > 0] and dXp = dH . W1_e over the grouped rows, then
// dW2 = dYp_e^T H_e and dW1 = dH_e^T Xp_e per expert (fp32).
int launch_ffn_backward_bf16(const void* Xp, const void* H, const void* dYp, const void* W1,
                             const void* W2, int E, int d, int F, const int32_t* offsets,
                             int R_max, void* dH, void* dXp, float* dW1, float* dW2,
                             cudaStream_t st) {
    using namespace tc;
    using namespace tc::bwd;
    CUtensorMap a, b;
    const long long row_tiles = (long long)R_max / BM + E;
    // dH: A = dYp [R_max, d] K-major; B = W2 as [E*d rows (K), F (N)]
    if (make_tmap(&a, dYp, d, R_max, BM) != MOE_OK) return MOE_ERR_CUDA;
    if (make_tmap(&b, W2, F, E * d, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
    int rc = launch_bwd<false, false, EPI_BF16_RELU_MASK>(
        a, b, dH, static_cast<const __nv_bfloat16*>(H), 0, F, d, E, offsets, R_max,
        row_tiles * ((F + BN - 1) / BN), st);
    if (rc != MOE_OK) return rc;
    // dXp: A = dH [R_max, F] K-major; B = W1 as [E*F rows (K), d (N)]
    if (make_tmap(&a, dH, F, R_max, BM) != MOE_OK) return MOE_ERR_CUDA;
    if (make_tmap(&b, W1, d, E * F, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
    rc = launch_bwd<false, false, EPI_BF16>(a, b, dXp, nullptr, 0, d, F, E, offsets, R_max,
                                           row_tiles * ((d + BN - 1) / BN), st);
    if (rc != MOE_OK) return rc;
    if (dW2) {  // A = dYp rows as [K, M=d], B = H rows as [K, N=F]
        if (make_tmap(&a, dYp, d, R_max, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
        if (make_tmap(&b, H, F, R_max, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
        rc = launch_bwd<true, true, EPI_F32>(a, b, dW2, nullptr, d, F, 0, E, offsets, R_max,
                                             (long long)E * ((d + BM - 1) / BM) *
                                                 ((F + BN - 1) / BN),
                                             st);
        if (rc != MOE_OK) return rc;
    }
    if (dW1) {  // A = dH rows as [K, M=F], B = Xp rows as [K, N=d]
        if (make_tmap(&a, dH, F, R_max, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
        if (make_tmap(&b, Xp, d, R_max, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
        rc = launch_bwd<true, true, EPI_F32>(a, b, dW1, nullptr, F, d, 0, E, offsets, R_max,
                                             (long long)E * ((F + BM - 1) / BM) *
                                                 ((d + BN - 1) / BN),
                                             st);
        if (rc != MOE_OK) return rc;
    }
    return MOE_OK;
}

}  // namespace moe
