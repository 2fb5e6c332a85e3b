// gemm_tc.cu -- grouped bf16 GEMM on the 5th-generation tensor cores.
//
// Expert computation (PopFetcher, section 5.1: FC(d -> F), ReLU, FC(F -> d))
// over the contiguous per-expert row blocks of input encode ("A Survey on
// Mixture of Experts", section 5), and the gate projection as one group.
//
//   C[r][n] = act( sum_k A[r][k] * B_e[n][k] )   r in group e, fp32 accumulate
//
// A [R_max, K] and B [E*N, K] are bf16, K-major.  One persistent CTA per SM
// walks a static round-robin over the device-built tile table (grouped.cuh).
// Warp roles (192 threads):
//   warp 0     one lane issues TMA loads of 128x64 A and BNx64 B tiles (128-byte
//              swizzle) into a kStages-deep shared-memory ring;
//   warp 1     allocates TMEM; one lane issues tcgen05.mma (M=128, N=BN, K=16,
//              kind::f16, bf16 in, fp32 accumulate in TMEM) and tcgen05.commit
//              to free ring slots and publish finished accumulators;
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (one row per thread,
//              lane quadrant = warp % 4), ReLU, round to bf16 (or keep fp32),
//              row-masked 16-byte stores (rows past the group end belong to
//              the next group and are never written).
// Two TMEM accumulators (2 x BN columns) let the epilogue of tile i overlap the
// mainloop of tile i+1.
//
// Fused variants (ScatterMoE-style, "A Survey on Mixture of Experts",
// section 5; no dispatched copy of the tokens):
//   MODE_GATHER   the A tile's 128 rows are gathered straight from the token
//                 matrix x: grouped row r reads x[row_slot[r] / k], four rows
//                 per TMA tile::gather4 load, the 32 producer lanes issuing one
//                 each (rows past the group read out of bounds: zeros);
//   MODE_ROW_W    the epilogue scales grouped row r by its gate weight
//                 w[row_slot[r]] before rounding, so output decode becomes a
//                 plain sum of each token's rows.  Every mbarrier wait is bounded in time: on expiry the
// kernel flags MOE_DEVERR_TIMEOUT, drains its own TMA loads and MMAs, frees
// TMEM and returns.
#include "grouped.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moe {
namespace tc {

// Row capacity per expert (R_max / E) from which the FFN GEMMs use the 2-CTA
// kernel.
#ifndef MOE_PAIR_MIN_ROWS_PER_GROUP
#define MOE_PAIR_MIN_ROWS_PER_GROUP 1024
#endif
constexpr long long kPairMinRowsPerGroup = MOE_PAIR_MIN_ROWS_PER_GROUP;
// Dense groups: pair tiles for whole 256-row blocks plus 1-CTA tiles for the
// tails (0: pair tiles for everything).
#ifndef MOE_SPLIT_TAILS
#define MOE_SPLIT_TAILS 1
#endif
constexpr bool kSplitTails = MOE_SPLIT_TAILS != 0;


template <int BN>
struct Cfg {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    // ring depth: about 192 KB of stages in flight whatever the tile width
    static constexpr int STAGES = BN <= 64 ? 8 : (BN <= 128 ? 6 : 4);
    static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64
                                   : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
    // ring + barriers/flags (256 B) + warp scratch (128 B) + tile prefix + alignment slack
    static constexpr int fixed_bytes() { return STAGES * STAGE_BYTES + 256 + 128 + 1024; }
    static int smem_bytes(int E) { return fixed_bytes() + 4 * (E + 1); }
};

// -------------------------------------------------------------------- kernel
enum Mode { MODE_PLAIN = 0, MODE_GATHER = 1, MODE_ROW_W = 2 };

// Row-gather description for the fused modes: grouped row r is slot
// row_slot[r] = t * k + j of token t; w (MODE_ROW_W) is indexed by the slot.
struct Gather {
    const int32_t* row_slot;
    const float* w;
    int k, T;
};

__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y0, int y1, int y2, int y3) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y0), "r"(y1),
        "r"(y2), "r"(y3)
        : "memory");
}

template <int BN_MAX, bool RELU, typename TOut, int MODE = MODE_PLAIN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
               TOut* __restrict__ C, int N, int K, int E, const int32_t* __restrict__ offsets,
               int single_M, int R_max, Gather gat, int part, int32_t* err) {
    using G = Cfg<BN_MAX>;
    constexpr int S = G::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~static_cast<uintptr_t>(1023u));
    uint8_t* sA = smem;
    uint8_t* sB = smem + S * G::A_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + S * G::B_BYTES);
    uint64_t* full = bars;               // [S] TMA -> MMA
    uint64_t* empty = bars + S;          // [S] MMA -> TMA
    uint64_t* tfull = empty + S;         // [2] MMA -> epilogue
    uint64_t* tempty = tfull + 2;        // [2] epilogue -> MMA
    uint64_t* drain = tempty + 2;        // [1] final MMA completion
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* s_warp = reinterpret_cast<int32_t*>(bars) + 64;  // 256 B past the barriers
    int32_t* s_prefix = s_warp + 32;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
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
        tmem_alloc(tmem_slot, G::TMEM_COLS);
        tmem_relinquish();
    }
    pdl_wait();  // everything above touched only this CTA's on-chip state
    pdl_trigger();
    const int mtiles =
        build_tile_table(offsets, single_M, E, 1, BM, R_max, s_prefix, s_warp, err, part);
    constexpr int bn = BN_MAX;
    const int nt = (N + bn - 1) / bn;
    const int total = mtiles * nt;
    const uint32_t stage_tx = G::A_BYTES + bn * BK * 2;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int nk = (K + BK - 1) / BK;

    if (warp == 0 && MODE == MODE_GATHER) {
        // -------------------------------------------- TMA producer (gather)
        // lane l owns tile rows 4l .. 4l+3: their x rows are looked up once
        // per tile, then every k-block each lane issues one gather4
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)));
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)));
        }
        int stage = 0;
        uint32_t phase = 0;
        long long issued = 0;
        bool ok = true;
        const int n_slots = gat.T * gat.k;
        const int first = test_stall() ? total : blockIdx.x;
        for (int tile = first; ok && tile < total; tile += gridDim.x) {
            const TileCoord c = tile_coord(tile, s_prefix, E, offsets, single_M, BM, bn, nt, part);
            const int b_row = c.e * N + c.n0;
            int xr[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = 4 * lane + j;
                xr[j] = gat.T;  // out of bounds: the TMA fills zeros
                if (i < c.rows) {
                    const int slot = __ldg(gat.row_slot + c.row0 + i);
                    if (slot >= 0 && slot < n_slots) xr[j] = slot / gat.k;
                    else flag_error(err, MOE_DEVERR_ROW_INDEX);
                }
            }
            for (int kb = 0; kb < nk; ++kb) {
                int w_ok = 1;
                if (lane == 0) {
                    w_ok = mbar_wait(empty + stage, phase ^ 1u, abort_flag, err);
                    if (w_ok) mbar_arrive_expect_tx(full + stage, stage_tx);
                }
                if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
                    ok = false;
                    break;
                }
                tma_gather4(sA + stage * G::A_BYTES + lane * 512, &tmap_a, full + stage, kb * BK,
                            xr[0], xr[1], xr[2], xr[3]);
                if (lane == 0)
                    tma_load_2d(sB + stage * G::B_BYTES, &tmap_b, full + stage, kb * BK, b_row);
                ++issued;
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            const long long n = issued < S ? issued : S;
            for (long long i = issued - n; i < issued; ++i)
                mbar_wait(full + (int)(i % S), (uint32_t)((i / S) & 1), abort_flag, err, false);
        }
    } else if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            const CUtensorMap* mb = &tmap_b;
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)));
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(mb)));
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            const int first = test_stall() ? total : blockIdx.x;
            for (int tile = first; ok && tile < total; tile += gridDim.x) {
                const TileCoord c = tile_coord(tile, s_prefix, E, offsets, single_M, BM, bn, nt, part);
                const int b_row = c.e * N + c.n0;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full + stage, stage_tx);
                    tma_load_2d(sA + stage * G::A_BYTES, &tmap_a, full + stage, kb * BK, c.row0);
                    tma_load_2d(sB + stage * G::B_BYTES, mb, full + stage, kb * BK, b_row);
                    ++issued;
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // Let the loads already issued land before the CTA exits.
                const long long n = issued < S ? issued : S;
                for (long long i = issued - n; i < issued; ++i)
                    mbar_wait(full + (int)(i % S), (uint32_t)((i / S) & 1), abort_flag, err, false);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            const uint32_t idesc = idesc_bf16(BM, bn);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int it = 0;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                if (!mbar_wait(tempty + acc, ((it >> 1) & 1) ^ 1u, abort_flag, err)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN_MAX);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(full + stage, phase, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * G::A_BYTES);
                    const uint32_t b0 = smem_u32(sB + stage * G::B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_bf16(d_tmem, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc,
                                 (kb | kk) != 0 ? 1u : 0u);
                    mma_commit(empty + stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) mma_commit(tfull + acc);
            }
            // all MMAs this thread issued are complete once `drain` fires
            mma_commit(drain);
            mbar_wait(drain, 0, abort_flag, err, false);
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        int it = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
            const TileCoord c = tile_coord(tile, s_prefix, E, offsets, single_M, BM, bn, nt, part);
            const int acc = it & 1;
            if (!mbar_wait(tfull + acc, (it >> 1) & 1, abort_flag, err)) break;
            tc_fence_after();
            const bool row_ok = row < c.rows;
            TOut* crow = C + static_cast<size_t>(c.row0 + (row_ok ? row : 0)) * N;
            float wr = 1.0f;  // MODE_ROW_W: this row's gate weight
            if (MODE == MODE_ROW_W && row_ok) {
                const int slot = __ldg(gat.row_slot + c.row0 + row);
                if (slot >= 0 && slot < gat.T * gat.k) wr = __ldg(gat.w + slot);
                else flag_error(err, MOE_DEVERR_ROW_INDEX);
            }
#pragma unroll 1
            for (int cc = 0; cc < bn; cc += 32) {
                uint32_t r[32];
                tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(acc * BN_MAX + cc), r);
                if (MODE == MODE_ROW_W) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        r[i] = __float_as_uint(__fmul_rn(wr, __uint_as_float(r[i])));
                }
                const int col = c.n0 + cc;
                if (row_ok && col < N) Store32<TOut, RELU>::run(crow + col, r, N - col);
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
        tmem_dealloc(tmem_base, G::TMEM_COLS);
    }
}

// ----------------------------------------------------- 2-CTA (cta_group::2)
// A cluster of two CTAs on one TPC computes a 256 x 256 tile: CTA r loads rows
// [128r, 128r+128) of A and rows [128r, 128r+128) of the N-slice of B into its
// own ring; the leader (r = 0) issues tcgen05.mma.cta_group::2 (M=256, N=256),
// which reads both CTAs' shared memory and writes each CTA's 128 rows into that
// CTA's TMEM.  Each CTA streams half the B bytes of a 1-CTA 128x256 tile for
// the same MMA work, so a 6-deep ring fits and hides more latency.
//
// The same kernel serves the input gradients of the expert backward
// (B_MN: B read N-major, as the forward weights lie: [E*K rows][N], each CTA's
// 128 columns as two 64 x 64 boxes; MASK: the result zeroed where the forward
// activation Hmask was not positive, for dH = (dYp . W2_e) * [H > 0]).
namespace pair {

constexpr int kStages = 6;
constexpr int BM = 256;       // rows per pair tile (128 per CTA)
constexpr int BN = 256;
constexpr int HALF = 128;
constexpr int A_BYTES = HALF * BK * 2;   // 16 KB
constexpr int B_BYTES = HALF * BK * 2;   // 16 KB (half of the N slice)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;           // two 256-column accumulators
constexpr int fixed_bytes() { return kStages * STAGE_BYTES + 256 + 128 + 1024; }
inline int smem_bytes(int E) { return fixed_bytes() + 4 * (E + 1); }

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void remote_arrive(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t leader_bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives once on the barrier at this offset in both CTAs of the pair when all
// tcgen05 operations issued so far by this thread have completed.
__device__ __forceinline__ void commit_both(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

template <bool RELU, bool B_MN = false, bool MASK = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmap_a,
                const __grid_constant__ CUtensorMap tmap_b, __nv_bfloat16* __restrict__ C, int N,
                int K, int E, const int32_t* __restrict__ offsets, int R_max, int part,
                const __nv_bfloat16* __restrict__ Hmask, int32_t* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~static_cast<uintptr_t>(1023u));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * A_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kStages * B_BYTES);
    uint64_t* full = bars;               // [kStages] (leader's is the one signalled)
    uint64_t* empty = bars + kStages;    // [kStages] per CTA, both signalled by the leader
    uint64_t* tfull = empty + kStages;   // [2] per CTA, both signalled by the leader
    uint64_t* tempty = tfull + 2;        // [2] leader's, 2 x 128 epilogue arrivals
    uint64_t* drain = tempty + 2;        // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* s_warp = reinterpret_cast<int32_t*>(bars) + 64;
    int32_t* s_prefix = s_warp + 32;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, 2 * kEpiThreads);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    pdl_wait();  // everything above touched only this CTA's on-chip state
    pdl_trigger();
    const int pair_id = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int mtiles = build_tile_table(offsets, 0, E, 1, BM, R_max, s_prefix, s_warp, err, part);
    constexpr int bn = BN;
    const int nt = (N + bn - 1) / bn;
    const int total = mtiles * nt;
    const int b_half = bn / 2;  // B rows each CTA loads
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers exist before either signals the other
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int nk = (K + BK - 1) / BK;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer (both CTAs)
            const CUtensorMap* mb = &tmap_b;
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)));
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(mb)));
            const uint32_t pair_tx = 2u * (A_BYTES + b_half * BK * 2);
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            const int first = test_stall() ? total : pair_id;
            for (int tile = first; ok && tile < total; tile += npairs) {
                const TileCoord c = tile_coord(tile, s_prefix, E, offsets, 0, BM, bn, nt, part);
                const int a_row = c.row0 + HALF * (int)rank;
                const int b_row = c.e * N + c.n0 + b_half * (int)rank;  // K-major B
                const int b_col = c.n0 + b_half * (int)rank;            // N-major B
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t lbar = map_to(smem_u32(full + stage), 0);
                    if (leader) mbar_arrive_expect_tx(full + stage, pair_tx);
                    tma_load_2d_pair(sA + stage * A_BYTES, &tmap_a, lbar, kb * BK, a_row);
                    if constexpr (B_MN) {
                        // K rows c.e*K + kb*BK.. of the weight, this CTA's 128 columns
                        const int k_row = c.e * K + kb * BK;
                        tma_load_2d_pair(sB + stage * B_BYTES, mb, lbar, b_col, k_row);
                        tma_load_2d_pair(sB + stage * B_BYTES + kMnAtomBytes, mb, lbar,
                                         b_col + 64, k_row);
                    } else {
                        tma_load_2d_pair(sB + stage * B_BYTES, mb, lbar, kb * BK, b_row);
                    }
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                if (leader) {
                    // The leader's full barriers count both CTAs' bytes.
                    const long long n = issued < kStages ? issued : kStages;
                    for (long long i = issued - n; i < issued; ++i)
                        mbar_wait(full + (int)(i % kStages), (uint32_t)((i / kStages) & 1),
                                  abort_flag, err, false);
                } else {
                    // The peer cannot observe its loads' completion: give them time to land.
                    const unsigned long long t0 = globaltimer();
                    while (globaltimer() - t0 < 200000ull) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issuer (leader only)
            const uint32_t idesc = idesc_bf16(BM, bn) | (B_MN ? (1u << 16) : 0u);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int it = 0;
            for (int tile = pair_id; ok && tile < total; tile += npairs, ++it) {
                const int acc = it & 1;
                if (!mbar_wait(tempty + acc, ((it >> 1) & 1) ^ 1u, abort_flag, err)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(full + stage, phase, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
                    const uint32_t b0 = smem_u32(sB + stage * B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_pair(d_tmem, sw128_desc(a0 + kk * 32),
                                 B_MN ? sw128_mn_desc(b0 + kk * 2048) : sw128_desc(b0 + kk * 32),
                                 idesc, (kb | kk) != 0 ? 1u : 0u);
                    commit_both(empty + stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) commit_both(tfull + acc);
            }
            commit_both(drain);
            mbar_wait(drain, 0, abort_flag, err, false);
        }
    } else {
        // ---------------------------------------------------- epilogue (both CTAs)
        const int quad = warp & 3;
        const int row = quad * 32 + lane;  // row inside this CTA's half
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        int it = 0;
        for (int tile = pair_id; tile < total; tile += npairs, ++it) {
            const TileCoord c = tile_coord(tile, s_prefix, E, offsets, 0, BM, bn, nt, part);
            const int acc = it & 1;
            if (!mbar_wait(tfull + acc, (it >> 1) & 1, abort_flag, err)) break;
            tc_fence_after();
            const int r_tile = HALF * (int)rank + row;  // row inside the 256-row tile
            const bool row_ok = r_tile < c.rows;
            __nv_bfloat16* crow = C + static_cast<size_t>(c.row0 + (row_ok ? r_tile : 0)) * N;
            // MASK: bit i of hm[w] says column c.n0 + 32 w + i of this row has H > 0
            uint32_t hm[BN / 32];
#pragma unroll
            for (int w = 0; w < BN / 32; ++w) hm[w] = 0u;
            if constexpr (MASK) {
                if (row_ok) {
                    const uint4* h = reinterpret_cast<const uint4*>(
                        Hmask + static_cast<size_t>(c.row0 + r_tile) * N + c.n0);
                    const int nv = min(BN, N - c.n0) / 8;
#pragma unroll
                    for (int w = 0; w < BN / 32; ++w) {
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) {
                            const int q = 4 * w + qq;
                            const uint4 v = q < nv ? ldg_nc_v4(h + q) : make_uint4(0, 0, 0, 0);
                            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
                            uint32_t bits = 0;
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                bits |= ((i & 1 ? bf16hi(u[i >> 1]) : bf16lo(u[i >> 1])) > 0.0f
                                             ? 1u : 0u) << i;
                            hm[w] |= bits << (qq * 8);
                        }
                    }
                }
            }
#pragma unroll 1
            for (int cc = 0; cc < bn; cc += 32) {
                uint32_t r[32];
                tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(acc * BN + cc), r);
                const int col = c.n0 + cc;
                if constexpr (MASK) {
                    const uint32_t mw = hm[0];  // this 32-column block's bits
#pragma unroll
                    for (int w = 0; w + 1 < BN / 32; ++w) hm[w] = hm[w + 1];
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (!((mw >> i) & 1u)) r[i] = 0u;
                }
                if (row_ok && col < N) Store32<__nv_bfloat16, RELU>::run(crow + col, r, N - col);
            }
            tc_fence_before();
            remote_arrive(map_to(smem_u32(tempty + acc), 0));
        }
    }

    tc_fence_before();
    __syncthreads();
    __syncwarp();
    cluster_sync();  // no CTA frees TMEM or exits while its peer may still touch it
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

}  // namespace pair

// -------------------------------------------------------------------- host --
template <int BN, bool RELU, typename TOut, int MODE = MODE_PLAIN>
static int launch(const void* A, const void* B, TOut* C, int N, int K, int E,
                  const int32_t* offsets, int single_M, int R_max, cudaStream_t st,
                  Gather gat = Gather{nullptr, nullptr, 1, 0}, int part = PART_ALL) {
    using G = Cfg<BN>;
    if (R_max <= 0 || N <= 0) return MOE_OK;
    CUtensorMap ta, tb;
    if (MODE == MODE_GATHER) {  // A = the token matrix x [T, K], one-row boxes
        if (make_tmap(&ta, A, K, gat.T, 1) != MOE_OK) return MOE_ERR_CUDA;
    } else if (make_tmap(&ta, A, K, R_max, BM) != MOE_OK) {
        return MOE_ERR_CUDA;
    }
    if (make_tmap(&tb, B, K, E * N, BN) != MOE_OK) return MOE_ERR_CUDA;
    const int smem = G::smem_bytes(E);
    auto kern = gemm_tc_kernel<BN, RELU, TOut, MODE>;
    if (ensure_smem<gemm_tc_kernel<BN, RELU, TOut, MODE>>(smem) != MOE_OK) return MOE_ERR_CUDA;
    const int nt = (N + BN - 1) / BN;
    // tiles, upper bound (a tail part has at most kSplitRows / BM tiles per group)
    const long long ub = part == PART_TAIL ? (long long)E * (kSplitRows / BM) * nt
                                           : ((long long)R_max / BM + E) * nt;
    const int grid = test_cap((int)(ub < num_sms() ? ub : num_sms()));
    return launch_pdl(kern, grid, kThreads, smem, st, ta, tb, C, N, K, E, offsets, single_M, R_max,
                      gat, part, device_error_word());
}

template <bool RELU>
static int launch_pair(const void* A, const void* B, __nv_bfloat16* C, int N, int K, int E,
                       const int32_t* offsets, int R_max, cudaStream_t st, int part = PART_ALL) {
    if (R_max <= 0 || N <= 0) return MOE_OK;
    CUtensorMap ta, tb;
    if (make_tmap(&ta, A, K, R_max, pair::HALF) != MOE_OK) return MOE_ERR_CUDA;
    if (make_tmap(&tb, B, K, E * N, pair::HALF) != MOE_OK) return MOE_ERR_CUDA;
    const int smem = pair::smem_bytes(E);
    auto kern = pair::gemm_tc2_kernel<RELU>;
    if (ensure_smem<pair::gemm_tc2_kernel<RELU>>(smem) != MOE_OK) return MOE_ERR_CUDA;
    const int nt = (N + pair::BN - 1) / pair::BN;
    const long long ub = ((long long)R_max / pair::BM + E) * nt;  // pair tiles, upper bound
    const int pairs_max = num_sms() / 2;
    int pairs = (int)(ub < pairs_max ? ub : pairs_max);
    pairs = test_cap(2 * pairs) / 2 > 0 ? test_cap(2 * pairs) / 2 : 1;
    return launch_pdl(kern, 2 * pairs, kThreads, smem, st, ta, tb, C, N, K, E, offsets, R_max,
                      part, static_cast<const __nv_bfloat16*>(nullptr), device_error_word());
}

// Pair tiles with the weights read N-major: C[rows of group e] = A . B_e with
// B_e rows [e*K, e*K + K) of a [E*K, N] matrix, optionally masked by Hmask > 0.
template <bool MASK>
static int launch_pair_nmajor(const void* A, const void* B, __nv_bfloat16* C, int N, int K,
                              int E, const int32_t* offsets, int R_max, const void* Hmask,
                              cudaStream_t st) {
    if (R_max <= 0 || N <= 0) return MOE_OK;
    CUtensorMap ta, tb;
    if (make_tmap(&ta, A, K, R_max, pair::HALF) != MOE_OK) return MOE_ERR_CUDA;
    if (make_tmap(&tb, B, N, E * K, BK, 64) != MOE_OK) return MOE_ERR_CUDA;
    const int smem = pair::smem_bytes(E);
    auto kern = pair::gemm_tc2_kernel<false, true, MASK>;
    if (ensure_smem<pair::gemm_tc2_kernel<false, true, MASK>>(smem) != MOE_OK) return MOE_ERR_CUDA;
    const int nt = (N + pair::BN - 1) / pair::BN;
    const long long ub = ((long long)R_max / pair::BM + E) * nt;
    const int pairs_max = num_sms() / 2;
    int pairs = (int)(ub < pairs_max ? ub : pairs_max);
    pairs = test_cap(2 * pairs) / 2 > 0 ? test_cap(2 * pairs) / 2 : 1;
    return launch_pdl(kern, 2 * pairs, kThreads, smem, st, ta, tb, C, N, K, E, offsets, R_max,
                      (int)PART_ALL, static_cast<const __nv_bfloat16*>(Hmask),
                      device_error_word());
}

}  // namespace tc

#ifdef MOE_TEST_HOOKS
int test_stall_tc(int v) { return tc::set_test_stall(v); }
#endif

bool gemm_pair_tiles(int R_max, int E, int N) {
    const long long tiles_1cta = ((long long)R_max / tc::BM + E) * ((N + 255) / 256);
    return (long long)R_max >= tc::kPairMinRowsPerGroup * (long long)E ||
           tiles_1cta < 3LL * num_sms();
}

int launch_gemm_pair_nmajor_bf16(const void* A, const void* B, void* C, int N, int K, int E,
                                 const int32_t* offsets, int R_max, const void* Hmask,
                                 cudaStream_t st) {
    __nv_bfloat16* Cb = static_cast<__nv_bfloat16*>(C);
    if (Hmask)
        return tc::launch_pair_nmajor<true>(A, B, Cb, N, K, E, offsets, R_max, Hmask, st);
    return tc::launch_pair_nmajor<false>(A, B, Cb, N, K, E, offsets, R_max, nullptr, st);
}

int launch_gemm_tc_bf16(const void* A, const void* B, void* C, bool out_f32, int N, int K, int E,
                        const int32_t* offsets, int single_M, int R_max, bool relu,
                        cudaStream_t st) {
    using namespace tc;
    if (out_f32) {
        float* Cf = static_cast<float*>(C);
        if (relu) return MOE_ERR_UNSUPPORTED;
        if (N <= 32) return launch<32, false, float>(A, B, Cf, N, K, E, offsets, single_M, R_max, st);
        if (N <= 64) return launch<64, false, float>(A, B, Cf, N, K, E, offsets, single_M, R_max, st);
        if (N <= 128) return launch<128, false, float>(A, B, Cf, N, K, E, offsets, single_M, R_max, st);
        return launch<256, false, float>(A, B, Cf, N, K, E, offsets, single_M, R_max, st);
    }
    __nv_bfloat16* Cb = static_cast<__nv_bfloat16*>(C);
    // Dense groups (many rows per expert on average) take the 2-CTA 256-row
    // tiles; sparse ones keep 128-row tiles, which waste fewer padded rows --
    // unless the 128-row tiles would fill fewer than three waves of SMs, where
    // halving each SM's weight traffic outweighs the padding (measured on one
    // B200: the skewed_drops second GEMM, 1.2 waves, 63.2 -> 58.7 us; its first
    // GEMM, 8.6 waves, and both multistep_window GEMMs are slower with pairs).
    const long long tiles_1cta = ((long long)R_max / BM + E) * ((N + 255) / 256);
    const bool dense = (long long)R_max >= (long long)kPairMinRowsPerGroup * E;
    if (offsets != nullptr && dense && kSplitTails) {
        // whole 256-row blocks of every group on pair tiles, then the rows
        // after them on 128-row tiles: a group pads to 128 rows, not 256
        int rc = relu ? launch_pair<true>(A, B, Cb, N, K, E, offsets, R_max, st, PART_BLOCKS)
                      : launch_pair<false>(A, B, Cb, N, K, E, offsets, R_max, st, PART_BLOCKS);
        if (rc != MOE_OK) return rc;
        const Gather none{nullptr, nullptr, 1, 0};
        if (relu)
            return launch<256, true, __nv_bfloat16>(A, B, Cb, N, K, E, offsets, 0, R_max, st, none,
                                                     PART_TAIL);
        return launch<256, false, __nv_bfloat16>(A, B, Cb, N, K, E, offsets, 0, R_max, st, none,
                                                  PART_TAIL);
    }
    if (offsets != nullptr && (dense || tiles_1cta < 3LL * num_sms())) {
        if (relu) return launch_pair<true>(A, B, Cb, N, K, E, offsets, R_max, st);
        return launch_pair<false>(A, B, Cb, N, K, E, offsets, R_max, st);
    }
    if (relu) return launch<256, true, __nv_bfloat16>(A, B, Cb, N, K, E, offsets, single_M, R_max, st);
    return launch<256, false, __nv_bfloat16>(A, B, Cb, N, K, E, offsets, single_M, R_max, st);
}

int launch_ffn_gather_bf16(const void* x, int T, int k, const int32_t* row_slot, const float* w,
                           const void* W1, const void* W2, int E, int d, int F,
                           const int32_t* offsets, int R_max, void* H, void* Yp,
                           cudaStream_t st) {
    using namespace tc;
    const Gather g{row_slot, w, k, T};
    __nv_bfloat16* Hb = static_cast<__nv_bfloat16*>(H);
    __nv_bfloat16* Yb = static_cast<__nv_bfloat16*>(Yp);
    int rc = launch<256, true, __nv_bfloat16, MODE_GATHER>(x, W1, Hb, F, d, E, offsets, 0, R_max,
                                                           st, g);
    if (rc != MOE_OK) return rc;
    if (w != nullptr)
        return launch<256, false, __nv_bfloat16, MODE_ROW_W>(H, W2, Yb, d, F, E, offsets, 0,
                                                             R_max, st, g);
    return launch<256, false, __nv_bfloat16>(H, W2, Yb, d, F, E, offsets, 0, R_max, st);
}

}  // namespace moe
