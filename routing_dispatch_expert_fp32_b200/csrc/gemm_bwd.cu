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
// producer warp, one MMA-issuing thread, eight epilogue warps draining two TMEM
// accumulators, every wait bounded in time.  For the weight gradients a
// group's last K block can run past the group's rows: its 16-row MMA steps
// past the end are not issued, and in the step where the group ends the MMA
// warp zeroes the remaining K-rows of A (and of B where they lie past the last
// group, rows nobody wrote) in shared memory, so that nothing outside the
// group enters the sum.  A group with no rows gets zero weight gradients.
// The fp32 weight-gradient tiles leave through shared memory and tensor
// stores; the bf16 outputs (dH, dXp) are stored row by row, masked to the
// group.  The same kernel, with a K loop over three planes of A, computes the
// bf16 gate backward from dlogits split exactly into three bf16 planes.
#include <cstring>

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
// Epilogue warps: two per TMEM lane quadrant, each draining half of the 256
// accumulator columns (4: one per quadrant, all columns).  The weight-gradient
// tiles have short K loops, so a tile's time is mostly its epilogue.
#ifndef MOE_BWD_EPI_WARPS
#define MOE_BWD_EPI_WARPS 8
#endif
constexpr int kEpiWarps = MOE_BWD_EPI_WARPS;
static_assert(kEpiWarps == 4 || kEpiWarps == 8, "epilogue warps");
constexpr int kBwdThreads = 64 + 32 * kEpiWarps;  // TMA warp, MMA warp, epilogue
constexpr int kBwdEpiThreads = 32 * kEpiWarps;
constexpr int kColsPerWarp = BN / (kEpiWarps / 4);
// fp32 epilogue: per warp kEpiBufs staging tiles of 32 rows x 32 columns,
// written in turn while earlier tensor stores drain; the operand ring gives
// up one stage for them (64 KB in all).
constexpr int kEpiBufs = kEpiWarps == 8 ? 2 : 4;
constexpr int EPI_STAGE_BYTES = kEpiWarps * kEpiBufs * 32 * 128;
constexpr int stages_for(int EPI) { return EPI == 2 ? 3 : kStages; }
template <int EPI>
constexpr int fixed_bytes() {
    return stages_for(EPI) * STAGE_BYTES + (EPI == 2 ? EPI_STAGE_BYTES : 0) + 256 + 128 + 1024;
}

enum Epi { EPI_BF16 = 0, EPI_BF16_RELU_MASK = 1, EPI_F32 = 2, EPI_BF16_ADD = 3 };

// Input gradients of dense groups on the forward pass's 2-CTA pair tiles
// (gemm_tc.cu; 0: the 1-CTA kernel below for every layout).
#ifndef MOE_BWD_PAIR
#define MOE_BWD_PAIR 1
#endif
constexpr bool kBwdPair = MOE_BWD_PAIR != 0;

// Problem description of one launch.
//   Fixed K: groups of rows from `offsets` (or one group of single_M rows
//   when offsets is null), K = K_fix, B rows e*K_fix + k.
//   Per-group K: output [E][M_fix][N], K = the rows of group e, from
//   `offsets` or, when null, consecutive slices of slice_rows rows of
//   single_M rows in all.
//   planes > 1: the K loop runs `planes` times, the A coordinate along the
//   rows moved by plane_rows each time, B unchanged (A = several row blocks
//   that all multiply the same B and add into one result).
struct BwdArgs {
    void* C;
    const __nv_bfloat16* Hmask;
    int M_fix, N, K_fix, E;
    const int32_t* offsets;
    int single_M, R_max, planes, plane_rows, slice_rows;
};

__device__ __forceinline__ float bf(uint32_t u, int hi) { return hi ? bf16hi(u) : bf16lo(u); }

template <bool A_MN, bool KVAR, int EPI>
__global__ void __launch_bounds__(kBwdThreads, 1)
gemm_bwd_kernel(const __grid_constant__ CUtensorMap tmap_a,
                const __grid_constant__ CUtensorMap tmap_b,
                const __grid_constant__ CUtensorMap tmap_c, const BwdArgs args, int32_t* err) {
    void* __restrict__ Cv = args.C;
    const __nv_bfloat16* __restrict__ Hmask = args.Hmask;
    const int M_fix = args.M_fix, N = args.N, K_fix = args.K_fix, E = args.E;
    const int32_t* __restrict__ offsets = args.offsets;
    const int single_M = args.single_M, R_max = args.R_max, planes = args.planes;
    const int plane_rows = args.plane_rows, slice_rows = args.slice_rows;
    constexpr int kS = stages_for(EPI);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~static_cast<uintptr_t>(1023u));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kS * A_BYTES;
    uint8_t* sC = sB + kS * B_BYTES;  // fp32 epilogue staging (1024-byte aligned)
    uint64_t* bars =
        reinterpret_cast<uint64_t*>(sC + (EPI == EPI_F32 ? EPI_STAGE_BYTES : 0));
    uint64_t* full = bars;
    uint64_t* empty = bars + kS;
    uint64_t* tfull = empty + kS;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* s_warp = reinterpret_cast<int32_t*>(bars) + 64;
    int32_t* s_prefix = s_warp + 32;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kS; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, kBwdEpiThreads);
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
        // the group bounds every role reads per tile, kept in shared memory
        for (int i = threadIdx.x; i <= E; i += kBwdThreads)
            s_prefix[i] = offsets ? offsets[i] : min(single_M, i * slice_rows);
        if (offsets && threadIdx.x == 0) {  // validate the offsets the K loops will follow
            for (int e = 0; e < E; ++e) {
                const int a = offsets[e], b = offsets[e + 1];
                if (a < 0 || b < a || b > R_max) flag_error(err, MOE_DEVERR_OFFSETS);
            }
        }
    } else {
        total =
            nt * build_tile_table(offsets, single_M, E, 1, BM, R_max, s_prefix, s_warp, err);
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
            int a = s_prefix[e], b = s_prefix[e + 1];
            if (a < 0 || b < a || b > R_max) b = a = 0;  // flagged above
            k0 = a;
            kr = b - a;
            nk = (kr + BK - 1) / BK;
        } else {
            const TileCoord c = tile_coord(tile, s_prefix, E, offsets, single_M, BM, BN, nt);
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
            const int first = test_stall() ? total : blockIdx.x;
            for (int tile = first; ok && tile < total; tile += gridDim.x) {
                int e, m0, rows, n0, k0, nk, kr;
                coord(tile, e, m0, rows, n0, k0, nk, kr);
                for (int b = 0; b < planes * nk; ++b) {
                    const int pl = b / nk, kb = b - pl * nk;
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
                                        m0 + j * MN_BOX, pl * plane_rows + k0 + kb * BK);
                    } else {
                        tma_load_2d(a_st, &tmap_a, full + stage, kb * BK, pl * plane_rows + m0);
                    }
                    // B: K rows of the weight (group e's block) or of the activations
                    const int b_row = KVAR ? k0 + kb * BK : e * K_fix + kb * BK;
                    for (int j = 0; j < BN / MN_BOX; ++j)
                        tma_load_2d(b_st + j * MN_BOX_BYTES, &tmap_b, full + stage,
                                    n0 + j * MN_BOX, b_row);
                    ++issued;
                    if (++stage == kS) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                const long long n = issued < kS ? issued : kS;
                for (long long i = issued - n; i < issued; ++i)
                    mbar_wait(full + (int)(i % kS), (uint32_t)((i / kS) & 1), abort_flag,
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
            for (int b = 0; b < planes * nk; ++b) {
                const int kb = b % nk;
                if (lane == 0) w_ok = mbar_wait(full + stage, phase, abort_flag, err);
                if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint8_t* a_st = sA + stage * A_BYTES;
                uint8_t* b_st = sB + stage * B_BYTES;
                const int valid = kr - kb * BK;
                int nsub = BK / 16;  // MMA steps of 16 K-rows this k-block issues
                if (KVAR && valid < BK) {
                    // the group ends inside this block: steps past its end are
                    // skipped; in the step it ends in, K-rows [valid, 16*nsub)
                    // are zeroed in A (each K-row is 128 bytes of one box,
                    // whatever the swizzle inside it), and in B too where the
                    // rows lie past the last group (rows no one wrote); other B
                    // rows there belong to the next group, finite, and meet
                    // zeros in A
                    nsub = (valid + 15) / 16;
                    const int zr = nsub * 16 - valid;  // rows to zero
                    if (zr > 0) {
                        const bool past_end = k0 + kb * BK + nsub * 16 > s_prefix[E];
                        const int per_box = zr * 8;  // 16-byte chunks
                        const int nbox = BM / MN_BOX + (past_end ? BN / MN_BOX : 0);
                        const uint4 z = make_uint4(0, 0, 0, 0);
                        for (int i = lane; i < nbox * per_box; i += 32) {
                            const int box = i / per_box, q = i - box * per_box;
                            uint8_t* base = box < BM / MN_BOX
                                                ? a_st + box * MN_BOX_BYTES
                                                : b_st + (box - BM / MN_BOX) * MN_BOX_BYTES;
                            reinterpret_cast<uint4*>(base + valid * 128)[q] = z;
                        }
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    }
                    __syncwarp();
                }
                if (lane == 0) {
                    const uint32_t a0 = smem_u32(a_st);
                    const uint32_t b0 = smem_u32(b_st);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        if (kk >= nsub) break;
                        const uint64_t ad =
                            A_MN ? sw128_mn_desc(a0 + kk * 2048) : sw128_desc(a0 + kk * 32);
                        mma_bf16(d_tmem, ad, sw128_mn_desc(b0 + kk * 2048), idesc,
                                 (b | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(empty + stage);
                }
                __syncwarp();
                if (++stage == kS) {
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
        // warp 2 + ew drains TMEM lane quadrant warp % 4 (a warp's fixed
        // quadrant), columns [c_lo, c_lo + kColsPerWarp) of the accumulator
        const int ew = warp - 2;
        const int quad = warp & 3;
        const int c_lo = (ew >> 2) * kColsPerWarp;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        uint8_t* stage_c = sC + ew * (kEpiBufs * 4096);  // this warp's staging tiles
        int it = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
            int e, m0, rows, n0, k0, nk, kr;
            coord(tile, e, m0, rows, n0, k0, nk, kr);
            const int acc = it & 1;
            const bool row_ok = row < rows;
            // dH: the ReLU mask of this row's columns, as bits, loaded from H
            // while the tile's MMAs still run (bit i of word w: column
            // n0 + c_lo + 32 w + i has H > 0)
            uint32_t hm[kColsPerWarp / 32];
#pragma unroll
            for (int w = 0; w < kColsPerWarp / 32; ++w) hm[w] = 0u;
            if (EPI == EPI_BF16_RELU_MASK && row_ok) {
                const uint4* h = reinterpret_cast<const uint4*>(
                    Hmask + static_cast<size_t>(m0 + row) * N + n0 + c_lo);
                const int nv = min(kColsPerWarp, N - n0 - c_lo) / 8;
#pragma unroll
                for (int b = 0; b < kColsPerWarp / 64; ++b) {
                    uint4 v[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        v[q] = b * 8 + q < nv ? ldg_nc_v4(h + b * 8 + q) : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const uint32_t u[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
                        uint32_t bits = 0;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            bits |= (bf(u[i >> 1], i & 1) > 0.0f ? 1u : 0u) << i;
                        hm[(b * 8 + q) >> 2] |= bits << (((b * 8 + q) & 3) * 8);
                    }
                }
            }
            if (!mbar_wait(tfull + acc, (it >> 1) & 1, abort_flag, err)) break;
            tc_fence_after();
            if (EPI == EPI_F32) {
                // fp32 weight gradient: the warp's 32 x 32 blocks go one at a time
                // through its kEpiBufs staging buffers (128-byte swizzle), each
                // written by one tensor store while the next block is staged;
                // rows past M_fix and columns past N are clipped by the map
                const bool rows_in = m0 + quad * 32 < M_fix;
#pragma unroll 1
                for (int cb = c_lo; cb < c_lo + kColsPerWarp; cb += 32) {
                    // one 32 x 32 block per step into staging buffer (step % kEpiBufs);
                    // the store that last used that buffer was committed kEpiBufs
                    // groups ago, so wait until at most kEpiBufs - 1 groups still read
                    const int u = ((cb - c_lo) >> 5) % kEpiBufs;
                    if (lane == 0) bulk_wait_read_allow<kEpiBufs - 1>();
                    __syncwarp();
                    uint32_t r[32];
                    tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(acc * BN + cb), r);
                    if (nk == 0) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = 0u;  // group without rows
                    }
                    uint8_t* buf = stage_c + u * 4096;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4*>(buf + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                            make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        const int col = n0 + cb;
                        if (rows_in && col < N) tma_store_3d(&tmap_c, buf, col, m0 + quad * 32, e);
                        bulk_commit();
                    }
                }
            } else {
#pragma unroll 1
                for (int cc = c_lo; cc < c_lo + kColsPerWarp; cc += 32) {
                    uint32_t r[32];
                    tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(acc * BN + cc), r);
                    const int col = n0 + cc;
                    const uint32_t mw = hm[0];
#pragma unroll
                    for (int w = 0; w + 1 < kColsPerWarp / 32; ++w) hm[w] = hm[w + 1];
                    if (!row_ok || col >= N) continue;
                    __nv_bfloat16* dst =
                        static_cast<__nv_bfloat16*>(Cv) + static_cast<size_t>(m0 + row) * N + col;
                    if (EPI == EPI_BF16_RELU_MASK) {
                        // dH = (dYp . W2) where the forward activation was positive
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (!((mw >> i) & 1u)) r[i] = 0u;
                    }
                    if (EPI == EPI_BF16_ADD) {
                        // C += product: the stored values plus the fp32 sum, rounded once
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if (q * 8 >= N - col) break;
                            const uint4 cv = *reinterpret_cast<const uint4*>(dst + q * 8);
                            const uint32_t cu[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                r[q * 8 + i] = __float_as_uint(__fadd_rn(
                                    __uint_as_float(r[q * 8 + i]), bf(cu[i >> 1], i & 1)));
                        }
                    }
                    Store32<__nv_bfloat16, false>::run(dst, r, N - col);
                }
            }
            tc_fence_before();
            mbar_arrive(tempty + acc);
        }
        if (EPI == EPI_F32 && lane == 0) bulk_wait_all();  // stores complete before exit
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
int launch_bwd(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc_map,
               const BwdArgs& args, long long ub, cudaStream_t st) {
    const int smem = fixed_bytes<EPI>() + 4 * (args.E + 1);
    if (ensure_smem<gemm_bwd_kernel<A_MN, KVAR, EPI>>(smem) != MOE_OK) return MOE_ERR_CUDA;
    const int grid = test_cap((int)(ub < num_sms() ? ub : num_sms()));
    if (grid <= 0) return MOE_OK;
    return launch_pdl(gemm_bwd_kernel<A_MN, KVAR, EPI>, grid, kBwdThreads, smem, st, ta, tb, tc_map,
                      args, device_error_word());
}

inline BwdArgs grouped(void* C, const void* Hmask, int M_fix, int N, int K_fix, int E,
                       const int32_t* offsets, int R_max) {
    BwdArgs a;
    a.C = C;
    a.Hmask = static_cast<const __nv_bfloat16*>(Hmask);
    a.M_fix = M_fix;
    a.N = N;
    a.K_fix = K_fix;
    a.E = E;
    a.offsets = offsets;
    a.single_M = 0;
    a.R_max = R_max;
    a.planes = 1;
    a.plane_rows = 0;
    a.slice_rows = 0;
    return a;
}

}  // namespace bwd
}  // namespace tc

#ifdef MOE_TEST_HOOKS
int test_stall_bwd(int v) { return tc::set_test_stall(v); }
#endif

// dH = (dYp . W2_e) * [H > 0] and dXp = dH . W1_e over the grouped rows, then
// dW2 = dYp_e^T H_e and dW1 = dH_e^T Xp_e per expert (fp32).
int launch_ffn_backward_bf16(const void* Xp, const void* H, const void* dYp, const void* W1,
                             const void* W2, int E, int d, int F, const int32_t* offsets,
                             int R_max, void* dH, void* dXp, float* dW1, float* dW2,
                             cudaStream_t st) {
    using namespace tc;
    using namespace tc::bwd;
    CUtensorMap a, b, c;
    std::memset(&c, 0, sizeof(c));  // unused by the bf16 epilogues
    const long long row_tiles = (long long)R_max / BM + E;
    int rc;
    // Each input gradient takes the forward pass's 2-CTA 256 x 256 tiles (weights
    // read N-major) where the forward pass would for its N, else 1-CTA tiles.
    // dH: A = dYp [R_max, d] K-major; B = W2 as [E*d rows (K), F (N)]
    if (kBwdPair && offsets != nullptr && gemm_pair_tiles(R_max, E, F)) {
        rc = launch_gemm_pair_nmajor_bf16(dYp, W2, dH, F, d, E, offsets, R_max, H, st);
    } else {
        if (make_tmap(&a, dYp, d, R_max, BM) != MOE_OK) return MOE_ERR_CUDA;
        if (make_tmap(&b, W2, F, E * d, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
        rc = launch_bwd<false, false, EPI_BF16_RELU_MASK>(
            a, b, c, grouped(dH, H, 0, F, d, E, offsets, R_max), row_tiles * ((F + BN - 1) / BN),
            st);
    }
    if (rc != MOE_OK) return rc;
    // dXp: A = dH [R_max, F] K-major; B = W1 as [E*F rows (K), d (N)]
    if (kBwdPair && offsets != nullptr && gemm_pair_tiles(R_max, E, d)) {
        rc = launch_gemm_pair_nmajor_bf16(dH, W1, dXp, d, F, E, offsets, R_max, nullptr, st);
    } else {
        if (make_tmap(&a, dH, F, R_max, BM) != MOE_OK) return MOE_ERR_CUDA;
        if (make_tmap(&b, W1, d, E * F, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
        rc = launch_bwd<false, false, EPI_BF16>(a, b, c, grouped(dXp, nullptr, 0, d, F, E,
                                                                 offsets, R_max),
                                               row_tiles * ((d + BN - 1) / BN), st);
    }
    if (rc != MOE_OK) return rc;
    if (dW2) {  // A = dYp rows as [K, M=d], B = H rows as [K, N=F]
        if (make_tmap(&a, dYp, d, R_max, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
        if (make_tmap(&b, H, F, R_max, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
        if (make_tmap_f32_3d(&c, dW2, F, d, E, 32) != MOE_OK) return MOE_ERR_CUDA;
        rc = launch_bwd<true, true, EPI_F32>(a, b, c, grouped(dW2, nullptr, d, F, 0, E, offsets,
                                                              R_max),
                                             (long long)E * ((d + BM - 1) / BM) *
                                                 ((F + BN - 1) / BN),
                                             st);
        if (rc != MOE_OK) return rc;
    }
    if (dW1) {  // A = dH rows as [K, M=F], B = Xp rows as [K, N=d]
        if (make_tmap(&a, dH, F, R_max, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
        if (make_tmap(&b, Xp, d, R_max, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
        if (make_tmap_f32_3d(&c, dW1, d, F, E, 32) != MOE_OK) return MOE_ERR_CUDA;
        rc = launch_bwd<true, true, EPI_F32>(a, b, c, grouped(dW1, nullptr, F, d, 0, E, offsets,
                                                              R_max),
                                             (long long)E * ((F + BM - 1) / BM) *
                                                 ((d + BN - 1) / BN),
                                             st);
        if (rc != MOE_OK) return rc;
    }
    return MOE_OK;
}

// ---------------------------------------------------------------------------
// Gate projection backward for bf16 layers on the tensor cores, without
// giving up the fp32 router gradient: dlogits (fp32) is split exactly into
// three bf16 planes, v = hi + mid + lo (each the bf16 rounding of what the
// previous ones leave; fp32 has 24 significant bits, three bf16 carry 8 each),
// and every product of a plane with the bf16 x or Wg is exact in the fp32
// accumulator.  The three planes run as one K loop (planes = 3):
//   dx  += [hi | mid | lo] . Wg     (rows of one group of T tokens, K = E)
//   dWg  = sum over token slices of [hi; mid; lo]^T . x    (fp32 partials of
//          consecutive token slices, added in slice order)
namespace {

__global__ void __launch_bounds__(256)
split3_kernel(const float* __restrict__ v, size_t n, __nv_bfloat16* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (size_t)gridDim.x * 256) {
        const float x = v[i];
        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
        const float r1 = __fsub_rn(x, __bfloat162float(hi));
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = __fsub_rn(r1, __bfloat162float(mid));
        out[i] = hi;
        out[n + i] = mid;
        out[2 * n + i] = __float2bfloat16_rn(r2);
    }
}

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace

bool gate_backward_tc_ok(int d, int E) { return d % 8 == 0 && E % 8 == 0; }

void gate_backward_tc_slices(int T, int d, int E, int* S, int* slice_rows) {
    using namespace tc;
    using namespace tc::bwd;
    const long long tiles = (long long)((E + BM - 1) / BM) * ((d + BN - 1) / BN);
    long long s = (296 + tiles - 1) / tiles;
    const long long cap = ((long long)T + 255) / 256;
    if (s > cap) s = cap;
    if (s < 1) s = 1;
    int sr = (int)(((T + s - 1) / s + 63) / 64 * 64);
    if (sr < 64) sr = 64;
    *slice_rows = sr;
    *S = (T + sr - 1) / sr;
}

size_t gate_backward_tc_workspace(int T, int d, int E) {
    int S, sr;
    gate_backward_tc_slices(T, d, E, &S, &sr);
    return align256((size_t)3 * T * E * 2) + (S > 1 ? (size_t)S * E * d * 4 : 0) + 256;
}

int launch_gate_backward_bf16(const void* x, const void* Wg, int T, int d, int E,
                              const float* dlogits, void* dx, float* dWg, void* ws,
                              cudaStream_t st) {
    using namespace tc;
    using namespace tc::bwd;
    char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(ws) + 255u) &
                                         ~uintptr_t(255u));
    __nv_bfloat16* planes = reinterpret_cast<__nv_bfloat16*>(base);
    float* part = reinterpret_cast<float*>(base + align256((size_t)3 * T * E * 2));
    const size_t n = (size_t)T * E;
    long long g = (long long)((n + 255) / 256);
    if (g > (long long)num_sms() * 8) g = (long long)num_sms() * 8;
    int rc = launch_pdl(split3_kernel, (int)g, 256, 0, st, dlogits, n, planes);
    if (rc != MOE_OK) return rc;
    CUtensorMap a, b, c;
    std::memset(&c, 0, sizeof(c));
    // dx += planes . Wg: A = [3T, E] K-major, B = Wg [E rows (K), d (N)]
    if (make_tmap(&a, planes, E, 3 * T, BM) != MOE_OK) return MOE_ERR_CUDA;
    if (make_tmap(&b, Wg, d, E, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
    BwdArgs args = grouped(dx, nullptr, 0, d, E, 1, nullptr, T);
    args.single_M = T;
    args.planes = 3;
    args.plane_rows = T;
    rc = launch_bwd<false, false, EPI_BF16_ADD>(
        a, b, c, args, (long long)((T + BM - 1) / BM) * ((d + BN - 1) / BN), st);
    if (rc != MOE_OK || !dWg) return rc;
    // dWg: A = planes as [3T rows (K), E (M)], B = x [T rows (K), d (N)]
    int S, sr;
    gate_backward_tc_slices(T, d, E, &S, &sr);
    float* out = S > 1 ? part : dWg;
    if (make_tmap(&a, planes, E, 3 * T, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
    if (make_tmap(&b, x, d, T, BK, MN_BOX) != MOE_OK) return MOE_ERR_CUDA;
    if (make_tmap_f32_3d(&c, out, d, E, S, 32) != MOE_OK) return MOE_ERR_CUDA;
    args = grouped(out, nullptr, E, d, 0, S, nullptr, T);
    args.single_M = T;
    args.planes = 3;
    args.plane_rows = T;
    args.slice_rows = sr;
    rc = launch_bwd<true, true, EPI_F32>(
        a, b, c, args, (long long)S * ((E + BM - 1) / BM) * ((d + BN - 1) / BN), st);
    if (rc != MOE_OK || S == 1) return rc;
    return launch_split_reduce(part, S, (size_t)E * d, dWg, st);
}

}  // namespace moe
