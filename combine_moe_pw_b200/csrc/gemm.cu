// gemm.cu - bf16 tensor-core GEMM on tcgen05 (sm_100a) for the latent
// projections, with a fused "project and pack" epilogue.
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 二: a latent projection
// compresses the routed activations from the 6144-wide model state to 3072
// before the expert-parallel exchange, and the outputs are projected back
// before they meet the shared experts.  Both are dense contractions, so they
// run on the tensor cores:
//   C[m][n] = bf16( sum_k A[m][k] * Bt[n][k] )      (fp32 accumulation)
// with A (activations) and Bt (weights, one row per output column) both
// K-major bf16.
//
// Two kernels share the epilogue.  The default pairs two SMs on one
// 256 x 256 tile (gemm_pair_kernel, below); the one-SM kernel here is used
// when a cluster of two cannot be launched, or when the environment sets
// MOE_PW_GEMM_PAIR=0.  Both give bit-identical results (same MMA steps in
// the same K order per output element).
//
// One-SM kernel shape: persistent, one CTA per SM, 6 warps.
//   warp 0      TMA producer: 128x64 A and 256x64 B tiles (128-byte
//               swizzle) into a 4-stage ring, one mbarrier per stage
//   warp 1      MMA issuer: allocates 512 TMEM columns (two 128x256 fp32
//               accumulators), issues tcgen05.mma M=128 N=256 K=16 from one
//               thread, commits each stage back to the producer and each
//               finished tile to the epilogue
//   warps 2..5  epilogue: tcgen05.ld the accumulator (warp w reads TMEM
//               lanes 32*(w%4)...), round to bf16 into a padded shared-memory
//               copy of its 32 rows, release the accumulator, then write each
//               row segment as one coalesced 512-byte warp store; the two
//               accumulators let the epilogue of tile i overlap the MMAs of
//               tile i+1
// Tiles are visited n-fastest so the 12 column tiles of one row block run
// together and the A rows are read from HBM about once (the weights stay in
// L2).  Every mbarrier wait is bounded; on a timeout the kernel records
// MOE_PW_DEVERR_TIMEOUT, every role stops, and TMEM is freed.
//
// Epilogue modes:
//   ROWS     C row-major [M, ldc]
//   SCATTER  project-and-pack: row m (token t) is written straight into the
//            pool slot of every (t, j) the sender kept (slot_map), one
//            coalesced 512-byte store per slot and column tile, and the tile
//            at column 0 writes the slot header; the latent rows are never
//            materialised.
#include <atomic>
#include <cstdlib>

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cuda_bf16.h>

#include "common.cuh"
#include "umma.cuh"

namespace moe_pw {

namespace {

#ifndef MOE_PW_GEMM_STAGES
#define MOE_PW_GEMM_STAGES 4
#endif
constexpr int BM = 128, BN = 256, BK = 64, STAGES = MOE_PW_GEMM_STAGES;
constexpr uint32_t A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr uint32_t GEMM_WAIT_LIMIT = 1u << 24;
// epilogue staging: per epilogue warp 32 rows x half a tile (128 bf16 =
// 256 bytes); the 16-byte chunk c of row r is stored at chunk c ^ (r & 7), so
// both the per-row writes and the per-chunk reads spread over the banks
constexpr int HALF = BN / 2;
constexpr int SLOTS_IN_REGS = 8;  // choices per token whose slots the epilogue keeps in registers
constexpr uint32_t ROW_PITCH = HALF * 2;
constexpr uint32_t STAGING_BYTES = 4 * 32 * ROW_PITCH;
constexpr size_t SMEM_BYTES =
    size_t(STAGES) * STAGE_BYTES + STAGING_BYTES + 1024 /*align*/ + 256 /*barriers*/;

enum Mode { ROWS = 0, SCATTER = 1 };

struct GemmArgs {
    int32_t M, N, K;
    int32_t mode;
    // ROWS
    uint16_t *C;
    int64_t ldc;
    const uint16_t *add;  // ROWS, optional: bf16 [M, ldc] added in fp32 before rounding
                          // (may be C itself: each element is read before it is written)
    // SCATTER
    const int32_t *slot_map;
    const int32_t *idx;
    int32_t topk;
    uint16_t *pool_x;
    int32_t *pool_hdr;
    int64_t n_slots;
    moe_pw_counters *ctr;
};

struct Shared {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int32_t abort;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, Shared *sh,
                                              moe_pw_counters *ctr)
{
    for (uint32_t i = 0; i < GEMM_WAIT_LIMIT; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 1023) == 1023 && *(volatile int32_t *)&sh->abort) return false;
    }
    atomicExch(&sh->abort, 1);
    set_error(ctr, MOE_PW_DEVERR_TIMEOUT);
    return false;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&r);
}

// SCATTER: the slots of this thread's own row (row my_m), fetched before the
// accumulator is read so the store loop needs no global loads; the tile at
// column 0 writes the slot headers.
__device__ __forceinline__ void fetch_row_slots(const GemmArgs &p, int64_t my_m, int n_blk,
                                                int32_t (&row_slot)[SLOTS_IN_REGS])
{
#pragma unroll
    for (int j = 0; j < SLOTS_IN_REGS; ++j) row_slot[j] = -1;
    if (p.mode == SCATTER && my_m < p.M && p.topk <= SLOTS_IN_REGS) {
#pragma unroll
        for (int j = 0; j < SLOTS_IN_REGS; ++j) {
            if (j >= p.topk) break;
            int32_t sl = p.slot_map[my_m * p.topk + j];
            if (sl >= p.n_slots) {
                set_error(p.ctr, MOE_PW_DEVERR_SLOT);
                sl = -1;
            }
            row_slot[j] = sl;
            if (sl >= 0 && n_blk == 0) p.pool_hdr[sl] = p.idx[my_m * p.topk + j];
        }
    }
}

// Epilogue of one accumulator: 128 rows (m0 + 0..127) x BN columns (column
// tile n_blk) held in TMEM columns acc*BN.., read by the four epilogue warps
// (warp quarter q reads TMEM lanes 32q..32q+31, one row per thread).
// row_slot: SCATTER mode's slots of this thread's row.  release() runs in
// every thread once the accumulator has been read into shared memory.
template <class Release>
__device__ __forceinline__ void epilogue_tile(const GemmArgs &p, uint8_t *stage_rows,
                                              uint32_t tmem_base, int acc, int q, int lane,
                                              int64_t m0, int n_blk,
                                              const int32_t (&row_slot)[SLOTS_IN_REGS],
                                              Release release)
{
    const int n0 = n_blk * BN;
    const int hw = lane >> 4, l16 = lane & 15;
    for (int h = 0; h < 2; ++h) {
        // 1. TMEM -> bf16 -> this thread's row (half h) in shared memory
        uint8_t *my_row = stage_rows + size_t(lane) * ROW_PITCH;
        const int64_t my_m = m0 + q * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < HALF / 32; ++c) {
            // merge operand of this thread's row, 32 columns (loaded before
            // the accumulator so the two latencies overlap)
            uint32_t ad[16];
            if (p.add) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int col = n0 + h * HALF + c * 32 + 8 * i;
                    uint4 a4 = make_uint4(0, 0, 0, 0);
                    if (my_m < p.M && col + 8 <= p.N)
                        a4 = __ldcs(reinterpret_cast<const uint4 *>(p.add + my_m * p.ldc + col));
                    ad[4 * i + 0] = a4.x;
                    ad[4 * i + 1] = a4.y;
                    ad[4 * i + 2] = a4.z;
                    ad[4 * i + 3] = a4.w;
                }
            }
            uint32_t v[32];
            umma::tmem_ld32(tmem_base + (uint32_t(q * 32) << 16) +
                                uint32_t(acc * BN + h * HALF + c * 32),
                            v);
            float f[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
            if (p.add) {
                // the merge: fp32 sum, one rounding to bf16 below
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    f[2 * i] = __fadd_rn(f[2 * i], __uint_as_float(ad[i] << 16));
                    f[2 * i + 1] = __fadd_rn(f[2 * i + 1], __uint_as_float(ad[i] & 0xFFFF0000u));
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint4 o;
                o.x = pack_bf16(f[8 * i + 0], f[8 * i + 1]);
                o.y = pack_bf16(f[8 * i + 2], f[8 * i + 3]);
                o.z = pack_bf16(f[8 * i + 4], f[8 * i + 5]);
                o.w = pack_bf16(f[8 * i + 6], f[8 * i + 7]);
                const int chunk = (c * 4 + i) ^ (lane & 7);
                reinterpret_cast<uint4 *>(my_row)[chunk] = o;
            }
        }
        if (h == 1) release();  // 2. the accumulator is free for the next tile's MMAs
        __syncwarp();
        // 3. each half-warp writes one 256-byte row segment per store:
        //    rows r + hw, chunk l16 (ROWS), or that segment into every
        //    kept slot of the row (SCATTER)
        const int ncol = n0 + h * HALF + 8 * l16;
        const bool col_ok = ncol + 8 <= p.N;
        for (int r = 0; r < 32; r += 2) {
            const int row = r + hw;
            const int64_t m = m0 + q * 32 + row;
            const bool row_ok = m < p.M;
            const uint4 val = reinterpret_cast<const uint4 *>(
                stage_rows + size_t(row) * ROW_PITCH)[l16 ^ (row & 7)];
            if (p.mode == ROWS) {
                if (row_ok && col_ok) __stcs(reinterpret_cast<uint4 *>(p.C + m * p.ldc + ncol), val);
                continue;
            }
            if (p.topk <= SLOTS_IN_REGS) {
#pragma unroll
                for (int j = 0; j < SLOTS_IN_REGS; ++j) {
                    const int32_t slot = __shfl_sync(FULL_MASK, row_slot[j], row);
                    if (j < p.topk && slot >= 0 && col_ok)
                        __stcs(reinterpret_cast<uint4 *>(p.pool_x + int64_t(slot) * p.N + ncol), val);
                }
                continue;
            }
            // more choices than registers hold: read the slots here
            for (int jb = 0; jb < p.topk; jb += 16) {
                int32_t my_slot = -1;
                if (row_ok && jb + l16 < p.topk) {
                    my_slot = p.slot_map[m * p.topk + jb + l16];
                    if (my_slot >= p.n_slots) {
                        set_error(p.ctr, MOE_PW_DEVERR_SLOT);
                        my_slot = -1;
                    }
                    if (my_slot >= 0 && n_blk == 0 && h == 0)
                        p.pool_hdr[my_slot] = p.idx[m * p.topk + jb + l16];
                }
                const int jn = p.topk - jb < 16 ? p.topk - jb : 16;
                for (int j = 0; j < jn; ++j) {
                    const int32_t slot = __shfl_sync(FULL_MASK, my_slot, (lane & 16) | j);
                    if (slot >= 0 && col_ok)
                        __stcs(reinterpret_cast<uint4 *>(p.pool_x + int64_t(slot) * p.N + ncol), val);
                }
            }
        }
        __syncwarp();
    }
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                GemmArgs p)
{
    extern __shared__ uint8_t smem_raw[];
    // stage buffers need 1024-byte alignment for the 128-byte swizzle atoms
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *staging = smem + size_t(STAGES) * STAGE_BYTES;
    Shared *sh = reinterpret_cast<Shared *>(staging + STAGING_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int m_tiles = (p.M + BM - 1) / BM, n_tiles = (p.N + BN - 1) / BN;
    const int num_tiles = m_tiles * n_tiles;
    const int k_iters = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sh->full[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sh->tfull[a], 1);
            mbar_init(&sh->tempty[a], 4 * 32);
        }
        sh->abort = 0;
        fence_init_and_proxy();
    }
    if (warp == 1) {
        umma::tmem_alloc(&sh->tmem_base, TMEM_COLS);
        umma::tmem_relinquish();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem_base = sh->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            // the weights are re-read by every row block: keep them in L2
            const uint64_t pol_b = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
                const int m_blk = tile / n_tiles, n_blk = tile - m_blk * n_tiles;
                for (int kk = 0; kk < k_iters; ++kk) {
                    if (!wait_or_abort(&sh->empty[stage], phase ^ 1u, sh, p.ctr)) goto done;
                    uint8_t *a_dst = smem + size_t(stage) * STAGE_BYTES;
                    mbar_arrive_expect_tx(&sh->full[stage], STAGE_BYTES);
                    umma::tma_load_2d(a_dst, &tmA, kk * BK, m_blk * BM, &sh->full[stage]);
                    umma::tma_load_2d_hint(a_dst + A_BYTES, &tmB, kk * BK, n_blk * BN,
                                           &sh->full[stage], pol_b);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = umma::idesc_f16(BM, BN, true);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
                if (!wait_or_abort(&sh->tempty[acc], acc_phase ^ 1u, sh, p.ctr)) goto done;
                umma::fence_after_sync();
                const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
                for (int kk = 0; kk < k_iters; ++kk) {
                    if (!wait_or_abort(&sh->full[stage], phase, sh, p.ctr)) goto done;
                    umma::fence_after_sync();
                    const uint32_t a_addr = smem_addr(smem + size_t(stage) * STAGE_BYTES);
                    const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
                    for (int k16 = 0; k16 < BK / 16; ++k16) {
                        // K advances 16 elements = 32 bytes inside the 128-byte swizzle row
                        const uint64_t ad = umma::smem_desc(a_addr + 32u * k16, 16u, 1024u,
                                                            umma::LAYOUT_SWIZZLE_128B);
                        const uint64_t bd = umma::smem_desc(b_addr + 32u * k16, 16u, 1024u,
                                                            umma::LAYOUT_SWIZZLE_128B);
                        umma::mma_bf16(d_tmem, ad, bd, idesc, (kk | k16) != 0);
                    }
                    umma::commit(&sh->empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                umma::commit(&sh->tfull[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
    } else {
        // epilogue: TMEM lane quarter of this warp; each thread owns one row
        const int q = warp & 3;
        uint8_t *stage_rows = staging + size_t(warp - 2) * 32 * ROW_PITCH;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int m_blk = tile / n_tiles, n_blk = tile - m_blk * n_tiles;
            int32_t row_slot[SLOTS_IN_REGS];
            fetch_row_slots(p, int64_t(m_blk) * BM + q * 32 + lane, n_blk, row_slot);
            const bool ok = wait_or_abort(&sh->tfull[acc], acc_phase, sh, p.ctr);
            if (!__all_sync(FULL_MASK, ok)) break;
            umma::fence_after_sync();
            epilogue_tile(p, stage_rows, tmem_base, acc, q, lane, int64_t(m_blk) * BM, n_blk,
                          row_slot, [&] {
                              umma::fence_before_sync();
                              mbar_arrive(&sh->tempty[acc]);
                          });
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }
done:
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 1) umma::tmem_dealloc(tmem_base, TMEM_COLS);
}


// --------------------------------------------------------------------------
// Two-SM kernel: a cluster of 2 CTAs computes one 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256: 128 rows of A from each CTA; N = 256:
// the 128-row halves of the B tile come from the two CTAs).  Per SM, each
// MMA step then moves 8 KB of operands through shared memory instead of
// 12 KB, and each CTA loads half the weights' tile; a 5-stage ring of
// 32 KB stages.  Measured on B200 with clocks free (16K-64K rows): 3-5%
// more TFLOP/s than the one-SM kernel; at 262,144 rows both run at the
// power cap and match.
//   warp 0 (both CTAs)   TMA producer for this CTA's halves; completion is
//                        counted on the even CTA's stage barrier
//   warp 1 (even CTA)    MMA issuer for the pair
//   warps 2..5 (both)    epilogue of this CTA's 128 rows, as above
// Each MMA completion is committed to the same barrier in both CTAs at once
// (tcgen05.commit to the pair's CTA mask): the odd CTA's producer and
// epilogue learn of it as early as the even CTA's.  (Forwarding it from the
// even CTA with a remote mbarrier arrive instead measured 40% slower.)
// Every TMA load writes only the issuing CTA's own shared memory.  Every
// wait is bounded as above, and a timeout in one CTA also raises the abort
// flag of the other.
// --------------------------------------------------------------------------
#ifndef MOE_PW_GEMM_PAIR_STAGES
#define MOE_PW_GEMM_PAIR_STAGES 5
#endif
constexpr int STAGES2 = MOE_PW_GEMM_PAIR_STAGES;
constexpr int BM2 = 2 * BM;  // rows per pair tile
constexpr uint32_t B2_BYTES = (BN / 2) * BK * 2, STAGE2_BYTES = A_BYTES + B2_BYTES;
constexpr size_t SMEM2_BYTES =
    size_t(STAGES2) * STAGE2_BYTES + STAGING_BYTES + 1024 /*align*/ + 256 /*barriers*/;

struct Shared2 {
    uint64_t full[STAGES2];   // even CTA: both CTAs' loads of a stage landed
    uint64_t empty[STAGES2];  // stage free again (MMA commit, in both CTAs)
    uint64_t tfull[2];        // accumulator ready (MMA commit, in both CTAs)
    uint64_t tempty[2];       // even CTA: the 8 epilogue warps of the pair read it
    uint32_t tmem_base;
    int32_t abort;
};

__device__ __forceinline__ bool wait_or_abort2(uint64_t *bar, uint32_t parity, Shared2 *sh,
                                               uint32_t peer_abort, moe_pw_counters *ctr)
{
    for (uint32_t i = 0; i < GEMM_WAIT_LIMIT; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 1023) == 1023 && *(volatile int32_t *)&sh->abort) return false;
    }
    atomicExch(&sh->abort, 1);
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort), "r"(1) : "memory");
    set_error(ctr, MOE_PW_DEVERR_TIMEOUT);
    return false;
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, GemmArgs p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *staging = smem + size_t(STAGES2) * STAGE2_BYTES;
    Shared2 *sh = reinterpret_cast<Shared2 *>(staging + STAGING_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = umma::cluster_ctarank();
    const uint32_t cid = umma::cluster_id_x(), ncl = umma::cluster_count_x();
    const uint32_t peer = rank ^ 1u;
    const uint32_t peer_abort = umma::mapa_shared(smem_addr(&sh->abort), peer);

    const int m_tiles = (p.M + BM2 - 1) / BM2, n_tiles = (p.N + BN - 1) / BN;
    const int num_tiles = m_tiles * n_tiles;
    const int k_iters = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES2; ++s) {
            mbar_init(&sh->full[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sh->tfull[a], 1);
            mbar_init(&sh->tempty[a], 2 * 4);
        }
        sh->abort = 0;
        fence_init_and_proxy();
    }
    if (warp == 1) {
        umma::tmem_alloc_pair(&sh->tmem_base, TMEM_COLS);
        umma::tmem_relinquish_pair();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::cluster_sync();  // both CTAs' barriers exist before any remote arrive
    umma::fence_after_sync();
    const uint32_t tmem_base = sh->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_normal();
            const uint64_t pol_b = policy_evict_last();  // weights: re-read by every row block
            const uint32_t full0 = umma::mapa_shared(smem_addr(&sh->full[0]), 0);
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = int(cid); tile < num_tiles; tile += int(ncl)) {
                const int m_blk = tile / n_tiles, n_blk = tile - m_blk * n_tiles;
                const int a_row = m_blk * BM2 + int(rank) * BM;
                const int b_row = n_blk * BN + int(rank) * (BN / 2);
                for (int kk = 0; kk < k_iters; ++kk) {
                    if (!wait_or_abort2(&sh->empty[stage], phase ^ 1u, sh, peer_abort, p.ctr))
                        goto done;
                    if (rank == 0) mbar_arrive_expect_tx(&sh->full[stage], 2 * STAGE2_BYTES);
                    uint8_t *a_dst = smem + size_t(stage) * STAGE2_BYTES;
                    const uint32_t bar = full0 + 8u * uint32_t(stage);
                    umma::tma_load_2d_pair(a_dst, &tmA, kk * BK, a_row, bar, pol_a);
                    umma::tma_load_2d_pair(a_dst + A_BYTES, &tmB, kk * BK, b_row, bar, pol_b);
                    if (++stage == STAGES2) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (rank == 0 && lane == 0) {
            const uint32_t idesc = umma::idesc_f16(BM2, BN, true);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int tile = int(cid); tile < num_tiles; tile += int(ncl)) {
                if (!wait_or_abort2(&sh->tempty[acc], acc_phase ^ 1u, sh, peer_abort, p.ctr))
                    goto done;
                umma::fence_after_sync();
                const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
                for (int kk = 0; kk < k_iters; ++kk) {
                    if (!wait_or_abort2(&sh->full[stage], phase, sh, peer_abort, p.ctr)) goto done;
                    umma::fence_after_sync();
                    const uint32_t a_addr = smem_addr(smem + size_t(stage) * STAGE2_BYTES);
                    const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
                    for (int k16 = 0; k16 < BK / 16; ++k16) {
                        const uint64_t ad = umma::smem_desc(a_addr + 32u * k16, 16u, 1024u,
                                                            umma::LAYOUT_SWIZZLE_128B);
                        const uint64_t bd = umma::smem_desc(b_addr + 32u * k16, 16u, 1024u,
                                                            umma::LAYOUT_SWIZZLE_128B);
                        umma::mma_bf16_pair(d_tmem, ad, bd, idesc, (kk | k16) != 0);
                    }
                    umma::commit_pair_both(&sh->empty[stage]);
                    if (++stage == STAGES2) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                umma::commit_pair_both(&sh->tfull[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
    } else {
        const int q = warp & 3;
        uint8_t *stage_rows = staging + size_t(warp - 2) * 32 * ROW_PITCH;
        const uint32_t tempty0 = umma::mapa_shared(smem_addr(&sh->tempty[0]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = int(cid); tile < num_tiles; tile += int(ncl)) {
            const int m_blk = tile / n_tiles, n_blk = tile - m_blk * n_tiles;
            const int64_t m0 = int64_t(m_blk) * BM2 + int64_t(rank) * BM;
            int32_t row_slot[SLOTS_IN_REGS];
            fetch_row_slots(p, m0 + q * 32 + lane, n_blk, row_slot);
            const bool ok = wait_or_abort2(&sh->tfull[acc], acc_phase, sh, peer_abort, p.ctr);
            if (!__all_sync(FULL_MASK, ok)) break;
            umma::fence_after_sync();
            epilogue_tile(p, stage_rows, tmem_base, acc, q, lane, m0, n_blk, row_slot, [&] {
                umma::fence_before_sync();
                __syncwarp();
                if (lane == 0) umma::mbar_arrive_cluster(tempty0 + 8u * uint32_t(acc));
            });
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }
done:
    umma::fence_before_sync();
    __syncthreads();
    umma::cluster_sync();  // no MMA, TMEM read or remote arrive of the pair is left
    umma::fence_after_sync();
    if (warp == 1) umma::tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

// --------------------------------------------------------------------------
// host side
// --------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// Row-major bf16 [rows, cols] tensor, box [box_rows, 64 cols], 128-byte swizzle.
bool make_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {uint32_t(BK), box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

#ifndef MOE_PW_GEMM_PAIR
#define MOE_PW_GEMM_PAIR 1
#endif

// The two-SM kernel unless the environment sets MOE_PW_GEMM_PAIR=0 (read once).
bool pair_kernel_enabled()
{
    static const bool on = [] {
        const char *e = std::getenv("MOE_PW_GEMM_PAIR");
        return MOE_PW_GEMM_PAIR && !(e && e[0] == '0' && e[1] == 0);
    }();
    return on;
}

// Clusters of two CTAs of the pair kernel that fit on the current device at
// once (0: the pair kernel cannot be launched here).  Cached per device.
int pair_clusters_resident()
{
    static std::atomic<int> cached[64];  // value + 1; 0 = not yet known
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    const int c = cached[dev].load();
    if (c) return c - 1;
    int n = 0;
    if (cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(SMEM2_BYTES)) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = 2;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(THREADS);
        cfg.dynamicSmemBytes = SMEM2_BYTES;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();  // a refusal above only means: use the one-SM kernel
    cached[dev].store(n + 1);
    return n;
}

}  // namespace

cudaError_t launch_gemm(const uint16_t *A, const uint16_t *Bt, int64_t M, int32_t N, int32_t K,
                        int32_t mode, uint16_t *C, int64_t ldc, const int32_t *slot_map,
                        const int32_t *idx, int32_t topk, uint16_t *pool_x, int32_t *pool_hdr,
                        int64_t n_slots, moe_pw_counters *ctr, cudaStream_t st,
                        const uint16_t *add)
{
    if (M == 0 || N == 0) return cudaSuccess;
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    const int clusters = pair_kernel_enabled() ? pair_clusters_resident() : 0;
    alignas(64) CUtensorMap ta, tb;
    if (!make_map(&ta, A, uint64_t(M), uint64_t(K), BM) ||
        !make_map(&tb, Bt, uint64_t(N), uint64_t(K), clusters > 0 ? BN / 2 : BN))
        return cudaErrorInvalidValue;
    GemmArgs p;
    p.M = int32_t(M);
    p.N = N;
    p.K = K;
    p.mode = mode;
    p.C = C;
    p.ldc = ldc;
    p.add = add;
    p.slot_map = slot_map;
    p.idx = idx;
    p.topk = topk;
    p.pool_x = pool_x;
    p.pool_hdr = pool_hdr;
    p.n_slots = n_slots;
    p.ctr = ctr;
    if (clusters > 0) {
        // pairs of SMs on 256 x 256 tiles, one cluster per resident pair
        cudaError_t err = cudaFuncSetAttribute(
            gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM2_BYTES));
        if (err != cudaSuccess) return err;
        const int64_t tiles = ((M + BM2 - 1) / BM2) * ((N + BN - 1) / BN);
        const int n_cl = int(tiles < clusters ? tiles : clusters);
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = 2;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(unsigned(2 * n_cl));
        cfg.blockDim = dim3(THREADS);
        cfg.dynamicSmemBytes = SMEM2_BYTES;
        cfg.stream = st;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        err = cudaLaunchKernelEx(&cfg, gemm_pair_kernel, ta, tb, p);
        if (err != cudaSuccess) return err;
        return cudaGetLastError();
    }
    cudaError_t err = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(SMEM_BYTES));
    if (err != cudaSuccess) return err;
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int grid = int(tiles < di.sms ? tiles : di.sms);
    gemm_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(ta, tb, p);
    return cudaGetLastError();
}

}  // namespace moe_pw
