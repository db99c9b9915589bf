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
// Kernel shape: persistent, one CTA per SM, 6 warps.
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
            // SCATTER: the slots of this thread's own row, fetched before the
            // accumulator is read so the store loop needs no global loads
            int32_t row_slot[SLOTS_IN_REGS];
            {
                const int64_t my_m = int64_t(m_blk) * BM + q * 32 + lane;
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
            const bool ok = wait_or_abort(&sh->tfull[acc], acc_phase, sh, p.ctr);
            if (!__all_sync(FULL_MASK, ok)) break;
            umma::fence_after_sync();
            const int n0 = n_blk * BN;
            const int hw = lane >> 4, l16 = lane & 15;
            for (int h = 0; h < 2; ++h) {
                // 1. TMEM -> bf16 -> this thread's row (half h) in shared memory
                uint8_t *my_row = stage_rows + size_t(lane) * ROW_PITCH;
#pragma unroll 1
                for (int c = 0; c < HALF / 32; ++c) {
                    uint32_t v[32];
                    umma::tmem_ld32(tmem_base + (uint32_t(q * 32) << 16) +
                                        uint32_t(acc * BN + h * HALF + c * 32),
                                    v);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint4 o;
                        o.x = pack_bf16(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
                        o.y = pack_bf16(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
                        o.z = pack_bf16(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
                        o.w = pack_bf16(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
                        const int chunk = (c * 4 + i) ^ (lane & 7);
                        reinterpret_cast<uint4 *>(my_row)[chunk] = o;
                    }
                }
                if (h == 1) {
                    // 2. the accumulator is free for the next tile's MMAs
                    umma::fence_before_sync();
                    mbar_arrive(&sh->tempty[acc]);
                }
                __syncwarp();
                // 3. each half-warp writes one 256-byte row segment per store:
                //    rows r + hw, chunk l16 (ROWS), or that segment into every
                //    kept slot of the row (SCATTER)
                const int ncol = n0 + h * HALF + 8 * l16;
                const bool col_ok = ncol + 8 <= p.N;
                for (int r = 0; r < 32; r += 2) {
                    const int row = r + hw;
                    const int64_t m = int64_t(m_blk) * BM + q * 32 + row;
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

}  // namespace

cudaError_t launch_gemm(const uint16_t *A, const uint16_t *Bt, int64_t M, int32_t N, int32_t K,
                        int32_t mode, uint16_t *C, int64_t ldc, const int32_t *slot_map,
                        const int32_t *idx, int32_t topk, uint16_t *pool_x, int32_t *pool_hdr,
                        int64_t n_slots, moe_pw_counters *ctr, cudaStream_t st)
{
    if (M == 0 || N == 0) return cudaSuccess;
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    alignas(64) CUtensorMap ta, tb;
    if (!make_map(&ta, A, uint64_t(M), uint64_t(K), BM) ||
        !make_map(&tb, Bt, uint64_t(N), uint64_t(K), BN))
        return cudaErrorInvalidValue;
    GemmArgs p;
    p.M = int32_t(M);
    p.N = N;
    p.K = K;
    p.mode = mode;
    p.C = C;
    p.ldc = ldc;
    p.slot_map = slot_map;
    p.idx = idx;
    p.topk = topk;
    p.pool_x = pool_x;
    p.pool_hdr = pool_hdr;
    p.n_slots = n_slots;
    p.ctr = ctr;
    cudaError_t err = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(SMEM_BYTES));
    if (err != cudaSuccess) return err;
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int grid = int(tiles < di.sms ? tiles : di.sms);
    gemm_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(ta, tb, p);
    return cudaGetLastError();
}

}  // namespace moe_pw
