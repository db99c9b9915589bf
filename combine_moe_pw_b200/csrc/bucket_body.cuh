// bucket_body.cuh - receiver bucketing of one (destination, wave) item,
// shared by the bucketing kernel (bucket.cu) and the fused pack + bucketing
// kernel (pack.cu).  Internal; not part of the public ABI.
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 二: the 1.15 receiver factor
// caps the rows a local expert accepts; overflow is dropped and counted apart
// from sender drops.
//
// Item (d, w): its positions q = s * C_s + c run over the R pools (s, d, w) in
// arrival order (sources ascending, then slots ascending); slots c >= occ are
// empty.  The row of an arrival with local expert pp is the number of earlier
// positions with the same expert, i.e. an exclusive prefix count over q, so
// the NT threads taking part work in tiles of NT * BK_ITEMS positions:
//   1. local experts of the tile into shared memory, position j of the tile
//      by thread j % NT (every header and occupancy read of a thread issued
//      together; empty and dropped positions get recv_row -1 here);
//   2. per local expert: thread t counts its contiguous run of BK_ITEMS
//      positions, an exclusive scan over the NT threads gives the run's first
//      row, and the thread numbers its arrivals in order into shared memory;
//   3. recv_row and bucket_slot are written in position order (coalesced),
//      and the per-expert carry moves to the next tile.
#pragma once

#include "common.cuh"

namespace moe_pw {

constexpr int BK_ITEMS = 32;
static_assert(BK_ITEMS == 32, "a thread's run is one 32-bit mask per local expert");

struct BucketArgs {
    const int32_t *pool_hdr;
    const int32_t *occ;
    int32_t *recv_row;
    int32_t *bucket_slot;
    int32_t *expert_counts;
    moe_pw_counters *ctr;
    Geo g;
    uint32_t wave_mask;  // waves whose items run
    // fused with the pack: the assignment pass wrote the kept slots' headers
    // and the bucketing writes -1 into the empty ones (the pack writes none)
    int32_t *hdr_out;
};

// Barrier among the NT threads that take part: the whole block (BAR 0, NT =
// blockDim.x) or a named barrier of a sub-group of whole warps.
template <int NT, int BAR>
__device__ __forceinline__ void bk_sync()
{
    if (BAR == 0)
        __syncthreads();
    else
        asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
}

// Exclusive scan of v over the NT threads (tid = 0 .. NT-1; all call it);
// *total gets the sum.
template <int NT, int BAR>
__device__ __forceinline__ int32_t bk_exclusive_scan(int32_t v, int tid, int32_t *wsum,
                                                     int32_t *total)
{
    constexpr int NW = NT / 32;
    const int warp = tid >> 5, lane = tid & 31;
    int32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(FULL_MASK, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) wsum[warp] = inc;
    bk_sync<NT, BAR>();
    if (warp == 0) {
        const int32_t x = lane < NW ? wsum[lane] : 0;
        int32_t xi = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(FULL_MASK, xi, o);
            if (lane >= o) xi += u;
        }
        if (lane < NW) wsum[lane] = xi - x;
        if (lane == NW - 1) wsum[NW] = xi;
    }
    bk_sync<NT, BAR>();
    const int32_t r = wsum[warp] + inc - v;
    *total = wsum[NW];
    bk_sync<NT, BAR>();  // wsum is reused by the next scan
    return r;
}

// Shared memory of one item worker: local experts [TILE] int8, rows
// [TILE + TILE/32] int32 (padded), carry [P], scan partials [NT/32 + 1].
inline size_t bucket_smem_bytes(int NT, int P)
{
    const size_t tile = size_t(NT) * BK_ITEMS;
    return tile + sizeof(int32_t) * (tile + tile / 32 + size_t(P) + NT / 32 + 1);
}

// Bucket item dw = d * W + w (d: this GPU's d-th destination rank, all of
// them on one GPU).  sm: bucket_smem_bytes(NT, P) bytes, 16-byte aligned.
template <int NT, int BAR, bool FUSED>
__device__ __forceinline__ void bucket_item(const BucketArgs &p, int dw, int tid, int32_t *sm)
{
    constexpr int TILE = NT * BK_ITEMS;
    const int P = p.g.P, R = p.g.R;
    int8_t *pe_sm = reinterpret_cast<int8_t *>(sm);  // [TILE]
    int32_t *row_sm = sm + TILE / 4;                 // [TILE + TILE / 32], padded
    int32_t *carry = row_sm + TILE + TILE / 32;      // [P]
    int32_t *wsum = carry + P;                       // [NT / 32 + 1]
    // the item's pools (s, d, w) for the R sources s sit at pool_s0 + s * pool_step
    const int d = dw / p.g.W, w = dw - d * p.g.W;
    const int32_t e_base = p.g.ep_g * p.g.Rn * p.g.L;  // first expert on this GPU
    const int32_t E_out = p.g.Rn * p.g.L;              // experts of this GPU
    const int32_t e0 = (p.g.ep_g * p.g.Rn + d) * p.g.L + w * p.g.P;
    const int64_t C_s = p.g.C_s, C_r = p.g.C_r;
    const int64_t npos = int64_t(R) * C_s;
    const int64_t pool_s0 = int64_t(d) * p.g.W + w;
    const int64_t pool_step = int64_t(p.g.Rn) * p.g.W;
    for (int i = tid; i < P; i += NT) carry[i] = 0;

    for (int64_t t0 = 0; t0 < npos; t0 += TILE) {
        // 1. local experts of the tile (positions fit in 32 bits: npos <= n_slots)
        constexpr int U = 4;
        const uint32_t Cs32 = uint32_t(C_s);
        for (int j0 = 0; j0 < TILE; j0 += U * NT) {
            int32_t hdr[U], occ[U];
            uint32_t cc[U], slot[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t q = t0 + j0 + u * NT + tid;
                hdr[u] = -1;
                occ[u] = 0;
                cc[u] = 0;
                slot[u] = 0;
                if (q < npos) {
                    const uint32_t sq = uint32_t(q) / Cs32;
                    cc[u] = uint32_t(q) - sq * Cs32;
                    const int64_t pool = pool_s0 + int64_t(sq) * pool_step;
                    slot[u] = uint32_t(pool * C_s + cc[u]);
                    occ[u] = p.occ ? p.occ[pool] : 0;
                    hdr[u] = p.pool_hdr[slot[u]];
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = j0 + u * NT + tid;
                int pe = -1;
                if (t0 + j < npos) {
                    // filled: below the pool's occupancy, or (no counts
                    // exchanged) a header other than -1
                    if (p.occ ? int32_t(cc[u]) < occ[u] : hdr[u] != -1) {
                        pe = hdr[u] - e0;
                        if (pe < 0 || pe >= P) {
                            set_error(p.ctr, MOE_PW_DEVERR_HEADER);
                            pe = -1;
                        }
                    } else if (FUSED) {
                        p.hdr_out[slot[u]] = -1;  // empty slot
                    }
                    if (pe < 0) p.recv_row[slot[u]] = -1;
                }
                pe_sm[j] = int8_t(pe);
            }
        }
        bk_sync<NT, BAR>();

        // 2. rows, one local expert at a time; the thread's run of local
        //    experts is read once, 16 bytes at a time
        const int jr = tid * BK_ITEMS;  // this thread's run [jr, jr + BK_ITEMS)
        uint32_t run[BK_ITEMS / 4];
#pragma unroll
        for (int v = 0; v < BK_ITEMS / 16; ++v) {
            const uint4 x = reinterpret_cast<const uint4 *>(pe_sm + jr)[v];
            run[4 * v + 0] = x.x;
            run[4 * v + 1] = x.y;
            run[4 * v + 2] = x.z;
            run[4 * v + 3] = x.w;
        }
        for (int pp = 0; pp < P; ++pp) {
            // bit i: run position i holds local expert pp.  Four positions per
            // word: a bytewise compare, then the four byte flags gathered into
            // bits 28..31 by one multiply (the other partial products stay
            // below bit 24, so nothing carries into them)
            uint32_t mine = 0;
            const uint32_t key = uint32_t(pp) * 0x01010101u;
#pragma unroll
            for (int wi = 0; wi < BK_ITEMS / 4; ++wi) {
                const uint32_t eq = __vcmpeq4(run[wi], key) & 0x01010101u;
                mine |= ((eq * 0x10204080u) >> 28) << (4 * wi);
            }
            int32_t total;
            const int32_t first = bk_exclusive_scan<NT, BAR>(__popc(mine), tid, wsum, &total);
            int32_t r = carry[pp] + first;
            while (mine) {
                const int i = __ffs(mine) - 1;
                mine &= mine - 1;
                const int j = jr + i;
                row_sm[j + (j >> 5)] = r < C_r ? r : -1;  // -1: receiver-dropped
                ++r;
            }
            bk_sync<NT, BAR>();  // everyone has read carry[pp]
            if (tid == 0) carry[pp] += total;
        }
        bk_sync<NT, BAR>();

        // 3. arrivals' rows and bucket entries, in position order
        for (int j = tid; j < TILE; j += NT) {
            const int64_t q = t0 + j;
            const int pe = pe_sm[j];
            if (q < npos && pe >= 0) {
                const uint32_t sq = uint32_t(q) / Cs32, c = uint32_t(q) - sq * Cs32;
                const int64_t slot = (pool_s0 + int64_t(sq) * pool_step) * C_s + c;
                const int32_t row = row_sm[j + (j >> 5)];
                p.recv_row[slot] = row;
                if (row >= 0) p.bucket_slot[int64_t(e0 - e_base + pe) * C_r + row] = int32_t(slot);
            }
        }
        bk_sync<NT, BAR>();  // pe_sm and row_sm are refilled by the next tile
    }

    for (int pp = 0; pp < P; ++pp) {
        const int32_t arrivals = carry[pp];
        const int64_t kept = arrivals < C_r ? arrivals : C_r;
        const int32_t e = e0 - e_base + pp;  // index among this GPU's experts
        for (int64_t r = kept + tid; r < C_r; r += NT)
            p.bucket_slot[int64_t(e) * C_r + r] = -1;
        if (tid == 0) {
            p.expert_counts[e] = arrivals;
            p.expert_counts[E_out + e] = int32_t(kept);
            if (arrivals > kept)
                atomicAdd(&p.ctr->receiver_dropped, (unsigned long long)(arrivals - kept));
            atomicAdd(&p.ctr->kept, (unsigned long long)kept);
            atomicMax(&p.ctr->max_fill, int32_t(kept));
        }
    }
    if (FUSED) bk_sync<NT, BAR>();  // carry is reset by the worker's next item
}

}  // namespace moe_pw
