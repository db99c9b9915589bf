// bucket.cu - exchange (index relabel) + receiver bucketing.
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 二: the 1.15 receiver factor
// caps the rows a local expert accepts; overflow is dropped and counted apart
// from sender drops.  The all-to-all gives destination d the pools (s, d, w);
// on one GPU destination d simply reads them where source s wrote them.
//
// Pooled: one block per (d, w); an arrival's row in its expert bucket is the
// number of earlier arrivals (sources ascending, then slots ascending) with
// the same header.  Positions c >= occ are empty.
// Ragged: rows are already grouped by expert; row r of expert e is r - off[e].
#include "common.cuh"

namespace moe_pw {

namespace {

struct BucketArgs {
    const int32_t *pool_hdr;
    const int32_t *occ;
    int32_t *recv_row;
    int32_t *bucket_slot;
    int32_t *expert_counts;
    moe_pw_counters *ctr;
    Geo g;
    uint32_t wave_mask;  // waves whose blocks run
};

// One block per (destination d, wave w).  Its positions q = s * C_s + c run
// over the R pools (s, d, w) in arrival order (sources ascending, then slots
// ascending); slots c >= occ are empty.  The row of an arrival with local
// expert pp is the number of earlier positions with the same expert, i.e. an
// exclusive prefix count over q, so the block works in tiles of
// BK_THREADS * BK_ITEMS positions:
//   1. local experts of the tile into shared memory, position j of the tile
//      by thread j % BK_THREADS (every header and occupancy read of a thread
//      issued together; empty and dropped positions get recv_row -1 here);
//   2. per local expert: thread t counts its contiguous run of BK_ITEMS
//      positions, a block-wide exclusive scan gives the run's first row, and
//      the thread numbers its arrivals in order into shared memory;
//   3. recv_row and bucket_slot are written in position order (coalesced),
//      and the per-expert carry moves to the next tile.
constexpr int BK_THREADS = 512;
constexpr int BK_ITEMS = 32;
constexpr int BK_TILE = BK_THREADS * BK_ITEMS;
static_assert(BK_ITEMS == 32, "a thread's run is one 32-bit mask per local expert");

// Block-wide exclusive scan of v (all threads call it); *total gets the sum.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t *wsum, int32_t *total)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(FULL_MASK, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        constexpr int NW = BK_THREADS / 32;
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
    __syncthreads();
    const int32_t r = wsum[warp] + inc - v;
    *total = wsum[BK_THREADS / 32];
    __syncthreads();  // wsum is reused by the next scan
    return r;
}

__global__ void __launch_bounds__(BK_THREADS, 2) bucket_pooled(BucketArgs p)
{
    extern __shared__ __align__(16) int32_t sm[];
    const int P = p.g.P, R = p.g.R;
    int8_t *pe_sm = reinterpret_cast<int8_t *>(sm);  // [BK_TILE]
    int32_t *row_sm = sm + BK_TILE / 4;              // [BK_TILE + BK_TILE / 32], padded
    int32_t *carry = row_sm + BK_TILE + BK_TILE / 32;  // [P]
    int32_t *wsum = carry + P;                       // [BK_THREADS / 32 + 1]
    // block (d, w): d is this GPU's d-th destination rank (all of them on one
    // GPU); its pools (s, d, w) for the R sources s sit at pool_s0 + s * pool_step
    const int dw = blockIdx.x;
    const int d = dw / p.g.W, w = dw - d * p.g.W;
    if (!((p.wave_mask >> w) & 1u)) return;
    const int32_t e_base = p.g.ep_g * p.g.Rn * p.g.L;  // first expert on this GPU
    const int32_t E_out = p.g.Rn * p.g.L;              // experts of this GPU
    const int32_t e0 = (p.g.ep_g * p.g.Rn + d) * p.g.L + w * p.g.P;
    const int64_t C_s = p.g.C_s, C_r = p.g.C_r;
    const int64_t npos = int64_t(R) * C_s;
    const int64_t pool_s0 = int64_t(d) * p.g.W + w;
    const int64_t pool_step = int64_t(p.g.Rn) * p.g.W;
    for (int i = threadIdx.x; i < P; i += blockDim.x) carry[i] = 0;

    for (int64_t t0 = 0; t0 < npos; t0 += BK_TILE) {
        // 1. local experts of the tile (positions fit in 32 bits: npos <= n_slots)
        constexpr int U = 4;
        const uint32_t Cs32 = uint32_t(C_s);
        for (int j0 = 0; j0 < BK_TILE; j0 += U * BK_THREADS) {
            int32_t hdr[U], occ[U];
            uint32_t cc[U], slot[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t q = t0 + j0 + u * BK_THREADS + threadIdx.x;
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
                const int j = j0 + u * BK_THREADS + threadIdx.x;
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
                    }
                    if (pe < 0) p.recv_row[slot[u]] = -1;
                }
                pe_sm[j] = int8_t(pe);
            }
        }
        __syncthreads();

        // 2. rows, one local expert at a time; the thread's run of local
        //    experts is read once, 16 bytes at a time
        const int jr = threadIdx.x * BK_ITEMS;  // this thread's run [jr, jr + BK_ITEMS)
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
            const int32_t first = block_exclusive_scan(__popc(mine), wsum, &total);
            int32_t r = carry[pp] + first;
            while (mine) {
                const int i = __ffs(mine) - 1;
                mine &= mine - 1;
                const int j = jr + i;
                row_sm[j + (j >> 5)] = r < C_r ? r : -1;  // -1: receiver-dropped
                ++r;
            }
            __syncthreads();  // everyone has read carry[pp]
            if (threadIdx.x == 0) carry[pp] += total;
        }
        __syncthreads();

        // 3. arrivals' rows and bucket entries, in position order
        for (int j = threadIdx.x; j < BK_TILE; j += BK_THREADS) {
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
        __syncthreads();  // pe_sm and row_sm are refilled by the next tile
    }

    for (int pp = 0; pp < P; ++pp) {
        const int32_t arrivals = carry[pp];
        const int64_t kept = arrivals < C_r ? arrivals : C_r;
        const int32_t e = e0 - e_base + pp;  // index among this GPU's experts
        for (int64_t r = kept + threadIdx.x; r < C_r; r += blockDim.x)
            p.bucket_slot[int64_t(e) * C_r + r] = -1;
        if (threadIdx.x == 0) {
            p.expert_counts[e] = arrivals;
            p.expert_counts[E_out + e] = int32_t(kept);
            if (arrivals > kept)
                atomicAdd(&p.ctr->receiver_dropped, (unsigned long long)(arrivals - kept));
            atomicAdd(&p.ctr->kept, (unsigned long long)kept);
            atomicMax(&p.ctr->max_fill, int32_t(kept));
        }
    }
}

__global__ void bucket_ragged(BucketArgs p)
{
    const int64_t n = p.g.n_slots;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t q = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; q < n; q += stride) {
        const int32_t e = p.pool_hdr[q];
        int32_t row = -1;
        if (e >= 0 && e < p.g.E)
            row = int32_t(q - p.occ[e]);
        else
            set_error(p.ctr, MOE_PW_DEVERR_HEADER);
        p.recv_row[q] = row;
    }
    for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < p.g.E; e += stride) {
        const int32_t cnt = p.occ[e + 1] - p.occ[e];
        p.expert_counts[e] = cnt;
        p.expert_counts[p.g.E + e] = cnt;
        atomicMax(&p.ctr->max_fill, cnt);
        atomicAdd(&p.ctr->kept, (unsigned long long)cnt);
    }
}

}  // namespace

cudaError_t launch_bucket(const Geo &g, const int32_t *pool_hdr, const int32_t *occ,
                          int32_t *recv_row, int32_t *bucket_slot, int32_t *expert_counts,
                          moe_pw_counters *ctr, cudaStream_t st, uint32_t wave_mask)
{
    BucketArgs p;
    p.pool_hdr = pool_hdr;
    p.occ = occ;
    p.recv_row = recv_row;
    p.bucket_slot = bucket_slot;
    p.expert_counts = expert_counts;
    p.ctr = ctr;
    p.g = g;
    p.wave_mask = wave_mask;
    if (g.T == 0 && g.ep_n == 1)
        return cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * 2 * g.E, st);
    if (g.mode == MOE_PW_POOLED) {
        const size_t smem = BK_TILE + sizeof(int32_t) * (BK_TILE + BK_TILE / 32 + size_t(g.P) +
                                                         BK_THREADS / 32 + 1);
        const cudaError_t aerr = cudaFuncSetAttribute(
            bucket_pooled, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (aerr != cudaSuccess) return aerr;
        bucket_pooled<<<g.Rn * g.W, BK_THREADS, smem, st>>>(p);
    } else {
        DevInfo di;
        if (dev_info(&di) != 0) return cudaErrorUnknown;
        int64_t blocks = (g.n_slots + 255) / 256;
        if (blocks > int64_t(di.sms) * 8) blocks = int64_t(di.sms) * 8;
        bucket_ragged<<<unsigned(blocks), 256, 0, st>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace moe_pw
