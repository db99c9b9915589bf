// assign.cu - sender slot assignment (pooled) / expert row assignment (ragged).
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 二: one fixed pool per
// (source, destination) and wave; the 1.10 sender factor caps each pool and
// the overflow is dropped.  Section 四: the dropless ragged alternative.
//
// Both modes rank every assignment (t, j) among the earlier assignments of
// its group that fall in the same bin, in flat (t, j) order:
//   pooled: group = source shard s, bin = pool (d, w) = (e / L) * W + (e % L) / P,
//           slot = (s * R*W + bin) * C_s + rank, kept iff rank < C_s;
//   ragged: one group, bin = expert e, row = offset[e] + rank.
// Work is split into chunks of consecutive tokens inside a group and done in
// three deterministic passes (no order-giving atomics):
//   1. count : per chunk, per-warp histograms in shared memory (atomics),
//              summed per bin;
//   2. scan  : per (group, bin), exclusive prefix over the group's chunks;
//   3. rank  : per chunk, recount, per-warp bases = chunk base + earlier warps,
//              then each warp walks its assignments 32 at a time: lanes with
//              the same bin find each other (each sets its bit in a per-warp
//              mask word of the bin in shared memory and reads it back) and
//              take ranks in lane order.
// Passes 1 and 3 first read the chunk's expert ids with every thread's loads
// in flight at once and keep their bins in shared memory, so the walks above
// touch only shared memory (the latency of one global read per chunk instead
// of one per 32 assignments of a warp).
// Ragged mode adds a one-block scan of the per-expert totals into offsets.
#include <cstring>

#include "common.cuh"

namespace moe_pw {

namespace {

constexpr int AW = 8;  // warps per block in count/rank
// Blocks per SM the count and rank passes are compiled for (32 registers): a
// rack-size batch has 1024 chunks, which then all run in one wave on 148 SMs
// (at 38-40 registers only 6 blocks fit, and a seventh block per SM started
// one block's time late).
constexpr int AW_MIN_BLOCKS = 8;
constexpr int MAX_FUSED_CHUNKS = 32;

struct RankArgs {
    const int32_t *idx;
    int32_t *slot_map;
    int32_t *occ;
    int32_t *counts;   // [n_chunks][NB], becomes the chunk bases after the scan
    int32_t *totals;   // [n_groups][NB]
    moe_pw_counters *ctr;
    Geo g;
    int32_t fused_scan;  // pooled, few chunks per group: assign_rank takes the scan's part
    int32_t *pool_hdr;   // optional: the kept slots' headers (the expert id)
};

// Flat assignment range [a0, a1) of this block's chunk and its group.
__device__ __forceinline__ void chunk_range(const Geo &g, int chunk, int64_t &a0, int64_t &a1,
                                            int &group)
{
    group = chunk / g.chunks_per_group;
    const int c = chunk - group * g.chunks_per_group;
    const int64_t g0 = int64_t(group) * g.group_tokens;
    const int64_t t0 = g0 + int64_t(c) * g.chunk_tokens;
    int64_t t1 = t0 + g.chunk_tokens;
    if (t1 > g0 + g.group_tokens) t1 = g0 + g.group_tokens;
    a0 = t0 * g.k;
    a1 = t1 * g.k;
}

// Shared-memory layout shared by count and rank.
struct Smem {
    int32_t *bin_tab;  // [E]
    int32_t *hist;     // [AW][NB]
    int32_t *off;      // [E + 1] (ragged rank pass)
    // [chunk_tokens * k]: each assignment of the chunk as (expert << 16) | bin,
    // -1 if its id is invalid (bins and ids are below 2^11, so both fit)
    int32_t *bins;
    uint32_t *wmask;   // [AW][NB]: the rank walk's lane masks, zero between steps
};

__device__ __forceinline__ int32_t bin_part(int32_t v) { return v >= 0 ? (v & 0xFFFF) : -1; }

__device__ __forceinline__ Smem carve(const Geo &g, int32_t *sm)
{
    Smem s;
    s.bin_tab = sm;
    s.hist = sm + g.E;
    s.off = s.hist + AW * g.NB;
    s.bins = s.off + g.E + 1;
    s.wmask = reinterpret_cast<uint32_t *>(s.bins + g.chunk_tokens * g.k);
    return s;
}

// bins[i] for the chunk's assignments a0 + i, i < n; the loads of one thread
// are issued together.  flag: report ids outside [0, E) (rank pass).  The
// expert id stays beside the bin, so the rank walk's header stores need no
// second global read.
__device__ __forceinline__ void load_bins(const RankArgs &p, const Smem &s, int64_t a0, int n,
                                          bool flag)
{
    constexpr int U = 8;
    for (int i0 = threadIdx.x; i0 < n; i0 += U * blockDim.x) {
        int32_t e[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * int(blockDim.x);
            e[u] = i < n ? p.idx[a0 + i] : 0;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * int(blockDim.x);
            if (i < n) {
                int32_t v = -1;
                if (e[u] >= 0 && e[u] < p.g.E)
                    v = (e[u] << 16) | s.bin_tab[e[u]];
                else if (flag)
                    set_error(p.ctr, MOE_PW_DEVERR_EXPERT_ID);
                s.bins[i] = v;
            }
        }
    }
}

// Per-warp histogram of this warp's slice [w0, w1) of the chunk
// (shared-memory atomics: the counts do not depend on their order).
__device__ __forceinline__ void warp_hist(const RankArgs &p, const Smem &s, int w0, int w1,
                                          int warp, int lane)
{
    int32_t *h = s.hist + warp * p.g.NB;
    for (int i = w0 + lane; i < w1; i += 32) {
        const int32_t b = bin_part(s.bins[i]);
        if (b >= 0) atomicAdd(&h[b], 1);
    }
}

__device__ __forceinline__ void setup(const RankArgs &p, const Smem &s)
{
    for (int e = threadIdx.x; e < p.g.E; e += blockDim.x) s.bin_tab[e] = bin_of_expert(p.g, e);
    for (int i = threadIdx.x; i < AW * p.g.NB; i += blockDim.x) {
        s.hist[i] = 0;
        s.wmask[i] = 0u;
    }
}

size_t rank_smem_bytes(const Geo &g)
{
    return sizeof(int32_t) * (size_t(g.E) + 2 * size_t(AW) * g.NB + size_t(g.E) + 1 +
                              size_t(g.chunk_tokens) * g.k);
}

// Rank the assignments of one chunk (pass 3): recount, per-warp bases =
// chunk base + earlier warps, then each warp walks its assignments 32 at a
// time and writes their slots (and, with pool_hdr, the kept slots' headers).
// Expects bin_tab filled, hist and wmask zeroed and (ragged) off loaded, with the
// block synchronised after; AW warps take part.
__device__ __forceinline__ void rank_chunk(const RankArgs &p, const Smem &s, int chunk)
{
    const bool ragged = p.g.mode == MOE_PW_RAGGED;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int64_t a0, a1;
    int group;
    chunk_range(p.g, chunk, a0, a1, group);
    const int n = int(a1 - a0);
    load_bins(p, s, a0, n, true);
    __syncthreads();
    const int w0 = n * warp / AW, w1 = n * (warp + 1) / AW;
    warp_hist(p, s, w0, w1, warp, lane);
    __syncthreads();
    // turn per-warp counts into per-warp starting ranks.  The chunk's base
    // is the scan pass's output, or (few chunks per group) the sum of the
    // earlier chunks' raw counts, taken here; then the group's last chunk
    // also settles the pools' occupancy and drops, which the scan pass
    // would have done.
    const int cpg = p.g.chunks_per_group;
    const int ci = chunk - group * cpg;
    for (int b = threadIdx.x; b < p.g.NB; b += blockDim.x) {
        int32_t run = 0;
        if (p.fused_scan) {
            const int32_t *col = p.counts + int64_t(group) * cpg * p.g.NB + b;
            for (int c = 0; c < ci; ++c) run += col[int64_t(c) * p.g.NB];
        } else {
            run = p.counts[int64_t(chunk) * p.g.NB + b];
        }
        for (int w = 0; w < AW; ++w) {
            const int32_t v = s.hist[w * p.g.NB + b];
            s.hist[w * p.g.NB + b] = run;
            run += v;
        }
        if (p.fused_scan && ci == cpg - 1) {
            // run = the pool's total over the whole group
            const int64_t kept = run < p.g.C_s ? run : p.g.C_s;
            p.occ[int64_t(group) * p.g.NB + b] = int32_t(kept);
            if (run > kept) atomicAdd(&p.ctr->sender_dropped, (unsigned long long)(run - kept));
            atomicMax(&p.ctr->max_occ, int32_t(kept));
        }
    }
    __syncthreads();
    int32_t *h = s.hist + warp * p.g.NB;
    uint32_t *wm = s.wmask + warp * p.g.NB;
    const int64_t pool_base = int64_t(group) * p.g.NB;
    for (int a = w0; a < w1; a += 32) {
        const int i = a + lane;
        const int32_t v = i < w1 ? s.bins[i] : -1;
        const int32_t b = bin_part(v);
        const unsigned same = equal_lanes_smem(b, wm, lane);
        const int32_t r = (b >= 0 ? h[b] : 0) + __popc(same & lanemask_lt());
        __syncwarp();
        if (b >= 0 && lane == __ffs(same) - 1) {
            h[b] += __popc(same);
            wm[b] = 0u;
        }
        __syncwarp();
        if (i < w1) {
            int32_t slot = -1;
            if (b >= 0) {
                if (ragged)
                    slot = s.off[b] + r;
                else if (r < p.g.C_s)
                    slot = int32_t((pool_base + b) * p.g.C_s + r);
            }
            p.slot_map[a0 + i] = slot;
            if (p.pool_hdr && slot >= 0) p.pool_hdr[slot] = v >> 16;
        }
    }
}


// Launched as a programmatic dependent of the route: the shared-memory
// set-up overlaps the route's last blocks.  Zeroes the counters.
__global__ void __launch_bounds__(AW * 32, AW_MIN_BLOCKS) assign_count(RankArgs p)
{
    extern __shared__ int32_t sm[];
    const Smem s = carve(p.g, sm);
    setup(p, s);
    griddep_wait();
    if (blockIdx.x == 0 && threadIdx.x < sizeof(moe_pw_counters) / sizeof(uint32_t))
        reinterpret_cast<uint32_t *>(p.ctr)[threadIdx.x] = 0u;
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int64_t a0, a1;
    int group;
    chunk_range(p.g, blockIdx.x, a0, a1, group);
    const int n = int(a1 - a0);
    load_bins(p, s, a0, n, false);
    __syncthreads();
    warp_hist(p, s, n * warp / AW, n * (warp + 1) / AW, warp, lane);
    __syncthreads();
    int32_t *out = p.counts + int64_t(blockIdx.x) * p.g.NB;
    for (int b = threadIdx.x; b < p.g.NB; b += blockDim.x) {
        int32_t sum = 0;
        for (int w = 0; w < AW; ++w) sum += s.hist[w * p.g.NB + b];
        out[b] = sum;
    }
}

// Block (32 warps) per (group, 32-bin tile): exclusive scan over the group's
// chunks, in place; totals, occupancy and sender drops.
__global__ void __launch_bounds__(1024) assign_scan(RankArgs p)
{
    __shared__ int32_t part[32][33];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int group = blockIdx.y;
    const int b = blockIdx.x * 32 + lane;
    const int cpg = p.g.chunks_per_group;
    const int c0 = cpg * warp / 32, c1 = cpg * (warp + 1) / 32;
    int32_t *col = p.counts + int64_t(group) * cpg * p.g.NB + b;
    int32_t sum = 0;
    if (b < p.g.NB)
        for (int c = c0; c < c1; ++c) sum += col[int64_t(c) * p.g.NB];
    part[warp][lane] = sum;
    __syncthreads();
    if (warp == 0) {
        int32_t run = 0;
        for (int w = 0; w < 32; ++w) {
            const int32_t v = part[w][lane];
            part[w][lane] = run;
            run += v;
        }
        if (b < p.g.NB) {
            p.totals[int64_t(group) * p.g.NB + b] = run;
            if (p.g.mode == MOE_PW_POOLED) {
                const int64_t kept = run < p.g.C_s ? run : p.g.C_s;
                p.occ[int64_t(group) * p.g.NB + b] = int32_t(kept);
                if (run > kept) atomicAdd(&p.ctr->sender_dropped, (unsigned long long)(run - kept));
                atomicMax(&p.ctr->max_occ, int32_t(kept));
            }
        }
    }
    __syncthreads();
    if (b < p.g.NB) {
        int32_t run = part[warp][lane];
        for (int c = c0; c < c1; ++c) {
            const int32_t v = col[int64_t(c) * p.g.NB];
            col[int64_t(c) * p.g.NB] = run;
            run += v;
        }
    }
}

// Ragged: occ[0..E] = exclusive scan of the per-expert totals (one block).
__global__ void __launch_bounds__(1024) ragged_offsets(RankArgs p)
{
    __shared__ int32_t wsum[32];
    const int E = p.g.E;
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = threadIdx.x * per;
    int32_t local = 0;
    for (int e = e0; e < e0 + per && e < E; ++e) local += p.totals[e];
    // block exclusive scan of `local`
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t incl = local;
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(FULL_MASK, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int32_t v = lane < nw ? wsum[lane] : 0;
        int32_t inc = v;
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(FULL_MASK, inc, o);
            if (lane >= o) inc += u;
        }
        if (lane < nw) wsum[lane] = inc - v;
    }
    __syncthreads();
    int32_t run = wsum[warp] + incl - local;
    for (int e = e0; e < e0 + per && e < E; ++e) {
        p.occ[e] = run;
        run += p.totals[e];
    }
    if (threadIdx.x == blockDim.x - 1) p.occ[E] = run;
}

// Launched as a programmatic dependent of the count (or scan) pass.
__global__ void __launch_bounds__(AW * 32, AW_MIN_BLOCKS) assign_rank(RankArgs p)
{
    extern __shared__ int32_t sm[];
    const Smem s = carve(p.g, sm);
    setup(p, s);
    griddep_wait();
    if (p.g.mode == MOE_PW_RAGGED)
        for (int e = threadIdx.x; e <= p.g.E; e += blockDim.x) s.off[e] = p.occ[e];
    __syncthreads();
    rank_chunk(p, s, int(blockIdx.x));
}


}  // namespace

cudaError_t launch_assign(const Geo &g, const int32_t *idx, int32_t *slot_map, int32_t *occ,
                          moe_pw_counters *ctr, void *ws, cudaStream_t st, int32_t *pool_hdr)
{
    cudaError_t err;
    const int64_t occ_len = g.mode == MOE_PW_POOLED ? g.n_pools : int64_t(g.E) + 1;
    if (g.T == 0) {
        if ((err = cudaMemsetAsync(ctr, 0, sizeof(moe_pw_counters), st)) != cudaSuccess)
            return err;
        return cudaMemsetAsync(occ, 0, sizeof(int32_t) * occ_len, st);
    }

    RankArgs p;
    memset(&p, 0, sizeof(p));
    p.idx = idx;
    p.slot_map = slot_map;
    p.occ = occ;
    p.counts = static_cast<int32_t *>(ws);
    p.totals = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + ws_counts_bytes(g));
    p.ctr = ctr;
    p.g = g;
    p.pool_hdr = pool_hdr;

    const size_t smem = rank_smem_bytes(g);
    if (smem > 48 * 1024) {
        // the opt-in is a per-function attribute; setting it again is harmless
        DevInfo di;
        if (dev_info(&di) != 0) return cudaErrorUnknown;
        if ((err = cudaFuncSetAttribute(assign_count, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        di.smem_optin)) != cudaSuccess)
            return err;
        if ((err = cudaFuncSetAttribute(assign_rank, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        di.smem_optin)) != cudaSuccess)
            return err;
    }
    // with at most MAX_FUSED_CHUNKS chunks per source the rank pass sums the
    // earlier chunks' counts itself and the scan pass is skipped (pooled mode)
    p.fused_scan = g.mode == MOE_PW_POOLED && g.chunks_per_group <= MAX_FUSED_CHUNKS;
    // the count and rank passes start under the previous kernel's tail
    // (programmatic dependent launch; they wait for it before any global access)
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(unsigned(g.n_chunks));
    cfg.blockDim = dim3(AW * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((err = cudaLaunchKernelEx(&cfg, assign_count, p)) != cudaSuccess) return err;
    if (!p.fused_scan) {
        dim3 sgrid((g.NB + 31) / 32, g.n_groups);
        assign_scan<<<sgrid, 1024, 0, st>>>(p);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    if (g.mode == MOE_PW_RAGGED) {
        ragged_offsets<<<1, 1024, 0, st>>>(p);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    return cudaLaunchKernelEx(&cfg, assign_rank, p);
}

}  // namespace moe_pw
