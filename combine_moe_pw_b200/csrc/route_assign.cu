// route_assign.cu - router and sender slot assignment in one launch (pooled
// mode, one GPU).
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 二: the router picks 8 of the
// 384 experts per token; each source fills one fixed pool per (destination,
// wave), capped by the 1.10 sender factor.  The results are those of the
// route kernel followed by the assignment passes (assign.cu): choice (t, j)
// of source s with pool b = (e / L) * W + (e % L) / P takes rank r = the
// number of earlier choices of s in flat (t, j) order with the same pool;
// slot = (s * R*W + b) * C_s + r, kept iff r < C_s.
//
// One thread-block cluster of c blocks per source shard.  Block j of the
// cluster routes the tokens [T_s*j/c, T_s*(j+1)/c) of the source, warp w a
// contiguous eighth of them (the selection of route_body.cuh), and keeps each
// choice's expert id in shared memory with a per-warp pool histogram.  Then
//   1. per pool: the warps' exclusive prefix and the block's total;
//   2. cluster barrier; the block sums the totals of the cluster's earlier
//      blocks through distributed shared memory (its base per pool); the
//      cluster's last block also writes the occupancies and sender drops;
//   3. each warp ranks its own choices in (t, j) order, 32 at a time (lanes
//      with the same pool find each other through shared-memory lane masks)
//      and writes slot_map and the kept slots' headers;
//   4. cluster barrier before exit, so no block leaves while another may
//      still read its shared memory.
// The only waits are the two hardware cluster barriers: no block waits on
// another cluster, so clusters may run in any order and in any number of
// waves.  The cluster size is the largest (up to 16) at which every source's
// cluster is resident at once.
//
// Larger batches take route_kernel and the assignment passes instead: a
// cluster is tied to one source shard, so its blocks cannot spread the route
// work evenly over the SMs (see ra_form below).
#include <cooperative_groups.h>

#include <map>
#include <mutex>
#include <tuple>

#include "route_body.cuh"

namespace cg = cooperative_groups;

namespace moe_pw {

namespace {

#ifndef MOE_PW_RA_WARPS
#define MOE_PW_RA_WARPS 8
#endif
constexpr int RA_WARPS = MOE_PW_RA_WARPS;   // warps per block
constexpr int RA_MIN_BLOCKS = 32 / RA_WARPS;  // as the route kernel: 64 registers
constexpr int RA_MAX_CLUSTER = 16;
constexpr size_t RA_MAX_SMEM = 40 * 1024;  // dynamic, beside the static; keeps 4 blocks per SM

struct RouteAssignArgs {
    const float *logits;
    int32_t *idx;
    float *gates;
    int32_t *slot_map;
    int32_t *occ;
    int32_t *pool_hdr;
    moe_pw_counters *ctr;
    Geo g;
    int32_t c;  // blocks per source (the cluster size)
};

// Dynamic shared memory: pool of each expert [E], per-warp pool counts and
// lane masks [2][RA_WARPS][NB], block totals [NB], expert id of each choice
// [tokens * k] (int16).
inline size_t ra_smem_bytes(const Geo &g, int64_t tok_cap)
{
    const size_t ints = size_t(g.E) + size_t(2 * RA_WARPS + 1) * g.NB;
    return (sizeof(int32_t) * ints + sizeof(int16_t) * size_t(tok_cap) * g.k + 15) & ~size_t(15);
}

template <int NV, bool FULL, int KC>
__global__ void __launch_bounds__(RA_WARPS * 32, RA_MIN_BLOCKS)
route_assign_kernel(RouteAssignArgs p)
{
    __shared__ __align__(16) unsigned long long cand_sm[RA_WARPS][32];
    __shared__ unsigned long long sel_sm[RA_WARPS][32];
    __shared__ uint4 key_sm[RA_WARPS][KeyRows<NV>::V][32];
    extern __shared__ __align__(16) int32_t dsm[];
    cg::cluster_group cluster = cg::this_cluster();
    const int NB = p.g.NB;
    int32_t *bin_tab = dsm;                                    // [E]
    int32_t *hist = bin_tab + p.g.E;                           // [RA_WARPS][NB]
    uint32_t *wmask = reinterpret_cast<uint32_t *>(hist + RA_WARPS * NB);  // [RA_WARPS][NB]
    int32_t *tot = reinterpret_cast<int32_t *>(wmask + RA_WARPS * NB);     // [NB]
    int16_t *choice = reinterpret_cast<int16_t *>(tot + NB);              // [tokens * k]
    const int k = KC ? KC : p.g.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c = p.c;
    const int j = int(cluster.block_rank());
    const int s = int(blockIdx.x) / c;
    const int64_t Ts = p.g.T_s;
    const int64_t tb0 = int64_t(s) * Ts + Ts * j / c;
    const int nb = int(int64_t(s) * Ts + Ts * (j + 1) / c - tb0);
    const int tw0 = nb * warp / RA_WARPS, tw1 = nb * (warp + 1) / RA_WARPS;

    for (int e = threadIdx.x; e < p.g.E; e += blockDim.x) bin_tab[e] = bin_of_expert(p.g, e);
    for (int i = threadIdx.x; i < RA_WARPS * NB; i += blockDim.x) {
        hist[i] = 0;
        wmask[i] = 0u;
    }
    __syncthreads();

    // route this warp's tokens (the next row loads during the selection)
    const int E4 = p.g.E >> 2;
    int32_t *h = hist + warp * NB;
    auto one = [&](int t, const float4 (&row)[NV]) {
        int32_t e;
        float ex, sum;
        route_select<NV, FULL, KC, RA_WARPS>(row, k, E4, lane, warp, cand_sm, sel_sm, key_sm, e,
                                             ex, sum);
        if (lane < k) {
            const int64_t a = (tb0 + t) * k + lane;
            p.idx[a] = e;
            p.gates[a] = ex / sum;
            choice[t * k + lane] = int16_t(e);
            atomicAdd(&h[bin_tab[e]], 1);
        }
    };
    float4 cur[NV], nxt[NV];
    if (tw0 < tw1) load_row<NV, FULL>(p.logits, tb0 + tw0, E4, lane, cur);
    for (int t = tw0; t < tw1; ++t) {
        if (t + 1 < tw1) load_row<NV, FULL>(p.logits, tb0 + t + 1, E4, lane, nxt);
        one(t, cur);
#pragma unroll
        for (int v = 0; v < NV; ++v) cur[v] = nxt[v];
    }
    __syncthreads();

    // 1. warps' exclusive prefix and the block total, per pool
    for (int b = threadIdx.x; b < NB; b += blockDim.x) {
        int32_t run = 0;
        for (int w = 0; w < RA_WARPS; ++w) {
            const int32_t v = hist[w * NB + b];
            hist[w * NB + b] = run;
            run += v;
        }
        tot[b] = run;
    }
    cluster.sync();

    // 2. base = the totals of the cluster's earlier blocks
    const int64_t C_s = p.g.C_s;
    for (int b = threadIdx.x; b < NB; b += blockDim.x) {
        int32_t base = 0;
        for (int jj = 0; jj < j; ++jj) base += cluster.map_shared_rank(tot, jj)[b];
        if (j == c - 1) {
            const int32_t total = base + tot[b];
            const int32_t kept = total < C_s ? total : int32_t(C_s);
            p.occ[int64_t(s) * NB + b] = kept;
            if (total > kept)
                atomicAdd(&p.ctr->sender_dropped, (unsigned long long)(total - kept));
            atomicMax(&p.ctr->max_occ, kept);
        }
        for (int w = 0; w < RA_WARPS; ++w) hist[w * NB + b] += base;
    }
    __syncthreads();

    // 3. rank this warp's choices in (t, j) order
    const int64_t pool_base = int64_t(s) * NB;
    uint32_t *wm = wmask + warp * NB;
    const int aw0 = tw0 * k, aw1 = tw1 * k;
    for (int a = aw0; a < aw1; a += 32) {
        const int i = a + lane;
        const int32_t e = i < aw1 ? int32_t(choice[i]) : -1;
        const int32_t b = e >= 0 ? bin_tab[e] : -1;
        const unsigned same = equal_lanes_smem(b, wm, lane);
        const int32_t r = (b >= 0 ? h[b] : 0) + __popc(same & lanemask_lt());
        __syncwarp();
        if (b >= 0 && lane == __ffs(same) - 1) {
            h[b] += __popc(same);
            wm[b] = 0u;
        }
        __syncwarp();
        if (i < aw1) {
            int32_t slot = -1;
            if (r < C_s) slot = int32_t((pool_base + b) * C_s + r);
            p.slot_map[tb0 * k + i] = slot;
            if (slot >= 0) p.pool_hdr[slot] = e;
        }
    }
    cluster.sync();  // the other blocks have finished reading tot
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline void cluster_config(cudaLaunchConfig_t &cfg, cudaLaunchAttribute *attr, const Geo &g,
                           int c, size_t smem)
{
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = dim3(unsigned(g.R) * unsigned(c));
    cfg.blockDim = dim3(RA_WARPS * 32);
    cfg.dynamicSmemBytes = smem;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(c);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
}

// Cluster size per (kernel, device, batch shape): the largest
// c <= min(16, T_s) whose blocks fit RA_MAX_SMEM and at which every source's
// cluster is resident at once, else the smallest c that fits and can be
// placed at all (the clusters then run in waves); 0 if none.  Cached: the
// occupancy queries run once per shape.
template <typename Kern>
int pick_cluster(Kern kern, const Geo &g)
{
    static std::mutex mu;
    static std::map<std::tuple<const void *, int, int64_t, int64_t, int32_t, int32_t, int32_t>,
                    int>
        cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    // everything the shared memory per block and the grid depend on
    const auto key = std::make_tuple(reinterpret_cast<const void *>(kern), dev, int64_t(g.R),
                                     g.T_s, g.E, g.NB, g.k);
    {
        std::lock_guard<std::mutex> lk(mu);
        const auto it = cache.find(key);
        if (it != cache.end()) return it->second;
    }
    int best = 0, fallback = 0;
    const int cmax = int(g.T_s < RA_MAX_CLUSTER ? g.T_s : RA_MAX_CLUSTER);
    for (int c = cmax; c >= 1; --c) {
        const size_t smem = ra_smem_bytes(g, ceil_div(g.T_s, c));
        if (smem > RA_MAX_SMEM) break;  // fewer blocks per source only need more
        cudaLaunchConfig_t cfg;
        cudaLaunchAttribute attr[1];
        cluster_config(cfg, attr, g, c, smem);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            cudaGetLastError();  // clear: a cluster size the device refuses
            continue;
        }
        if (n >= g.R) {
            best = c;
            break;
        }
        if (n > 0) fallback = c;
    }
    if (best == 0) best = fallback;
    std::lock_guard<std::mutex> lk(mu);
    cache[key] = best;
    return best;
}

// c_out: only pick the cluster size (0: the one launch does not apply)
template <int NV, bool FULL, int KC>
cudaError_t launch_ra(const RouteAssignArgs &p0, cudaStream_t st, int *c_out)
{
    auto kern = route_assign_kernel<NV, FULL, KC>;
    const Geo &g = p0.g;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
    // up to RA_MAX_SMEM of dynamic shared memory beside the static arrays
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(RA_MAX_SMEM));
    if (err != cudaSuccess) return err;
    const int c = pick_cluster(kern, g);
    if (c_out) {
        *c_out = c;
        return cudaSuccess;
    }
    if (c == 0) return cudaErrorNotSupported;
    const size_t smem = ra_smem_bytes(g, ceil_div(g.T_s, c));
    RouteAssignArgs p = p0;
    p.c = c;
    if ((err = cudaMemsetAsync(p.ctr, 0, sizeof(moe_pw_counters), st)) != cudaSuccess) return err;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    cluster_config(cfg, attr, g, c, smem);
    cfg.stream = st;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int NV>
cudaError_t launch_ra_k(const RouteAssignArgs &p, cudaStream_t st, int *c_out)
{
    const bool full = p.g.E == 128 * NV;
    if (p.g.k == 8)
        return full ? launch_ra<NV, true, 8>(p, st, c_out) : launch_ra<NV, false, 8>(p, st, c_out);
    return full ? launch_ra<NV, true, 0>(p, st, c_out) : launch_ra<NV, false, 0>(p, st, c_out);
}

cudaError_t launch_ra_nv(const RouteAssignArgs &p, cudaStream_t st, int *c_out)
{
    const int nv = (p.g.E / 4 + 31) / 32;
    switch (nv) {
    case 1: return launch_ra_k<1>(p, st, c_out);
    case 2: return launch_ra_k<2>(p, st, c_out);
    case 3: return launch_ra_k<3>(p, st, c_out);
    case 4: return launch_ra_k<4>(p, st, c_out);
    case 5: case 6: return launch_ra_k<6>(p, st, c_out);
    case 7: case 8: return launch_ra_k<8>(p, st, c_out);
    case 9: case 10: case 11: case 12: return launch_ra_k<12>(p, st, c_out);
    default: return launch_ra_k<16>(p, st, c_out);
    }
}

// Which form takes the batch.  The clustered launch pays off on small
// batches, where the separate kernels' fixed latency (three launches) weighs
// most; on larger ones a cluster, tied to one source shard, cannot spread the
// route's token work evenly over the SMs (placement leaves some SMs a block
// more than others, up to ~15% more tokens than the even share).  Measured
// on B200 with 384 experts over 64 sources (kernels alone, route + assignment
// with its count and rank passes launched as programmatic dependents):
// 19.0 / 26.6 us (clustered / separate) at 8,192 tokens, 27.1 / 28.0 at
// 32,768, 45.5 / 44.4 at 65,536, 80.1 / 76.6 at 131,072, 149.4 / 135.7 at
// 262,144: the crossover lies near 256 tokens per SM.
constexpr int64_t RA_MAX_TOKENS_PER_SM = 256;

bool ra_shape_ok(const Geo &g)
{
    return g.mode == MOE_PW_POOLED && g.ep_n == 1 && g.T > 0 && g.E % 4 == 0 && g.E <= 32767 &&
           g.k <= 32;
}

RouteAssignArgs ra_args(const Geo &g, const float *logits, int32_t *idx, float *gates,
                        int32_t *slot_map, int32_t *occ, int32_t *pool_hdr, moe_pw_counters *ctr)
{
    RouteAssignArgs p;
    p.logits = logits;
    p.idx = idx;
    p.gates = gates;
    p.slot_map = slot_map;
    p.occ = occ;
    p.pool_hdr = pool_hdr;
    p.ctr = ctr;
    p.g = g;
    p.c = 1;
    return p;
}

// Whether the clustered launch fits the batch on the current device.
cudaError_t ra_cluster_fits(const Geo &g, bool *fits)
{
    *fits = false;
    if (!ra_shape_ok(g)) return cudaSuccess;
    int c = 0;
    const cudaError_t err =
        launch_ra_nv(ra_args(g, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr),
                     nullptr, &c);
    *fits = c > 0;
    return err;
}

// The form the batch takes by default (MOE_PW_RA_*).
cudaError_t ra_form(const Geo &g, int *form)
{
    *form = MOE_PW_RA_SEPARATE;
    bool cluster = false;
    const cudaError_t err = ra_cluster_fits(g, &cluster);
    if (err != cudaSuccess) return err;
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    if (cluster && g.T <= RA_MAX_TOKENS_PER_SM * di.sms) *form = MOE_PW_RA_CLUSTER;
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_route_assign(const Geo &g, const float *logits, int32_t *idx, float *gates,
                                int32_t *slot_map, int32_t *occ, int32_t *pool_hdr,
                                moe_pw_counters *ctr, cudaStream_t st, int form)
{
    cudaError_t err;
    if (form < 0) {
        if ((err = ra_form(g, &form)) != cudaSuccess) return err;
    } else if (form == MOE_PW_RA_CLUSTER) {
        bool fits = false;
        if ((err = ra_cluster_fits(g, &fits)) != cudaSuccess) return err;
        if (!fits) return cudaErrorInvalidValue;
    } else if (form != MOE_PW_RA_SEPARATE) {
        return cudaErrorInvalidValue;
    }
    if (form == MOE_PW_RA_CLUSTER)
        return launch_ra_nv(ra_args(g, logits, idx, gates, slot_map, occ, pool_hdr, ctr), st,
                            nullptr);
    return cudaErrorNotSupported;
}

cudaError_t route_assign_plan(const Geo &g, int *form) { return ra_form(g, form); }

}  // namespace moe_pw
