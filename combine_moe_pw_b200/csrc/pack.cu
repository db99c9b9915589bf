// pack.cu - copy each kept row into its pool slot(s) with TMA bulk copies.
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 二: the sender fills fixed
// per-destination pools and the expert id travels with the row, so the
// receiver needs no separate counts.  Empty slots get a zero row and header -1
// (this library's reading), which makes the pools deterministic byte for byte.
//
// Design (HBM-bound permutation, no tensor cores):
//   - persistent grid, one CTA per SM; each CTA runs MOE_PW_PACK_WARPS
//     independent pipelines (one warp each) over a ring of row stages in
//     shared memory (up to MOE_PW_PACK_MAX_STAGES, fewer for very wide rows);
//   - warps sweep the batch together: step i of warp g handles token
//     g + i * (number of warps), so the stores in flight at any moment land in
//     neighbouring slots of the pools of one source shard instead of being
//     spread over the whole pool array (measured: ~8% faster on B200);
//   - for token t one lane issues a single cp.async.bulk load of the whole row
//     x[t] (2*D bytes) into a stage, tracked by an mbarrier;
//   - when the row has landed, lane j (< k) issues the bulk store of that
//     stage into slot slot_map[t][j] and writes the slot header: one HBM read
//     of x[t] feeds up to k HBM writes, with no register traffic;
//   - a stage is refilled once the stores reading it are done
//     (cp.async.bulk.wait_group.read), LAG tokens later, so about NS - LAG row
//     loads and LAG tokens of stores stay in flight per warp;
//   - afterwards the warps zero-fill the empty tails (positions >= occ) of the
//     pools from a zeroed shared-memory row, taking pools one at a time from
//     a counter (counters->work) so that uneven tails even out.
// x is read once (evict_first); pool rows are written once (see the store policy below).
// The defaults below came from a sweep on the 262,144-token batch: deeper
// rings with fewer warps beat more warps with shallow rings; the lag between
// 8 and 20 made no measurable difference.
#include <cstring>

#include "bucket_body.cuh"
#include "common.cuh"

namespace moe_pw {

namespace {

// Pipeline shape (build-time knobs; the defaults are the tuned values).
#ifndef MOE_PW_PACK_WARPS
#define MOE_PW_PACK_WARPS 1
#endif
#ifndef MOE_PW_PACK_LAG
#define MOE_PW_PACK_LAG 12
#endif
#ifndef MOE_PW_PACK_MAX_STAGES
#define MOE_PW_PACK_MAX_STAGES 32
#endif
#ifndef MOE_PW_PACK_ZERO_TMA
#define MOE_PW_PACK_ZERO_TMA 1
#endif
#ifndef MOE_PW_PACK_INTERLEAVE
#define MOE_PW_PACK_INTERLEAVE 1
#endif
// L2 policy of the row stores: 0 evict_first, 1 evict_normal, 2 evict_last.
// Pooled pools take evict_first (each source's pools are written in a narrow
// window of the array); the dropless rows, spread over the whole expert-
// ordered array, measured 5% faster with evict_normal (and the pooled pack 1%
// slower with it).
#ifndef MOE_PW_PACK_STORE_POLICY_POOLED
#define MOE_PW_PACK_STORE_POLICY_POOLED 0
#endif
#ifndef MOE_PW_PACK_STORE_POLICY_RAGGED
#define MOE_PW_PACK_STORE_POLICY_RAGGED 1
#endif
constexpr int MAX_PACK_WARPS = MOE_PW_PACK_WARPS;
constexpr int LAG = MOE_PW_PACK_LAG;      // store groups left in flight before a refill
                                          // (smaller when the ring is shallow)
constexpr uint32_t WAIT_LIMIT = 1u << 24; // bounded mbarrier polls

struct PackArgs {
    const uint16_t *x;
    const int32_t *idx;
    const int32_t *slot_map;
    const int32_t *occ;
    uint16_t *pool_x;
    int32_t *pool_hdr;
    moe_pw_counters *ctr;
    int64_t T;
    int64_t n_slots;
    int64_t n_pools;
    int64_t C_s;
    int32_t k;
    int32_t D;
    int32_t stages;
    uint32_t rowbytes;
    // expert-parallel runs: the receive pools of every GPU and the waves sent
    Geo geo;
    uint32_t wave_mask;
    EpRows ep;
};

// Shared memory of the pack: one mbarrier per stage of every warp, the zero
// row, then the warps' rings of row stages.
__host__ __device__ inline size_t pack_bar_bytes(int warps, int stages)
{
    return (size_t(warps) * stages * sizeof(uint64_t) + 127) & ~size_t(127);
}

// Zero row and barriers, by the first `nthreads` threads of the block (the
// caller then synchronises them).
__device__ __forceinline__ void pack_init(const PackArgs &p, unsigned char *smem, int pack_warps,
                                          int nthreads)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NS = p.stages;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    unsigned char *zero = smem + pack_bar_bytes(pack_warps, NS);
    for (uint32_t i = threadIdx.x; i < p.rowbytes / 16; i += nthreads)
        reinterpret_cast<uint4 *>(zero)[i] = make_uint4(0, 0, 0, 0);
    if (lane == 0 && warp < pack_warps)
        for (int s = 0; s < NS; ++s) mbar_init(&bars[warp * NS + s], 1);
    fence_init_and_proxy();
}

// One pack warp (warp of PACK_WARPS per block) after pack_init.
// EP: rows and tails go to the destination GPUs' receive pools (peer stores).
// HDR: the pack writes the slot headers (kept: the expert; empty tail: -1);
// without it (fused with the bucketing) the assignment pass has written the
// kept slots' headers and the bucketing writes the empty ones.
template <int LAG, bool EP, bool HDR>
__device__ __forceinline__ void pack_warp(const PackArgs &p, unsigned char *smem, int warp,
                                          int lane, int PACK_WARPS)
{
    const int NS = p.stages;
    const uint32_t rb = p.rowbytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    unsigned char *zero = smem + pack_bar_bytes(PACK_WARPS, NS);
    unsigned char *bufs = zero + rb;

    const uint64_t pol_x = policy_evict_first();
    const int pol_kind = p.geo.mode == MOE_PW_RAGGED ? MOE_PW_PACK_STORE_POLICY_RAGGED
                                                     : MOE_PW_PACK_STORE_POLICY_POOLED;
    const uint64_t pol_pool = pol_kind == 0   ? policy_evict_first()
                              : pol_kind == 1 ? policy_evict_normal()
                                              : policy_evict_last();
    uint64_t *bar = bars + warp * NS;
    unsigned char *buf = bufs + size_t(warp) * NS * rb;

    const int64_t gw = int64_t(blockIdx.x) * PACK_WARPS + warp;
    const int64_t GW = int64_t(gridDim.x) * PACK_WARPS;
#if MOE_PW_PACK_INTERLEAVE
    // token of this warp's i-th step: gw + i * GW (all warps sweep the batch together)
    const int64_t t0 = gw, tstride = GW;
    const int64_t n = gw < p.T ? (p.T - gw + GW - 1) / GW : 0;
#else
    const int64_t t0 = p.T * gw / GW, tstride = 1;
    const int64_t n = p.T * (gw + 1) / GW - t0;
#endif
    const int64_t D = p.D;
    const int k = p.k;

    auto issue_load = [&](int64_t i) {
        const int s = int(i % NS);
        mbar_arrive_expect_tx(&bar[s], rb);
        bulk_g2s(buf + size_t(s) * rb, p.x + (t0 + i * tstride) * D, rb, &bar[s], pol_x);
    };

    if (lane == 0)
        for (int64_t i = 0; i < n && i < NS; ++i) issue_load(i);

    // metadata of the next token, one (slot, expert) pair per lane j < k
    int32_t nslot = -1, nexp = -1;
    if (n > 0 && lane < k) {
        nslot = p.slot_map[t0 * k + lane];
        if (HDR) nexp = p.idx[t0 * k + lane];
    }
    bool ok = true;
    for (int64_t i = 0; i < n; ++i) {
        const int32_t slot = nslot, e = nexp;
        if (i + 1 < n && lane < k) {
            const int64_t tn = t0 + (i + 1) * tstride;
            nslot = p.slot_map[tn * k + lane];
            if (HDR) nexp = p.idx[tn * k + lane];
        }
        const int s = int(i % NS);
        const uint32_t parity = uint32_t((i / NS) & 1);
        const bool landed = mbar_wait_bounded(&bar[s], parity, WAIT_LIMIT);
        if (!__all_sync(FULL_MASK, landed)) {
            // Give up on this warp's rows, but not on its own copies: the
            // loads already issued (tokens i .. last, one per stage, each on
            // its own barrier phase) still write this CTA's shared memory, so
            // wait for each of them before going on, within one more
            // WAIT_LIMIT polls in all.
            ok = false;
            const int64_t last = i < LAG ? (n < NS ? n : NS) - 1
                                         : (i - 1 - LAG + NS < n ? i - 1 - LAG + NS : n - 1);
            for (int64_t ii = i; ii <= last; ++ii)
                mbar_wait_bounded(&bar[ii % NS], uint32_t((ii / NS) & 1), WAIT_LIMIT / NS);
            break;
        }
        if (slot >= p.n_slots) {
            set_error(p.ctr, MOE_PW_DEVERR_SLOT);
        } else if (slot >= 0) {
            if (EP) {
                int h, w;
                const uint32_t rq = ep_send_to_recv(p.geo, uint32_t(slot), h, w);
                if ((p.wave_mask >> w) & 1u) {
                    bulk_s2g(p.ep.x[h] + int64_t(rq) * D, buf + size_t(s) * rb, rb, pol_pool);
                    p.ep.hdr[h][rq] = e;
                }
            } else {
                bulk_s2g(p.pool_x + int64_t(slot) * D, buf + size_t(s) * rb, rb, pol_pool);
                if (HDR) p.pool_hdr[slot] = e;
            }
        }
        bulk_commit();
        if (i >= LAG) {
            bulk_wait_read<LAG>();
            __syncwarp();
            const int64_t ii = i - LAG + NS;  // reuses the stage of token i - LAG
            if (lane == 0 && ii < n) issue_load(ii);
        }
    }
    if (!ok && lane == 0) set_error(p.ctr, MOE_PW_DEVERR_TIMEOUT);

    // zero-fill the empty tail of each pool (pooled mode).  Tails differ in
    // length (0..C_s rows), so a fixed share per warp leaves some warps with
    // far more rows than others; instead each warp takes the next pool from a
    // counter once its copies are issued (which warp fills a tail does not
    // change the result).  The next pool's number is fetched while the
    // current tail is being filled, so the counter's round trip is hidden.
    int32_t q_next = 0;
    if (lane == 0) q_next = atomicAdd(&p.ctr->work, 1);
    for (;;) {
        const int64_t q = __shfl_sync(FULL_MASK, q_next, 0);
        if (q >= p.n_pools) break;
        if (lane == 0) q_next = atomicAdd(&p.ctr->work, 1);
        int64_t filled = p.occ[q];
        if (filled < 0) filled = 0;
        if (filled > p.C_s) filled = p.C_s;
        if (EP) {
            // across GPUs only the headers of the empty tail travel: -1 marks
            // the slot empty and nothing reads an empty slot's row, so the
            // zero rows would be link bytes without information
            int h, w;
            const uint32_t rq0 = ep_send_to_recv(p.geo, uint32_t(q * p.C_s), h, w);
            if (!((p.wave_mask >> w) & 1u)) continue;
            for (int64_t c = filled + lane; c < p.C_s; c += 32) p.ep.hdr[h][rq0 + c] = -1;
            continue;
        }
#if MOE_PW_PACK_ZERO_TMA
        for (int64_t c = filled + lane; c < p.C_s; c += 32) {
            const int64_t slot = q * p.C_s + c;
            bulk_s2g(p.pool_x + slot * D, zero, rb, pol_pool);
            if (HDR) p.pool_hdr[slot] = -1;
        }
        bulk_commit();
        bulk_wait_read<8>();
#else
        // the tail is contiguous: plain 16-byte stores by the whole warp
        uint4 *tail = reinterpret_cast<uint4 *>(p.pool_x + (q * p.C_s + filled) * D);
        const int64_t n16 = (p.C_s - filled) * (rb / 16);
        for (int64_t i = lane; i < n16; i += 32) __stcs(tail + i, make_uint4(0, 0, 0, 0));
        if (HDR)
            for (int64_t c = filled + lane; c < p.C_s; c += 32) p.pool_hdr[q * p.C_s + c] = -1;
#endif
    }
    bulk_wait_all();
    if (EP) {
        // the peer stores (bulk and plain) are performed; order them before
        // anything this GPU signals to the others after the kernel
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence_system();
    }
}

template <int LAG, bool EP>
__global__ void __launch_bounds__(MAX_PACK_WARPS * 32) pack_kernel(PackArgs p)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int PACK_WARPS = blockDim.x >> 5;
    pack_init(p, smem, PACK_WARPS, blockDim.x);
    __syncthreads();
    pack_warp<LAG, EP, true>(p, smem, threadIdx.x >> 5, threadIdx.x & 31, PACK_WARPS);
}

// Pack and receiver bucketing in one launch (one GPU, pooled mode).  The
// bucketing needs only the occupancies and the kept slots' headers, which
// the assignment pass has written, so it does not wait for the rows: warp 0
// of every block runs the pack pipeline (the HBM-bound copy, which leaves
// the SM's issue slots nearly idle), and the block's other BKF_THREADS
// threads take bucket items (d, w) blockIdx.x, blockIdx.x + gridDim.x, ...
// meanwhile.  The two roles write disjoint words: the pack the rows, the
// bucketing recv_row, bucket_slot, the counts and the empty slots' headers.
constexpr int BKF_THREADS = 128;
constexpr int BKF_BAR = 1;  // named barrier of the bucketing threads

template <int LAG>
__global__ void __launch_bounds__(32 + BKF_THREADS) pack_bucket_kernel(PackArgs p, BucketArgs b,
                                                                      uint32_t bucket_off)
{
    extern __shared__ __align__(128) unsigned char smem[];
    pack_init(p, smem, 1, blockDim.x);
    griddep_wait();  // launched as a programmatic dependent of the assignment
    __syncthreads();
    if (threadIdx.x < 32) {
        pack_warp<LAG, false, false>(p, smem, 0, threadIdx.x, 1);
        return;
    }
    int32_t *bsm = reinterpret_cast<int32_t *>(smem + bucket_off);
    const int items = b.g.Rn * b.g.W;
    for (int dw = blockIdx.x; dw < items; dw += gridDim.x)
        bucket_item<BKF_THREADS, BKF_BAR, true>(b, dw, int(threadIdx.x) - 32, bsm);
}

// Blocks of a persistent launch: one wave of resident blocks, no more than
// `need`.
template <typename Kern>
cudaError_t persistent_blocks(Kern kern, int threads, size_t smem, const DevInfo &di,
                              int64_t need, int64_t *blocks)
{
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    int64_t n = int64_t(di.sms) * per_sm;
    if (n > need) n = need;
    if (n < 1) n = 1;
    *blocks = n;
    return cudaSuccess;
}

template <int LAGT, bool EP>
cudaError_t launch_lag(const PackArgs &p, const DevInfo &di, const Geo &g, int nw, size_t smem,
                       cudaStream_t st)
{
    const int64_t units = (g.T > g.n_pools ? g.T : g.n_pools);
    int64_t blocks = 0;
    cudaError_t err =
        persistent_blocks(pack_kernel<LAGT, EP>, nw * 32, smem, di, (units + nw - 1) / nw, &blocks);
    if (err != cudaSuccess) return err;
    // the zero-fill phase's pool counter starts at 0 for every launch
    if ((err = cudaMemsetAsync(&p.ctr->work, 0, sizeof(int32_t), st)) != cudaSuccess) return err;
    pack_kernel<LAGT, EP><<<unsigned(blocks), nw * 32, smem, st>>>(p);
    return cudaGetLastError();
}

template <bool EP>
cudaError_t launch_ep(const PackArgs &p, const DevInfo &di, const Geo &g, int nw, size_t smem,
                      int lag_cap, cudaStream_t st)
{
    if (lag_cap >= 12 && LAG >= 12) return launch_lag<12, EP>(p, di, g, nw, smem, st);
    if (lag_cap >= 8) return launch_lag<8, EP>(p, di, g, nw, smem, st);
    if (lag_cap >= 4) return launch_lag<4, EP>(p, di, g, nw, smem, st);
    return launch_lag<2, EP>(p, di, g, nw, smem, st);
}

template <int LAGT>
cudaError_t launch_fused_lag(const PackArgs &p, const BucketArgs &b, uint32_t bucket_off,
                             const DevInfo &di, const Geo &g, size_t smem, cudaStream_t st)
{
    const int64_t units = (g.T > g.n_pools ? g.T : g.n_pools);
    int64_t blocks = 0;
    cudaError_t err =
        persistent_blocks(pack_bucket_kernel<LAGT>, 32 + BKF_THREADS, smem, di, units, &blocks);
    if (err != cudaSuccess) return err;
    // the zero-fill hand-out counter (counters->work) starts at 0: the
    // assignment before this launch zeroed the counters.  The launch is a
    // programmatic dependent of it, so its set-up overlaps the assignment's
    // last blocks.
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(unsigned(blocks));
    cfg.blockDim = dim3(32 + BKF_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, pack_bucket_kernel<LAGT>, p, b, bucket_off);
}

PackArgs pack_args(const Geo &g, const uint16_t *x, const int32_t *idx, const int32_t *slot_map,
                   const int32_t *occ, uint16_t *pool_x, int32_t *pool_hdr, moe_pw_counters *ctr,
                   const EpRows *ep, uint32_t wave_mask)
{
    PackArgs p;
    p.x = x;
    p.idx = idx;
    p.slot_map = slot_map;
    p.occ = occ;
    p.pool_x = pool_x;
    p.pool_hdr = pool_hdr;
    p.ctr = ctr;
    p.T = g.T;
    p.n_slots = g.n_slots;
    p.n_pools = g.n_pools;
    p.C_s = g.C_s;
    p.k = g.k;
    p.D = g.D;
    p.rowbytes = uint32_t(g.D) * 2u;
    p.stages = 0;
    p.geo = g;
    p.wave_mask = wave_mask;
    if (ep) p.ep = *ep;
    else std::memset(&p.ep, 0, sizeof(p.ep));
    return p;
}

constexpr int MIN_STAGES = 4;

// Warps and stages per warp: as many rows as fit next to the zero row and
// `extra` bytes of other shared memory, MIN_STAGES .. MOE_PW_PACK_MAX_STAGES,
// dropping warps for very wide rows.  Returns false if even one warp's
// MIN_STAGES do not fit.
bool ring_shape(const DevInfo &di, uint32_t rowbytes, int max_warps, size_t extra, int *nw_out,
                int *stages_out)
{
    const size_t fixed = size_t(1024) + rowbytes + extra;
    if (size_t(di.smem_optin) < fixed) return false;
    const size_t budget = size_t(di.smem_optin) - fixed;
    int nw = max_warps;
    while (nw > 1 && budget / (size_t(nw) * rowbytes) < size_t(MIN_STAGES)) --nw;
    int stages = int(budget / (size_t(nw) * rowbytes));
    if (stages > MOE_PW_PACK_MAX_STAGES) stages = MOE_PW_PACK_MAX_STAGES;
    if (stages < MIN_STAGES) return false;
    *nw_out = nw;
    *stages_out = stages;
    return true;
}

}  // namespace

cudaError_t launch_pack(const Geo &g, const uint16_t *x, const int32_t *idx,
                        const int32_t *slot_map, const int32_t *occ, uint16_t *pool_x,
                        int32_t *pool_hdr, moe_pw_counters *ctr, cudaStream_t st,
                        const EpRows *ep, uint32_t wave_mask)
{
    if (g.T == 0 && g.n_pools == 0) return cudaSuccess;
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    PackArgs p = pack_args(g, x, idx, slot_map, occ, pool_x, pool_hdr, ctr, ep, wave_mask);
    int nw = 0, stages = 0;
    if (!ring_shape(di, p.rowbytes, MAX_PACK_WARPS, 0, &nw, &stages)) return cudaErrorInvalidValue;
    p.stages = stages;
    const size_t smem = pack_bar_bytes(nw, stages) + p.rowbytes + size_t(nw) * stages * p.rowbytes;
    // the deepest store lag (<= LAG) that leaves two stages for loads
    const int lag_cap = stages - 2 < LAG ? stages - 2 : LAG;
    return ep ? launch_ep<true>(p, di, g, nw, smem, lag_cap, st)
              : launch_ep<false>(p, di, g, nw, smem, lag_cap, st);
}

cudaError_t launch_pack_bucket(const Geo &g, const uint16_t *x, const int32_t *idx,
                               const int32_t *slot_map, const int32_t *occ, uint16_t *pool_x,
                               int32_t *pool_hdr, int32_t *recv_row, int32_t *bucket_slot,
                               int32_t *expert_counts, moe_pw_counters *ctr, cudaStream_t st)
{
    if (g.mode != MOE_PW_POOLED || g.ep_n != 1 || g.T == 0) return cudaErrorInvalidValue;
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    PackArgs p = pack_args(g, x, idx, slot_map, occ, pool_x, pool_hdr, ctr, nullptr, ~0u);
    const size_t bucket_bytes = (bucket_smem_bytes(BKF_THREADS, g.P) + 127) & ~size_t(127);
    int nw = 0, stages = 0;
    if (!ring_shape(di, p.rowbytes, 1, bucket_bytes, &nw, &stages)) return cudaErrorInvalidValue;
    p.stages = stages;
    const size_t pack_bytes = pack_bar_bytes(1, stages) + p.rowbytes + size_t(stages) * p.rowbytes;
    const uint32_t bucket_off = uint32_t((pack_bytes + 127) & ~size_t(127));
    const size_t smem = bucket_off + bucket_bytes;

    BucketArgs b;
    b.pool_hdr = pool_hdr;
    b.occ = occ;
    b.recv_row = recv_row;
    b.bucket_slot = bucket_slot;
    b.expert_counts = expert_counts;
    b.ctr = ctr;
    b.g = g;
    b.wave_mask = ~0u;
    b.hdr_out = pool_hdr;

    const int lag_cap = stages - 2 < LAG ? stages - 2 : LAG;
    if (lag_cap >= 12 && LAG >= 12) return launch_fused_lag<12>(p, b, bucket_off, di, g, smem, st);
    if (lag_cap >= 8) return launch_fused_lag<8>(p, b, bucket_off, di, g, smem, st);
    if (lag_cap >= 4) return launch_fused_lag<4>(p, b, bucket_off, di, g, smem, st);
    return launch_fused_lag<2>(p, b, bucket_off, di, g, smem, st);
}

}  // namespace moe_pw
