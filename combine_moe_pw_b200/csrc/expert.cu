// expert.cu - per-expert op and return layout.
//
// The pages' experts are trained networks; this stand-in scales each row by
// a per-expert factor, y = bf16_rn(s_e * x) with the product in fp32.  The
// return pools keep the dispatch pools' slot ids, the geometry the second
// all-to-all ("535B大模型“直播”训练三个月", MoE / token dropping section) would
// carry back.  Slots the receiver did not keep return zeros and header -1.
//
// Two kernels.  expert_ring_kernel (one GPU, rows up to what a block's
// shared memory holds) streams the rows through shared memory with bulk
// copies: persistent, RING_WARPS warps per block; warp w walks slots
// w, w + GW, ... (GW warps in the grid) through a ring of RING_NS row
// buffers.  Lane 0 loads the kept rows of the next slots ahead
// (cp.async.bulk, evict-first), the lanes scale the current row in place,
// and lane 0 writes it back with one bulk store; a slot the receiver did not
// keep gets one bulk store from a zero row.  A row buffer is reloaded once
// the bulk store of its previous row has read it.  Measured on the
// 262,144-token rack batch (14.2 GB of return rows written, 9.1 GB of kept
// rows read): 3.59-3.63 ms, against 3.89 ms for expert_kernel's 16-byte
// loads and stores.  expert_kernel (expert-parallel runs, whose results go to peer
// GPUs, and wider rows): one warp per slot row, 16-byte loads and stores,
// four chunks in flight per lane.
#include <cuda_bf16.h>

#include <cstring>

#include "common.cuh"

namespace moe_pw {

namespace {

__device__ __forceinline__ uint32_t scale_pair(uint32_t packed, float s)
{
    const float lo = __uint_as_float(packed << 16);
    const float hi = __uint_as_float(packed & 0xFFFF0000u);
    const __nv_bfloat162 r = __floats2bfloat162_rn(__fmul_rn(s, lo), __fmul_rn(s, hi));
    return *reinterpret_cast<const uint32_t *>(&r);
}

// Where the result of slot `slot` goes: the same slot of the local return
// pool, or (expert-parallel runs) the source's send slot in the return pool of
// the source's GPU.
struct ExpertArgs {
    const uint4 *pool_x;
    const int32_t *pool_hdr;
    const int32_t *recv_row;
    const float *scale;
    uint4 *ret_x;
    int32_t *ret_hdr;
    int64_t n_slots;
    int cpr;
    int E;
    uint32_t wave_mask;
    Geo geo;
    EpRows ep;
    moe_pw_counters *ctr;  // expert_ring_kernel: MOE_PW_DEVERR_TIMEOUT
};

template <bool EP>
__global__ void __launch_bounds__(256) expert_kernel(ExpertArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;
    const int cpr = a.cpr;
    // one wave only (expert-parallel runs overlap the waves): walk just that
    // wave's slots, every W-th run of C_s slots of the receive pool
    const int one_wave = EP && __popc(a.wave_mask) == 1 ? __ffs(a.wave_mask) - 1 : -1;
    const int64_t n_walk = one_wave >= 0 ? a.n_slots / a.geo.W : a.n_slots;
    for (int64_t i = warp; i < n_walk; i += nwarp) {
        int64_t slot = i;
        if (one_wave >= 0) {
            const int64_t run = i / a.geo.C_s;
            slot = (run * a.geo.W + one_wave) * a.geo.C_s + (i - run * a.geo.C_s);
        }
        uint4 *dst;
        int32_t *dst_hdr;
        if (EP) {
            int h, w;
            const uint32_t q = ep_recv_to_send(a.geo, uint32_t(slot), h, w);
            if (!((a.wave_mask >> w) & 1u)) continue;
            dst = reinterpret_cast<uint4 *>(a.ep.x[h]) + int64_t(q) * cpr;
            dst_hdr = a.ep.hdr[h] + q;
        } else {
            dst = a.ret_x + slot * cpr;
            dst_hdr = a.ret_hdr + slot;
        }
        const int32_t e = a.pool_hdr[slot];
        const bool keep = a.recv_row[slot] >= 0 && e >= 0 && e < a.E;
        const float s = keep ? a.scale[e] : 0.0f;
        const uint4 *src = a.pool_x + slot * cpr;
        if (keep) {
            int c = lane;
            for (; c + 96 < cpr; c += 128) {
                uint4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) v[u] = __ldcs(src + c + 32 * u);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint4 y;
                    y.x = scale_pair(v[u].x, s);
                    y.y = scale_pair(v[u].y, s);
                    y.z = scale_pair(v[u].z, s);
                    y.w = scale_pair(v[u].w, s);
                    __stcs(dst + c + 32 * u, y);
                }
            }
            for (; c < cpr; c += 32) {
                const uint4 v = __ldcs(src + c);
                uint4 y;
                y.x = scale_pair(v.x, s);
                y.y = scale_pair(v.y, s);
                y.z = scale_pair(v.z, s);
                y.w = scale_pair(v.w, s);
                __stcs(dst + c, y);
            }
        } else if (!EP) {
            // (across GPUs the header -1 alone goes back: nothing reads the row)
            for (int c = lane; c < cpr; c += 32) __stcs(dst + c, make_uint4(0, 0, 0, 0));
        }
        if (lane == 0) *dst_hdr = keep ? e : -1;
    }
    if (EP) __threadfence_system();  // peer stores ordered before any later signal
}

constexpr int RING_WARPS = 4, RING_NS = 3;
constexpr uint32_t RING_WAIT_LIMIT = 1u << 22;
// barriers [RING_WARPS][RING_NS] in the first 128 bytes, a zero row, then
// each warp's RING_NS row buffers
constexpr size_t RING_BAR_BYTES = 128;
static_assert(RING_WARPS * RING_NS * 8 <= RING_BAR_BYTES, "barrier region");

inline size_t ring_smem_bytes(int cpr)
{
    return RING_BAR_BYTES + size_t(cpr) * 16 * (1 + RING_WARPS * RING_NS);
}

__device__ __forceinline__ bool keeps_slot(const ExpertArgs &a, int64_t slot, int32_t &e)
{
    e = a.pool_hdr[slot];
    return a.recv_row[slot] >= 0 && e >= 0 && e < a.E;
}

__global__ void __launch_bounds__(RING_WARPS * 32) expert_ring_kernel(ExpertArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int cpr = a.cpr;
    const uint32_t rb = uint32_t(cpr) * 16u;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem) + wib * RING_NS;
    unsigned char *zero = smem + RING_BAR_BYTES;
    unsigned char *ring = zero + rb + size_t(wib) * RING_NS * rb;
    for (int c = threadIdx.x; c < cpr; c += blockDim.x)
        reinterpret_cast<uint4 *>(zero)[c] = make_uint4(0, 0, 0, 0);
    if (lane == 0)
        for (int s = 0; s < RING_NS; ++s) mbar_init(&bar[s], 1);
    fence_init_and_proxy();
    __syncthreads();

    const int64_t gw = int64_t(blockIdx.x) * RING_WARPS + wib;
    const int64_t GW = int64_t(gridDim.x) * RING_WARPS;
    const int64_t n = a.n_slots;
    const uint64_t pol = policy_evict_first();
    // step i of this warp is slot gw + i * GW; a kept row uses stage i % RING_NS
    uint32_t armed = 0;  // lane 0: stages with a load in flight
    auto issue = [&](int64_t i) {
        const int64_t slot = gw + i * GW;
        int32_t e;
        if (slot >= n || !keeps_slot(a, slot, e)) return;
        const int s = int(i % RING_NS);
        mbar_arrive_expect_tx(&bar[s], rb);
        bulk_g2s(ring + size_t(s) * rb, a.pool_x + slot * cpr, rb, &bar[s], pol);
        armed |= 1u << s;
    };
    if (lane == 0)
        for (int i = 0; i < RING_NS; ++i) issue(i);

    uint32_t phase = 0;  // parity of each stage's next load completion
    bool ok = true;
    int64_t i = 0;
    for (int64_t slot = gw; slot < n; slot += GW, ++i) {
        const int s = int(i % RING_NS);
        int32_t e;
        const bool keep = keeps_slot(a, slot, e);
        uint4 *dst = a.ret_x + slot * cpr;
        if (keep) {
            const bool landed = mbar_wait_bounded(&bar[s], (phase >> s) & 1u, RING_WAIT_LIMIT);
            if (!__all_sync(FULL_MASK, landed)) {
                ok = false;
                break;
            }
            phase ^= 1u << s;
            armed &= ~(1u << s);
            const float sc = a.scale[e];
            uint4 *row = reinterpret_cast<uint4 *>(ring + size_t(s) * rb);
            for (int c = lane; c < cpr; c += 32) {
                const uint4 v = row[c];
                uint4 y;
                y.x = scale_pair(v.x, sc);
                y.y = scale_pair(v.y, sc);
                y.z = scale_pair(v.z, sc);
                y.w = scale_pair(v.w, sc);
                row[c] = y;
            }
            // the lanes' writes, then the bulk store that reads them
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) bulk_s2g(dst, row, rb, pol);
        } else if (lane == 0) {
            bulk_s2g(dst, zero, rb, pol);
        }
        if (lane == 0) {
            a.ret_hdr[slot] = keep ? e : -1;
            bulk_commit();
            // the previous step's row has been read out of its stage: load
            // the row RING_NS steps after it there
            if (i > 0) {
                bulk_wait_read<1>();
                issue(i - 1 + RING_NS);
            }
        }
        __syncwarp();
    }
    if (lane == 0) {
        if (!ok) {
            set_error(a.ctr, MOE_PW_DEVERR_TIMEOUT);
            // loads still in flight write this CTA's shared memory: wait for
            // each (bounded) before the CTA retires
            for (int s = 0; s < RING_NS; ++s)
                if ((armed >> s) & 1u)
                    mbar_wait_bounded(&bar[s], (phase >> s) & 1u, RING_WAIT_LIMIT);
        }
        bulk_wait_all();
    }
}

}  // namespace

cudaError_t launch_expert(const Geo &g, const uint16_t *pool_x, const int32_t *pool_hdr,
                          const int32_t *recv_row, const float *scale, uint16_t *ret_x,
                          int32_t *ret_hdr, moe_pw_counters *ctr, cudaStream_t st,
                          const EpRows *ep, uint32_t wave_mask)
{
    if (g.n_slots == 0) return cudaSuccess;
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    ExpertArgs a;
    a.pool_x = reinterpret_cast<const uint4 *>(pool_x);
    a.pool_hdr = pool_hdr;
    a.recv_row = recv_row;
    a.scale = scale;
    a.ret_x = reinterpret_cast<uint4 *>(ret_x);
    a.ret_hdr = ret_hdr;
    a.n_slots = g.n_slots;
    a.cpr = g.D / 8;
    a.E = g.E;
    a.wave_mask = wave_mask;
    a.geo = g;
    a.ctr = ctr;
    const size_t ring_smem = ring_smem_bytes(a.cpr);
    if (!ep && ctr && ring_smem <= size_t(di.smem_optin)) {
        std::memset(&a.ep, 0, sizeof(a.ep));
        cudaError_t err = cudaFuncSetAttribute(
            expert_ring_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(ring_smem));
        if (err != cudaSuccess) return err;
        int per_sm = 0;
        err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, expert_ring_kernel,
                                                            RING_WARPS * 32, ring_smem);
        if (err != cudaSuccess) return err;
        // On 6 KB rows, 2 blocks per SM measured best (96 KB of loads
        // ahead per SM; 3 stages per warp beat 2 and 4, and one block of 6
        // stages was slower still).  Narrower rows take more blocks, for
        // about the same bytes ahead, as far as they fit.
        const size_t ahead = size_t(RING_WARPS) * (RING_NS - 1) * a.cpr * 16;
        const int want = int((98304 + ahead - 1) / ahead);
        if (per_sm > want) per_sm = want;
        if (per_sm < 1) per_sm = 1;
        int64_t blocks = int64_t(di.sms) * per_sm;
        const int64_t need = (g.n_slots + RING_WARPS - 1) / RING_WARPS;
        if (blocks > need) blocks = need;
        expert_ring_kernel<<<unsigned(blocks), RING_WARPS * 32, ring_smem, st>>>(a);
        return cudaGetLastError();
    }
    int64_t blocks = (g.n_slots + 7) / 8;
    if (blocks > int64_t(di.sms) * 8) blocks = int64_t(di.sms) * 8;
    if (ep) {
        a.ep = *ep;
        expert_kernel<true><<<unsigned(blocks), 256, 0, st>>>(a);
    } else {
        std::memset(&a.ep, 0, sizeof(a.ep));
        expert_kernel<false><<<unsigned(blocks), 256, 0, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace moe_pw
