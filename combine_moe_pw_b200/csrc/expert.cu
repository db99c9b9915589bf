// expert.cu - per-expert op and return layout.
//
// The pages' experts are trained networks; this stand-in scales each row by
// a per-expert factor, y = bf16_rn(s_e * x) with the product in fp32.  The
// return pools keep the dispatch pools' slot ids, the geometry the second
// all-to-all ("535B大模型“直播”训练三个月", MoE / token dropping section) would
// carry back.  Slots the receiver did not keep return zeros and header -1.
//
// Streaming kernel over slots: one warp per slot row, 16-byte loads and
// stores, four chunks in flight per lane.
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

}  // namespace

cudaError_t launch_expert(const Geo &g, const uint16_t *pool_x, const int32_t *pool_hdr,
                          const int32_t *recv_row, const float *scale, uint16_t *ret_x,
                          int32_t *ret_hdr, cudaStream_t st, const EpRows *ep,
                          uint32_t wave_mask)
{
    if (g.n_slots == 0) return cudaSuccess;
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    int64_t blocks = (g.n_slots + 7) / 8;
    if (blocks > int64_t(di.sms) * 8) blocks = int64_t(di.sms) * 8;
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
