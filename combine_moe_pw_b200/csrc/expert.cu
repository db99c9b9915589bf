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

__global__ void __launch_bounds__(256) expert_kernel(const uint4 *__restrict__ pool_x,
                                                     const int32_t *__restrict__ pool_hdr,
                                                     const int32_t *__restrict__ recv_row,
                                                     const float *__restrict__ scale,
                                                     uint4 *__restrict__ ret_x,
                                                     int32_t *__restrict__ ret_hdr,
                                                     int64_t n_slots, int cpr, int E)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;
    for (int64_t slot = warp; slot < n_slots; slot += nwarp) {
        const int32_t e = pool_hdr[slot];
        const bool keep = recv_row[slot] >= 0 && e >= 0 && e < E;
        const float s = keep ? scale[e] : 0.0f;
        const uint4 *src = pool_x + slot * cpr;
        uint4 *dst = ret_x + slot * cpr;
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
        } else {
            for (int c = lane; c < cpr; c += 32) __stcs(dst + c, make_uint4(0, 0, 0, 0));
        }
        if (lane == 0) ret_hdr[slot] = keep ? e : -1;
    }
}

}  // namespace

cudaError_t launch_expert(const Geo &g, const uint16_t *pool_x, const int32_t *pool_hdr,
                          const int32_t *recv_row, const float *scale, uint16_t *ret_x,
                          int32_t *ret_hdr, cudaStream_t st)
{
    if (g.n_slots == 0) return cudaSuccess;
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    int64_t blocks = (g.n_slots + 7) / 8;
    if (blocks > int64_t(di.sms) * 8) blocks = int64_t(di.sms) * 8;
    expert_kernel<<<unsigned(blocks), 256, 0, st>>>(
        reinterpret_cast<const uint4 *>(pool_x), pool_hdr, recv_row, scale,
        reinterpret_cast<uint4 *>(ret_x), ret_hdr, g.n_slots, g.D / 8, g.E);
    return cudaGetLastError();
}

}  // namespace moe_pw
