// route.cu - top-k expert selection and softmax gates, one warp per token.
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 二: the router picks 8 of the
// 384 routed experts for every token.  Order (logit descending, expert id
// ascending) and softmax gates over the chosen logits are this library's
// reading.
//
// Layout: lane l holds float4 number l + 32*v of the row (v < NV), i.e. the
// logits of experts 4*(l + 32*v) + c.  Each logit becomes an order-preserving
// unsigned key (0 marks "taken or absent").  A selection round is one
// warp-wide max of the keys (redux.sync) followed by a warp-wide min of the
// expert ids holding that key, which settles ties toward the lower id.  The
// next token's row is loaded while the current one is being selected.
#include "common.cuh"

namespace moe_pw {

namespace {

// Order-preserving map float -> uint32 (-0.0 folded onto +0.0).  Finite
// floats map to keys >= 0x007FFFFF, so 0 never collides with a logit.
__device__ __forceinline__ uint32_t order_key(float f)
{
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t key)
{
    uint32_t u = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
    return __uint_as_float(u);
}

template <int NV>
__device__ __forceinline__ void load_row(const float *__restrict__ logits, int64_t t, int E4,
                                         int lane, float4 (&f)[NV])
{
    const float4 *row = reinterpret_cast<const float4 *>(logits) + t * E4;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
        const int q = lane + 32 * v;
        if (q < E4) f[v] = __ldcs(row + q);
    }
}

template <int NV>
__global__ void __launch_bounds__(256) route_kernel(const float *__restrict__ logits,
                                                    int32_t *__restrict__ idx,
                                                    float *__restrict__ gates, int64_t T,
                                                    int E, int k)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;
    const int E4 = E >> 2;
    const int base = 4 * lane;  // expert id of key[v][0] is base + 128*v

    float4 cur[NV], nxt[NV];
    if (warp < T) load_row<NV>(logits, warp, E4, lane, cur);

    for (int64_t t = warp; t < T; t += nwarp) {
        if (t + nwarp < T) load_row<NV>(logits, t + nwarp, E4, lane, nxt);

        uint32_t key[NV][4];
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const bool in = lane + 32 * v < E4;
            key[v][0] = in ? order_key(cur[v].x) : 0u;
            key[v][1] = in ? order_key(cur[v].y) : 0u;
            key[v][2] = in ? order_key(cur[v].z) : 0u;
            key[v][3] = in ? order_key(cur[v].w) : 0u;
        }

        uint32_t sel_key = 0;
        int32_t sel_idx = 0;
        for (int j = 0; j < k; ++j) {
            uint32_t lm = 0;
#pragma unroll
            for (int v = 0; v < NV; ++v)
#pragma unroll
                for (int c = 0; c < 4; ++c) lm = max(lm, key[v][c]);
            const uint32_t m = __reduce_max_sync(FULL_MASK, lm);
            // lowest expert id in this lane whose key equals the maximum
            int32_t cand = 0x7FFFFFFF;
#pragma unroll
            for (int v = NV - 1; v >= 0; --v)
#pragma unroll
                for (int c = 3; c >= 0; --c)
                    if (key[v][c] == m) cand = base + 128 * v + c;
            const int32_t gi = __reduce_min_sync(FULL_MASK, cand);
            const int32_t rel = gi - base;  // equals 128*v + c only in the owning lane
#pragma unroll
            for (int v = 0; v < NV; ++v)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (rel == 128 * v + c) key[v][c] = 0u;
            if (lane == j) {
                sel_key = m;
                sel_idx = gi;
            }
        }

        // softmax over the chosen logits: lane j holds choice j
        const float val = key_value(sel_key);
        const float top = __shfl_sync(FULL_MASK, val, 0);
        const float ex = (lane < k) ? expf(val - top) : 0.0f;
        float sum = 0.0f;
        for (int j = 0; j < k; ++j) sum += __shfl_sync(FULL_MASK, ex, j);
        if (lane < k) {
            idx[t * k + lane] = sel_idx;
            gates[t * k + lane] = ex / sum;
        }
#pragma unroll
        for (int v = 0; v < NV; ++v) cur[v] = nxt[v];
    }
}

template <int NV>
cudaError_t launch_nv(const Geo &g, const float *logits, int32_t *idx, float *gates,
                      cudaStream_t st)
{
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    const int64_t warps_needed = g.T;
    int64_t blocks = (warps_needed + 7) / 8;
    const int64_t cap = int64_t(di.sms) * 8;  // 64 resident warps per SM
    if (blocks > cap) blocks = cap;
    route_kernel<NV><<<unsigned(blocks), 256, 0, st>>>(logits, idx, gates, g.T, g.E, g.k);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const Geo &g, const float *logits, int32_t *idx, float *gates,
                         cudaStream_t st)
{
    if (g.T == 0) return cudaSuccess;
    const int E4 = g.E / 4;
    const int nv = (E4 + 31) / 32;
    switch (nv) {
    case 1: return launch_nv<1>(g, logits, idx, gates, st);
    case 2: return launch_nv<2>(g, logits, idx, gates, st);
    case 3: return launch_nv<3>(g, logits, idx, gates, st);
    case 4: return launch_nv<4>(g, logits, idx, gates, st);
    case 5: case 6: return launch_nv<6>(g, logits, idx, gates, st);
    case 7: case 8: return launch_nv<8>(g, logits, idx, gates, st);
    case 9: case 10: case 11: case 12: return launch_nv<12>(g, logits, idx, gates, st);
    default: return launch_nv<16>(g, logits, idx, gates, st);
    }
}

}  // namespace moe_pw
