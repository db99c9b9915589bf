// route.cu - top-k expert selection and softmax gates, one warp per token.
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 二: the router picks 8 of the
// 384 routed experts for every token.  The selection itself is in
// route_body.cuh.  The next token's row is loaded while the current one is
// being selected.
// The kernel is issue-bound (a few hundred warp instructions per token), so
// the common shapes are compiled with k = 8 and E = 128*NV fixed, and the
// grid is one wave of resident blocks at 64 registers (4 blocks per SM):
// on B200 that measured 17% faster than the same selection with run-time k
// and 60 registers over two waves.
#include "route_body.cuh"

namespace moe_pw {

namespace {

constexpr int ROUTE_WARPS = 8;
constexpr int ROUTE_MIN_BLOCKS = 4;  // caps registers at 64

// NV: float4s per lane; FULL: E == 128*NV (no bounds checks); KC: k fixed at
// compile time (0: run-time k).
template <int NV, bool FULL, int KC>
__global__ void __launch_bounds__(ROUTE_WARPS * 32, ROUTE_MIN_BLOCKS)
route_kernel(const float *__restrict__ logits, int32_t *__restrict__ idx,
             float *__restrict__ gates, int64_t T, int E, int k_rt)
{
    // per warp: candidate list and the selected compound keys in rank order
    __shared__ __align__(16) unsigned long long cand_sm[ROUTE_WARPS][32];
    __shared__ unsigned long long sel_sm[ROUTE_WARPS][32];
    __shared__ uint4 key_sm[ROUTE_WARPS][KeyRows<NV>::V][32];
    const int k = KC ? KC : k_rt;
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;
    const int E4 = E >> 2;

    auto one = [&](int64_t t, const float4 (&row)[NV]) {
        int32_t sel_idx;
        float ex, sum;
        route_select<NV, FULL, KC, ROUTE_WARPS>(row, k, E4, lane, wib, cand_sm, sel_sm, key_sm,
                                                sel_idx, ex, sum);
        if (lane < k) {
            idx[t * k + lane] = sel_idx;
            gates[t * k + lane] = ex / sum;
        }
    };
    float4 cur[NV], nxt[NV];
    if (warp < T) load_row<NV, FULL>(logits, warp, E4, lane, cur);
    for (int64_t t = warp; t < T; t += nwarp) {
        if (t + nwarp < T) load_row<NV, FULL>(logits, t + nwarp, E4, lane, nxt);
        one(t, cur);
#pragma unroll
        for (int v = 0; v < NV; ++v) cur[v] = nxt[v];
    }
}

template <int NV, bool FULL, int KC>
cudaError_t launch_nv(const Geo &g, const float *logits, int32_t *idx, float *gates,
                      cudaStream_t st)
{
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    // one wave of resident blocks; every warp strides over the tokens
    static const int per_sm = [] {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, route_kernel<NV, FULL, KC>,
                                                          ROUTE_WARPS * 32, 0) != cudaSuccess)
            cudaGetLastError();
        return n > 0 ? n : 1;
    }();
    int64_t blocks = (g.T + ROUTE_WARPS - 1) / ROUTE_WARPS;
    const int64_t cap = int64_t(di.sms) * per_sm;
    if (blocks > cap) blocks = cap;
    route_kernel<NV, FULL, KC>
        <<<unsigned(blocks), ROUTE_WARPS * 32, 0, st>>>(logits, idx, gates, g.T, g.E, g.k);
    return cudaGetLastError();
}

template <int NV>
cudaError_t launch_k(const Geo &g, const float *logits, int32_t *idx, float *gates,
                     cudaStream_t st)
{
    const bool full = g.E == 128 * NV;
    if (g.k == 8)
        return full ? launch_nv<NV, true, 8>(g, logits, idx, gates, st)
                    : launch_nv<NV, false, 8>(g, logits, idx, gates, st);
    return full ? launch_nv<NV, true, 0>(g, logits, idx, gates, st)
                : launch_nv<NV, false, 0>(g, logits, idx, gates, st);
}

}  // namespace

cudaError_t launch_route(const Geo &g, const float *logits, int32_t *idx, float *gates,
                         cudaStream_t st)
{
    if (g.T == 0) return cudaSuccess;
    const int E4 = g.E / 4;
    const int nv = (E4 + 31) / 32;
    switch (nv) {
    case 1: return launch_k<1>(g, logits, idx, gates, st);
    case 2: return launch_k<2>(g, logits, idx, gates, st);
    case 3: return launch_k<3>(g, logits, idx, gates, st);
    case 4: return launch_k<4>(g, logits, idx, gates, st);
    case 5: case 6: return launch_k<6>(g, logits, idx, gates, st);
    case 7: case 8: return launch_k<8>(g, logits, idx, gates, st);
    case 9: case 10: case 11: case 12: return launch_k<12>(g, logits, idx, gates, st);
    default: return launch_k<16>(g, logits, idx, gates, st);
    }
}

}  // namespace moe_pw
