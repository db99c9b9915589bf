// balance.cu - sequence-level balancing: a per-sequence balance term of the
// training loss and its gradient with respect to the router logits.
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 四, names sequence-level
// balancing as the third remedy when drops stay high (one that may make the
// experts re-specialise during training); the pages give no formula.  This
// library's reading, per sequence s of L tokens:
//   p[t][e] = softmax over all E logits of token t
//   f[s][e] = E / (k L) * (assignments of s to expert e)      (1 at balance)
//   P[s][e] = (1 / L) * sum over t in s of p[t][e]
//   loss[s] = alpha * sum_e f[s][e] P[s][e]
//   dlogits[t][e] = alpha / L * p[t][e] * (f[s][e] - sum_i f[s][i] p[t][i])
// (the routing held fixed: top-k is piecewise constant in the logits).
//
// Three kernels, all deterministic (fixed summation orders, integer counts):
//   1. stats: block per (sequence, chunk of BAL_CHUNK tokens); a warp per
//      token (the next row loaded while this one is reduced) computes the
//      row's max and sum of exponentials (warp reductions) and adds p into
//      per-lane accumulators of the experts it holds, tokens in order; the
//      block sums its warps in order and writes the chunk's partial sums; the
//      chunk's expert counts come from shared-memory atomics on idx
//      (integers: order does not matter);
//   2. finish: block per sequence; partial sums over chunks in order, f, P and
//      the loss (a fixed-order block reduction over experts);
//   3. grad (optional): a warp per token (next row in flight), p again,
//      dot = sum_i f_i p_i by a fixed xor tree, dlogits written or added.
// Reads the logits once per pass (HBM-bound); no tensor cores.
#include "common.cuh"

namespace moe_pw {

namespace {

constexpr int BAL_THREADS = 256;
constexpr int BAL_WARPS = BAL_THREADS / 32;
constexpr int BAL_CHUNK = 128;  // tokens per stats block

struct BalArgs {
    const float *logits;
    const int32_t *idx;
    float *f, *P, *loss, *dlogits;
    float *part;      // [n_seq][chunks][E] partial probability sums
    int32_t *cnt;     // [n_seq][chunks][E] partial assignment counts
    int64_t T, L;
    int32_t E, k, chunks;
    float alpha;
    int32_t accumulate;
};

// Lane l holds experts 4 * (l + 32 v) + c, v < NV, c < 4 (as the router).
template <int NV>
__device__ __forceinline__ void load_row(const BalArgs &a, int64_t t, int lane, float (&x)[NV * 4])
{
    const float4 *row = reinterpret_cast<const float4 *>(a.logits + t * a.E);
    const int E4 = a.E >> 2;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
        const int q = lane + 32 * v;
        float4 f4 = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (q < E4) f4 = __ldcs(row + q);
        x[4 * v + 0] = f4.x;
        x[4 * v + 1] = f4.y;
        x[4 * v + 2] = f4.z;
        x[4 * v + 3] = f4.w;
    }
}

// p[i] = softmax of the row (absent experts: 0)
template <int NV>
__device__ __forceinline__ void softmax_row(float (&x)[NV * 4])
{
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < NV * 4; ++i) mx = fmaxf(mx, x[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL_MASK, mx, o));
    float sum = 0.0f;
#pragma unroll
    for (int i = 0; i < NV * 4; ++i) {
        x[i] = expf(x[i] - mx);  // exp(-inf) = 0 for absent experts
        sum += x[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(FULL_MASK, sum, o);
    // one IEEE division per lane, then products (within 2 ulp of x / sum):
    // the per-element divisions made the pass issue-bound
    const float inv = 1.0f / sum;
#pragma unroll
    for (int i = 0; i < NV * 4; ++i) x[i] = x[i] * inv;
}

template <int NV>
__global__ void __launch_bounds__(BAL_THREADS) balance_stats(BalArgs a)
{
    extern __shared__ float bsm[];  // [BAL_WARPS][E] probabilities, then [E] counts
    int32_t *csm = reinterpret_cast<int32_t *>(bsm + BAL_WARPS * a.E);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t s = blockIdx.y, c = blockIdx.x;
    const int64_t t0 = s * a.L + c * BAL_CHUNK;
    int64_t t1 = t0 + BAL_CHUNK;
    if (t1 > (s + 1) * a.L) t1 = (s + 1) * a.L;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) csm[e] = 0;
    __syncthreads();
    // counts of the chunk's assignments
    for (int64_t i = t0 * a.k + threadIdx.x; i < t1 * a.k; i += blockDim.x) {
        const int32_t e = a.idx[i];
        if (e >= 0 && e < a.E) atomicAdd(&csm[e], 1);
    }
    // probabilities: warp w takes tokens t0 + w, t0 + w + BAL_WARPS, ...
    float acc[NV * 4];
#pragma unroll
    for (int i = 0; i < NV * 4; ++i) acc[i] = 0.0f;
    // the next token's row is loaded while the current one is reduced
    float nx[NV * 4];
    if (t0 + warp < t1) load_row<NV>(a, t0 + warp, lane, nx);
    for (int64_t t = t0 + warp; t < t1; t += BAL_WARPS) {
        float x[NV * 4];
#pragma unroll
        for (int i = 0; i < NV * 4; ++i) x[i] = nx[i];
        if (t + BAL_WARPS < t1) load_row<NV>(a, t + BAL_WARPS, lane, nx);
        softmax_row<NV>(x);
#pragma unroll
        for (int i = 0; i < NV * 4; ++i) acc[i] += x[i];
    }
    const int E4 = a.E >> 2;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
        const int q = lane + 32 * v;
        if (q < E4)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) bsm[warp * a.E + 4 * q + cc] = acc[4 * v + cc];
    }
    __syncthreads();
    const int64_t base = (s * a.chunks + c) * a.E;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        float sum = 0.0f;
        for (int w = 0; w < BAL_WARPS; ++w) sum += bsm[w * a.E + e];
        a.part[base + e] = sum;
        a.cnt[base + e] = csm[e];
    }
}

__global__ void __launch_bounds__(BAL_THREADS) balance_finish(BalArgs a)
{
    __shared__ float red[BAL_THREADS];
    const int64_t s = blockIdx.x;
    const float scale_f = float(a.E) / (float(a.k) * float(a.L));
    float mine = 0.0f;  // this thread's experts e = tid, tid + 256, ... in order
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        float sum = 0.0f;
        int64_t n = 0;
        // chunks in order; unrolled so the loads of 8 chunks are in flight together
#pragma unroll 8
        for (int c = 0; c < a.chunks; ++c) {
            sum += __ldcg(a.part + (s * a.chunks + c) * a.E + e);
            n += __ldcg(a.cnt + (s * a.chunks + c) * a.E + e);
        }
        const float P = sum / float(a.L);
        const float f = float(n) * scale_f;
        a.P[s * a.E + e] = P;
        a.f[s * a.E + e] = f;
        mine = fmaf(f, P, mine);
    }
    red[threadIdx.x] = mine;
    __syncthreads();
    for (int h = BAL_THREADS / 2; h > 0; h >>= 1) {
        if (threadIdx.x < h) red[threadIdx.x] += red[threadIdx.x + h];
        __syncthreads();
    }
    if (threadIdx.x == 0) a.loss[s] = a.alpha * red[0];
}

template <int NV>
__global__ void __launch_bounds__(BAL_THREADS) balance_grad(BalArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;
    const int E4 = a.E >> 2;
    // the next token's logits and its sequence's f row are loaded while the
    // current token is worked on
    float nx[NV * 4], nf[NV * 4];
    auto load_f = [&](int64_t t, float (&fo)[NV * 4]) {
        const float4 *frow = reinterpret_cast<const float4 *>(a.f + (t / a.L) * a.E);
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const int q = lane + 32 * v;
            const float4 f4 = q < E4 ? __ldg(frow + q) : make_float4(0.f, 0.f, 0.f, 0.f);
            fo[4 * v + 0] = f4.x;
            fo[4 * v + 1] = f4.y;
            fo[4 * v + 2] = f4.z;
            fo[4 * v + 3] = f4.w;
        }
    };
    if (warp < a.T) {
        load_row<NV>(a, warp, lane, nx);
        load_f(warp, nf);
    }
    for (int64_t t = warp; t < a.T; t += nwarp) {
        float x[NV * 4], fv[NV * 4];
#pragma unroll
        for (int i = 0; i < NV * 4; ++i) {
            x[i] = nx[i];
            fv[i] = nf[i];
        }
        if (t + nwarp < a.T) {
            load_row<NV>(a, t + nwarp, lane, nx);
            load_f(t + nwarp, nf);
        }
        softmax_row<NV>(x);
        float dot = 0.0f;
#pragma unroll
        for (int i = 0; i < NV * 4; ++i) dot = fmaf(fv[i], x[i], dot);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(FULL_MASK, dot, o);
        const float g = a.alpha / float(a.L);
        float4 *row = reinterpret_cast<float4 *>(a.dlogits + t * a.E);
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const int q = lane + 32 * v;
            if (q >= E4) continue;
            float4 d;
            d.x = g * x[4 * v + 0] * (fv[4 * v + 0] - dot);
            d.y = g * x[4 * v + 1] * (fv[4 * v + 1] - dot);
            d.z = g * x[4 * v + 2] * (fv[4 * v + 2] - dot);
            d.w = g * x[4 * v + 3] * (fv[4 * v + 3] - dot);
            if (a.accumulate) {
                const float4 o = row[q];
                d.x += o.x;
                d.y += o.y;
                d.z += o.z;
                d.w += o.w;
            }
            row[q] = d;
        }
    }
}

template <int NV>
cudaError_t launch_nv(const BalArgs &a, int64_t n_seq, cudaStream_t st)
{
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    const size_t smem = sizeof(float) * BAL_WARPS * a.E + sizeof(int32_t) * a.E;
    cudaError_t err;
    if (smem > 48 * 1024 &&
        (err = cudaFuncSetAttribute(balance_stats<NV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    int(smem))) != cudaSuccess)
        return err;
    balance_stats<NV><<<dim3(unsigned(a.chunks), unsigned(n_seq)), BAL_THREADS, smem, st>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    balance_finish<<<unsigned(n_seq), BAL_THREADS, 0, st>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if (a.dlogits) {
        int64_t blocks = (a.T + BAL_WARPS - 1) / BAL_WARPS;
        if (blocks > int64_t(di.sms) * 8) blocks = int64_t(di.sms) * 8;
        balance_grad<NV><<<unsigned(blocks), BAL_THREADS, 0, st>>>(a);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace

int64_t balance_ws_bytes(int64_t T, int64_t L, int32_t E)
{
    if (L <= 0) return 0;
    const int64_t chunks = (L + BAL_CHUNK - 1) / BAL_CHUNK;
    const int64_t n = (T / L) * chunks * E;
    return align256(4 * n) + align256(4 * n);
}

cudaError_t launch_balance(const Geo &g, int64_t seq_len, float alpha, const float *logits,
                           const int32_t *idx, float *f, float *P, float *loss, float *dlogits,
                           int32_t accumulate, void *ws, cudaStream_t st)
{
    if (g.T == 0) return cudaSuccess;
    BalArgs a;
    a.logits = logits;
    a.idx = idx;
    a.f = f;
    a.P = P;
    a.loss = loss;
    a.dlogits = dlogits;
    a.T = g.T;
    a.L = seq_len;
    a.E = g.E;
    a.k = g.k;
    a.chunks = int32_t((seq_len + BAL_CHUNK - 1) / BAL_CHUNK);
    a.alpha = alpha;
    a.accumulate = accumulate;
    const int64_t n_seq = g.T / seq_len;
    const int64_t n = n_seq * a.chunks * g.E;
    a.part = static_cast<float *>(ws);
    a.cnt = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + align256(4 * n));
    const int E4 = g.E / 4;
    const int nv = (E4 + 31) / 32;
    switch (nv) {
    case 1: return launch_nv<1>(a, n_seq, st);
    case 2: return launch_nv<2>(a, n_seq, st);
    case 3: return launch_nv<3>(a, n_seq, st);
    case 4: return launch_nv<4>(a, n_seq, st);
    case 5: case 6: return launch_nv<6>(a, n_seq, st);
    case 7: case 8: return launch_nv<8>(a, n_seq, st);
    case 9: case 10: case 11: case 12: return launch_nv<12>(a, n_seq, st);
    default: return launch_nv<16>(a, n_seq, st);
    }
}

}  // namespace moe_pw
