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
// The gradient needs f, which is fixed by the routing (the counts of idx),
// not by the probabilities, so the counts come first and one pass over the
// logits then gives both the probability sums and the gradient: the logits
// are read once.  Kernels, all deterministic (fixed summation orders,
// integer counts):
//   1. counts: block per (sequence, chunk of BAL_CHUNK tokens); the chunk's
//      ids counted in shared memory (atomics on integers: order does not
//      matter), then added to the sequence's counts in the workspace;
//   2. pass: block per (sequence, chunk); a warp per token (the next row
//      loaded while this one is reduced) computes the softmax (warp
//      reductions) and adds p into per-lane accumulators of the experts it
//      holds, tokens in order; the block sums its warps in order and writes
//      the chunk's partial sums.  With the gradient it also forms
//      dlogits = alpha / L * p * (f - dot), dot = sum_i f_i p_i by a fixed
//      xor tree, from its sequence's f (counts times E / (k L)), written or
//      added;
//   3. finish: block per sequence, a thread per expert; partial sums over
//      chunks in order, f, P and the loss (a fixed-order block reduction over
//      experts).
// HBM-bound (the logits in, dlogits out); no tensor cores.
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
    int32_t *cnt;     // [n_seq][E] assignment counts (zeroed before the counts pass)
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

// Token range of block (chunk c, sequence s).
__device__ __forceinline__ void chunk_tokens(const BalArgs &a, int64_t s, int64_t c, int64_t &t0,
                                             int64_t &t1)
{
    t0 = s * a.L + c * BAL_CHUNK;
    t1 = t0 + BAL_CHUNK;
    if (t1 > (s + 1) * a.L) t1 = (s + 1) * a.L;
}

__global__ void __launch_bounds__(BAL_THREADS) balance_counts(BalArgs a)
{
    extern __shared__ int32_t csm[];  // [E]
    const int64_t s = blockIdx.y;
    int64_t t0, t1;
    chunk_tokens(a, s, blockIdx.x, t0, t1);
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) csm[e] = 0;
    __syncthreads();
    for (int64_t i = t0 * a.k + threadIdx.x; i < t1 * a.k; i += blockDim.x) {
        const int32_t e = a.idx[i];
        if (e >= 0 && e < a.E) atomicAdd(&csm[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x)
        if (csm[e]) atomicAdd(&a.cnt[s * a.E + e], csm[e]);
}

// GRAD: also the gradient (launched as a programmatic dependent of the
// counts pass, whose counts it reads; without it, of nothing it reads).
template <int NV, bool GRAD>
__global__ void __launch_bounds__(BAL_THREADS) balance_pass(BalArgs a)
{
    extern __shared__ float bsm[];  // [BAL_WARPS][E] probabilities
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t s = blockIdx.y, c = blockIdx.x;
    int64_t t0, t1;
    chunk_tokens(a, s, c, t0, t1);
    const int E4 = a.E >> 2;
    griddep_wait();
    // the sequence's f, lane l holding the experts of its logits
    float fv[NV * 4];
    if (GRAD) {
        const float scale_f = float(a.E) / (float(a.k) * float(a.L));
        const int32_t *crow = a.cnt + s * a.E;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const int q = lane + 32 * v;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
                fv[4 * v + cc] = q < E4 ? float(crow[4 * q + cc]) * scale_f : 0.0f;
        }
    }
    const float g = a.alpha / float(a.L);
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
        if (GRAD) {
            float dot = 0.0f;
#pragma unroll
            for (int i = 0; i < NV * 4; ++i) dot = fmaf(fv[i], x[i], dot);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(FULL_MASK, dot, o);
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
    }
}

// 512 threads: one expert per thread for E <= 512, so that all of a thread's
// chunk loads are in flight together (with 256 threads the second expert's
// loads waited for the first's: the pass took ~23 us for 64 sequences).
constexpr int FIN_THREADS = 512;

// Launched as a programmatic dependent of the probability pass.
__global__ void __launch_bounds__(FIN_THREADS) balance_finish(BalArgs a)
{
    __shared__ float red[FIN_THREADS];
    const int64_t s = blockIdx.x;
    const float scale_f = float(a.E) / (float(a.k) * float(a.L));
    griddep_wait();
    float mine = 0.0f;  // this thread's experts e = tid, tid + 512, ... in order
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        float sum = 0.0f;
        // chunks in order; unrolled so the loads of 8 chunks are in flight together
#pragma unroll 8
        for (int c = 0; c < a.chunks; ++c) sum += __ldcg(a.part + (s * a.chunks + c) * a.E + e);
        const float P = sum / float(a.L);
        const float f = float(__ldcg(a.cnt + s * a.E + e)) * scale_f;
        a.P[s * a.E + e] = P;
        a.f[s * a.E + e] = f;
        mine = fmaf(f, P, mine);
    }
    red[threadIdx.x] = mine;
    __syncthreads();
    for (int h = FIN_THREADS / 2; h > 0; h >>= 1) {
        if (threadIdx.x < h) red[threadIdx.x] += red[threadIdx.x + h];
        __syncthreads();
    }
    if (threadIdx.x == 0) a.loss[s] = a.alpha * red[0];
}

template <int NV>
cudaError_t launch_nv(const BalArgs &a, int64_t n_seq, cudaStream_t st)
{
    cudaError_t err;
    if ((err = cudaMemsetAsync(a.cnt, 0, sizeof(int32_t) * size_t(n_seq) * a.E, st)) !=
        cudaSuccess)
        return err;
    const dim3 grid(unsigned(a.chunks), unsigned(n_seq));
    balance_counts<<<grid, BAL_THREADS, sizeof(int32_t) * a.E, st>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    // the probability pass and the finish start under their predecessor's
    // tail (programmatic dependent launches; each waits for it before
    // reading its outputs)
    const size_t smem = sizeof(float) * BAL_WARPS * a.E;
    auto pass = a.dlogits ? balance_pass<NV, true> : balance_pass<NV, false>;
    if (smem > 48 * 1024 &&
        (err = cudaFuncSetAttribute(pass, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    int(smem))) != cudaSuccess)
        return err;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.stream = st;
    cfg.gridDim = grid;
    cfg.blockDim = dim3(BAL_THREADS);
    cfg.dynamicSmemBytes = smem;
    if ((err = cudaLaunchKernelEx(&cfg, pass, a)) != cudaSuccess) return err;
    cfg.gridDim = dim3(unsigned(n_seq));
    cfg.blockDim = dim3(FIN_THREADS);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, balance_finish, a);
}

}  // namespace

int64_t balance_ws_bytes(int64_t T, int64_t L, int32_t E)
{
    if (L <= 0) return 0;
    const int64_t chunks = (L + BAL_CHUNK - 1) / BAL_CHUNK;
    const int64_t n = (T / L) * chunks * E;
    return align256(4 * n) + align256(4 * (T / L) * int64_t(E));
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
