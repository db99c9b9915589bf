// backward.cu - gradients of the combine and of the pack.
//
// The pages train this model ("Marin 开始公开训练 535B 参数 MoE 模型", section 一)
// but describe no backward; these kernels differentiate this library's own
// forward definitions.  Given dout = dL/dout [T, D] fp32:
//   combine backward, per surviving (t, j) (slot >= 0, ret_hdr[slot] >= 0):
//     d_ret[slot]   = bf16_rn(g_j * dout[t])         (fp32 product)
//     dgate[t][j]   = <dout[t], y_j>                 (fp32, fixed reduction order)
//   every other slot of the gradient pool is zero;
//   softmax over the k chosen logits:
//     dlogits[t][idx[t][j]] = g_j * (dgate_j - sum_i g_i dgate_i), others 0.
//   The stand-in expert op's backward is the same scale op on the gradient
//   pool (moe_pw_expert), and the pack's backward, dx[t] = sum over the
//   surviving j of d_pool[slot], is the combine kernel with unit gates.
//
// combine_bwd_kernel: one warp per token; lanes j < k read (slot, gate,
// ret_hdr) once and the warp broadcasts them; each lane owns 16-byte chunks
// of bf16 rows (and the matching 32 bytes of dout), two chunks per
// iteration with all their loads issued first, accumulates its share of
// every dot product with fmaf in chunk order, writes the gradient rows, and
// the warp reduces the dots with a fixed xor-butterfly.
#include <cuda_bf16.h>

#include "common.cuh"

namespace moe_pw {

namespace {

constexpr int BU = 2;  // chunks per lane per iteration (their loads are in flight together)

// two fp32 -> packed bf16 pair, round to nearest even (lo in the low half)
__device__ __forceinline__ uint32_t bf16x2_of(float lo, float hi)
{
    const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&r);
}

template <int KMAX>
__global__ void __launch_bounds__(256) combine_bwd_kernel(
    const float4 *__restrict__ dout, const uint4 *__restrict__ ret_x,
    const int32_t *__restrict__ ret_hdr, const int32_t *__restrict__ slot_map,
    const int32_t *__restrict__ idx, const float *__restrict__ gates, uint4 *__restrict__ d_ret,
    float *__restrict__ dgates, float *__restrict__ dlogits, int64_t T, int k, int cpr, int E,
    int64_t n_slots, moe_pw_counters *ctr)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;
    for (int64_t t = warp; t < T; t += nwarp) {
        int32_t my_slot = -1, my_e = 0;
        float my_gate = 0.0f;
        if (lane < k) {
            my_slot = slot_map[t * k + lane];
            my_gate = gates[t * k + lane];
            my_e = idx[t * k + lane];
            if (my_slot >= n_slots) {
                set_error(ctr, MOE_PW_DEVERR_SLOT);
                my_slot = -1;
            }
            if (my_slot >= 0 && ret_hdr[my_slot] < 0) my_slot = -1;
        }
        int32_t slot[KMAX];
        float gv[KMAX], dot[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            slot[j] = __shfl_sync(FULL_MASK, my_slot, j);
            gv[j] = __shfl_sync(FULL_MASK, my_gate, j);
            dot[j] = 0.0f;
        }
        const float4 *drow = dout + t * (2 * int64_t(cpr));
        for (int c0 = lane; c0 < cpr; c0 += 32 * BU) {
            float4 d0[BU], d1[BU];
#pragma unroll
            for (int u = 0; u < BU; ++u)
                if (c0 + 32 * u < cpr) {
                    d0[u] = __ldcs(drow + 2 * (c0 + 32 * u));
                    d1[u] = __ldcs(drow + 2 * (c0 + 32 * u) + 1);
                }
            // rows in groups of eight: the loads of a group, then its arithmetic.
            // The gathered rows take the read-only path with the default cache
            // policy, as in the forward combine (measured ~1.5% faster than
            // evict-first streaming loads)
#pragma unroll
            for (int jg = 0; jg < KMAX; jg += 8) {
                uint4 y[8][BU];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int j = jg + jj;
                    if (j < k && slot[j] >= 0)
#pragma unroll
                        for (int u = 0; u < BU; ++u)
                            if (c0 + 32 * u < cpr)
                                y[jj][u] = __ldg(ret_x + int64_t(slot[j]) * cpr + c0 + 32 * u);
                }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int j = jg + jj;
                    if (!(j < k && slot[j] >= 0)) continue;
                    const float g = gv[j];
#pragma unroll
                    for (int u = 0; u < BU; ++u) {
                        if (c0 + 32 * u >= cpr) continue;
                        float a = dot[j];
                        a = fmaf(d0[u].x, __uint_as_float(y[jj][u].x << 16), a);
                        a = fmaf(d0[u].y, __uint_as_float(y[jj][u].x & 0xFFFF0000u), a);
                        a = fmaf(d0[u].z, __uint_as_float(y[jj][u].y << 16), a);
                        a = fmaf(d0[u].w, __uint_as_float(y[jj][u].y & 0xFFFF0000u), a);
                        a = fmaf(d1[u].x, __uint_as_float(y[jj][u].z << 16), a);
                        a = fmaf(d1[u].y, __uint_as_float(y[jj][u].z & 0xFFFF0000u), a);
                        a = fmaf(d1[u].z, __uint_as_float(y[jj][u].w << 16), a);
                        a = fmaf(d1[u].w, __uint_as_float(y[jj][u].w & 0xFFFF0000u), a);
                        dot[j] = a;
                        uint4 gr;
                        gr.x = bf16x2_of(__fmul_rn(g, d0[u].x), __fmul_rn(g, d0[u].y));
                        gr.y = bf16x2_of(__fmul_rn(g, d0[u].z), __fmul_rn(g, d0[u].w));
                        gr.z = bf16x2_of(__fmul_rn(g, d1[u].x), __fmul_rn(g, d1[u].y));
                        gr.w = bf16x2_of(__fmul_rn(g, d1[u].z), __fmul_rn(g, d1[u].w));
                        __stcs(d_ret + int64_t(slot[j]) * cpr + c0 + 32 * u, gr);
                    }
                }
            }
        }
        // fixed butterfly: every lane ends with the same sums
        float my_dg = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            float v = dot[j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL_MASK, v, o);
            if (lane == j) my_dg = (j < k && slot[j] >= 0) ? v : 0.0f;
        }
        // softmax backward over the k chosen logits, weighted sum in j order
        float weighted = 0.0f;
        for (int j = 0; j < k; ++j)
            weighted = fmaf(__shfl_sync(FULL_MASK, my_gate, j), __shfl_sync(FULL_MASK, my_dg, j),
                            weighted);
        if (dgates && lane < k) dgates[t * k + lane] = my_dg;
        if (dlogits) {
            float *lrow = dlogits + t * int64_t(E);
            for (int q = lane; q < E; q += 32) lrow[q] = 0.0f;
            __syncwarp();
            if (lane < k) {
                if (my_e >= 0 && my_e < E)
                    lrow[my_e] = my_gate * (my_dg - weighted);
                else
                    set_error(ctr, MOE_PW_DEVERR_EXPERT_ID);
            }
        }
    }
}

// Zero the gradient rows of slots without a surviving assignment (hdr < 0).
__global__ void __launch_bounds__(256) zero_dead_rows_kernel(uint4 *__restrict__ rows,
                                                             const int32_t *__restrict__ hdr,
                                                             int64_t n_slots, int cpr)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;
    for (int64_t slot = warp; slot < n_slots; slot += nwarp) {
        if (hdr[slot] >= 0) continue;
        uint4 *r = rows + slot * cpr;
        for (int c = lane; c < cpr; c += 32) __stcs(r + c, make_uint4(0, 0, 0, 0));
    }
}

template <int KMAX>
cudaError_t launch_bwd(const Geo &g, const float *dout, const uint16_t *ret_x,
                       const int32_t *ret_hdr, const int32_t *slot_map, const int32_t *idx,
                       const float *gates, uint16_t *d_ret, float *dgates, float *dlogits,
                       moe_pw_counters *ctr, cudaStream_t st)
{
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    if (g.n_slots > 0) {
        int64_t zb = (g.n_slots + 7) / 8;
        if (zb > int64_t(di.sms) * 8) zb = int64_t(di.sms) * 8;
        zero_dead_rows_kernel<<<unsigned(zb), 256, 0, st>>>(reinterpret_cast<uint4 *>(d_ret),
                                                           ret_hdr, g.n_slots, g.D / 8);
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    if (g.T == 0) return cudaSuccess;
    int64_t blocks = (g.T + 7) / 8;
    if (blocks > int64_t(di.sms) * 8) blocks = int64_t(di.sms) * 8;
    combine_bwd_kernel<KMAX><<<unsigned(blocks), 256, 0, st>>>(
        reinterpret_cast<const float4 *>(dout), reinterpret_cast<const uint4 *>(ret_x), ret_hdr,
        slot_map, idx, gates, reinterpret_cast<uint4 *>(d_ret), dgates, dlogits, g.T, g.k,
        g.D / 8, g.E, g.n_slots, ctr);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine_backward(const Geo &g, const float *dout, const uint16_t *ret_x,
                                    const int32_t *ret_hdr, const int32_t *slot_map,
                                    const int32_t *idx, const float *gates, uint16_t *d_ret,
                                    float *dgates, float *dlogits, moe_pw_counters *ctr,
                                    cudaStream_t st)
{
    if (g.k <= 8)
        return launch_bwd<8>(g, dout, ret_x, ret_hdr, slot_map, idx, gates, d_ret, dgates,
                             dlogits, ctr, st);
    if (g.k <= 16)
        return launch_bwd<16>(g, dout, ret_x, ret_hdr, slot_map, idx, gates, d_ret, dgates,
                              dlogits, ctr, st);
    return launch_bwd<32>(g, dout, ret_x, ret_hdr, slot_map, idx, gates, d_ret, dgates, dlogits,
                          ctr, st);
}

}  // namespace moe_pw
