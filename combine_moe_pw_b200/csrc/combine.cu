// combine.cu - gate-weighted combine back to token order.
//
// out[t] = sum over j of g_j * y_j, y_j the returned row of assignment (t, j),
// in fp32, j ascending, one fmaf per term from +0.  Terms of assignments that
// were dropped (no slot, or ret_hdr -1) are absent and the surviving gates are
// not renormalised: "Marin 开始公开训练 535B 参数 MoE 模型", section 四 -- a
// dropped assignment leaves the token to the shared experts.
//
// With gates == nullptr every gate is 1: fmaf(1, y, acc) is the exact sum,
// which makes the same kernel the pack's backward (dx = sum of the slots'
// gradient rows).
//
// One warp per token.  Lanes j < k read (slot, gate, ret_hdr) once and the
// warp broadcasts them into registers; then each lane owns 16-byte chunks of
// the row (8 bf16), issues the loads of all k rows for two chunks before
// accumulating, and writes 2 x 16 bytes of fp32 per chunk.  Skipped terms are
// warp-uniform branches.  The row loads go through the read-only data path
// with the default cache policy: on B200 that measured 4% faster than
// evict-first streaming loads (rack batch 1.77 against 1.85 ms; dropless
// 2.37 against 2.47 ms), the output stores stream (evict-first).
#include <cuda_bf16.h>

#include "common.cuh"

namespace moe_pw {

namespace {

#ifndef MOE_PW_COMBINE_U
#define MOE_PW_COMBINE_U 2
#endif
#ifndef MOE_PW_COMBINE_MINB
#define MOE_PW_COMBINE_MINB 0  // 0: let the compiler pick the register budget
#endif
#ifndef MOE_PW_COMBINE_BLOCKS_PER_SM
#define MOE_PW_COMBINE_BLOCKS_PER_SM 8
#endif
#if MOE_PW_COMBINE_MINB > 0
#define MOE_PW_COMBINE_BOUNDS __launch_bounds__(256, MOE_PW_COMBINE_MINB)
#else
#define MOE_PW_COMBINE_BOUNDS __launch_bounds__(256)
#endif
constexpr int U = MOE_PW_COMBINE_U;  // chunks per lane per iteration

__device__ __forceinline__ void fma_row(float (&acc)[8], float gj, const uint4 &v)
{
    acc[0] = fmaf(gj, __uint_as_float(v.x << 16), acc[0]);
    acc[1] = fmaf(gj, __uint_as_float(v.x & 0xFFFF0000u), acc[1]);
    acc[2] = fmaf(gj, __uint_as_float(v.y << 16), acc[2]);
    acc[3] = fmaf(gj, __uint_as_float(v.y & 0xFFFF0000u), acc[3]);
    acc[4] = fmaf(gj, __uint_as_float(v.z << 16), acc[4]);
    acc[5] = fmaf(gj, __uint_as_float(v.z & 0xFFFF0000u), acc[5]);
    acc[6] = fmaf(gj, __uint_as_float(v.w << 16), acc[6]);
    acc[7] = fmaf(gj, __uint_as_float(v.w & 0xFFFF0000u), acc[7]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&r);
}

// OUT_BF16: write the sum rounded to bf16 (8 values per 16-byte chunk) instead
// of fp32, the input format of the up-projection on the tensor cores.
template <int KMAX, bool OUT_BF16>
__global__ void MOE_PW_COMBINE_BOUNDS combine_kernel(const uint4 *__restrict__ ret_x,
                                                      const int32_t *__restrict__ ret_hdr,
                                                      const int32_t *__restrict__ slot_map,
                                                      const float *__restrict__ gates,
                                                      void *__restrict__ out_raw, int64_t T,
                                                      int k, int cpr, int64_t n_slots,
                                                      moe_pw_counters *ctr)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;
    for (int64_t t = warp; t < T; t += nwarp) {
        int32_t my_slot = -1;
        float my_gate = 0.0f;
        if (lane < k) {
            my_slot = slot_map[t * k + lane];
            my_gate = gates ? gates[t * k + lane] : 1.0f;
            if (my_slot >= n_slots) {
                set_error(ctr, MOE_PW_DEVERR_SLOT);
                my_slot = -1;
            }
            if (my_slot >= 0 && ret_hdr[my_slot] < 0) my_slot = -1;
        }
        int32_t slot[KMAX];
        float gv[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            slot[j] = __shfl_sync(FULL_MASK, my_slot, j);
            gv[j] = __shfl_sync(FULL_MASK, my_gate, j);
        }
        float4 *orow = reinterpret_cast<float4 *>(out_raw) + t * (cpr * 2);
        uint4 *brow = reinterpret_cast<uint4 *>(out_raw) + t * cpr;
        for (int c0 = lane; c0 < cpr; c0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
            // rows in groups of eight: all loads of a group, then its fmaf chain
#pragma unroll
            for (int jg = 0; jg < KMAX; jg += 8) {
                uint4 v[8][U];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int j = jg + jj;
                    if (j < k && slot[j] >= 0) {
                        const uint4 *row = ret_x + int64_t(slot[j]) * cpr;
#pragma unroll
                        for (int u = 0; u < U; ++u)
                            if (c0 + 32 * u < cpr) v[jj][u] = __ldg(row + c0 + 32 * u);
                    }
                }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int j = jg + jj;
                    if (j < k && slot[j] >= 0) {
#pragma unroll
                        for (int u = 0; u < U; ++u) fma_row(acc[u], gv[j], v[jj][u]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + 32 * u;
                if (c < cpr) {
                    if (OUT_BF16) {
                        uint4 o;
                        o.x = pack_bf16x2(acc[u][0], acc[u][1]);
                        o.y = pack_bf16x2(acc[u][2], acc[u][3]);
                        o.z = pack_bf16x2(acc[u][4], acc[u][5]);
                        o.w = pack_bf16x2(acc[u][6], acc[u][7]);
                        __stcs(brow + c, o);
                    } else {
                        __stcs(orow + 2 * c, make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]));
                        __stcs(orow + 2 * c + 1, make_float4(acc[u][4], acc[u][5], acc[u][6], acc[u][7]));
                    }
                }
            }
        }
    }
}

template <int KMAX, bool OUT_BF16>
cudaError_t launch_k(const Geo &g, const uint16_t *ret_x, const int32_t *ret_hdr,
                     const int32_t *slot_map, const float *gates, void *out,
                     moe_pw_counters *ctr, cudaStream_t st)
{
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    int64_t blocks = (g.T + 7) / 8;
    if (blocks > int64_t(di.sms) * MOE_PW_COMBINE_BLOCKS_PER_SM)
        blocks = int64_t(di.sms) * MOE_PW_COMBINE_BLOCKS_PER_SM;
    combine_kernel<KMAX, OUT_BF16><<<unsigned(blocks), 256, 0, st>>>(
        reinterpret_cast<const uint4 *>(ret_x), ret_hdr, slot_map, gates, out, g.T, g.k, g.D / 8,
        g.n_slots, ctr);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(const Geo &g, const uint16_t *ret_x, const int32_t *ret_hdr,
                           const int32_t *slot_map, const float *gates, float *out,
                           moe_pw_counters *ctr, cudaStream_t st)
{
    if (g.T == 0) return cudaSuccess;
    if (g.k <= 8) return launch_k<8, false>(g, ret_x, ret_hdr, slot_map, gates, out, ctr, st);
    if (g.k <= 16) return launch_k<16, false>(g, ret_x, ret_hdr, slot_map, gates, out, ctr, st);
    return launch_k<32, false>(g, ret_x, ret_hdr, slot_map, gates, out, ctr, st);
}

cudaError_t launch_combine_bf16(const Geo &g, const uint16_t *ret_x, const int32_t *ret_hdr,
                                const int32_t *slot_map, const float *gates, uint16_t *out,
                                moe_pw_counters *ctr, cudaStream_t st)
{
    if (g.T == 0) return cudaSuccess;
    if (g.k <= 8) return launch_k<8, true>(g, ret_x, ret_hdr, slot_map, gates, out, ctr, st);
    if (g.k <= 16) return launch_k<16, true>(g, ret_x, ret_hdr, slot_map, gates, out, ctr, st);
    return launch_k<32, true>(g, ret_x, ret_hdr, slot_map, gates, out, ctr, st);
}

}  // namespace moe_pw
