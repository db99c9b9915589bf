// route_body.cuh - top-k selection and softmax gates of one token by one
// warp, shared by the route kernel (route.cu) and the route + assignment
// kernel (route_assign.cu).  Internal; not part of the public ABI.
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 二: the router picks 8 of the
// 384 routed experts for every token.  Order (logit descending, expert id
// ascending) and softmax gates over the chosen logits are this library's
// reading.
//
// Layout: lane l holds float4 number l + 32*v of the row (v < NV), i.e. the
// logits of experts 4*(l + 32*v) + c.  Each logit becomes an order-preserving
// unsigned key (0 marks "taken or absent").  For ranking, a candidate carries
// the compound 64-bit key (logit key, ~expert id), so one unsigned comparison
// orders by logit descending, then id ascending.
// Selection: tau = the k-th largest of the 32 lane maxima bounds the top k
// from below; the logits >= tau (typically ~k of them) are compacted into
// shared memory and ranked exactly by (key descending, id ascending).  When
// more than 32 logits pass (many equal values), k exact rounds run instead:
// a warp-wide max of the keys (redux.sync), then a warp-wide min of the ids
// holding it.
#pragma once

#include "common.cuh"

namespace moe_pw {

// Order-preserving map float -> uint32; -0.0 is folded onto +0.0 first, so
// the two compare equal as floats do.  Finite floats map to keys >=
// 0x007FFFFF, so 0 never collides with a logit.
__device__ __forceinline__ uint32_t order_key(float f)
{
    const uint32_t u = __float_as_uint(f + 0.0f);  // -0.0 + 0.0 = +0.0
    return u ^ (uint32_t(int32_t(u) >> 31) | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t key)
{
    return __uint_as_float(key ^ ((key & 0x80000000u) ? 0x80000000u : 0xFFFFFFFFu));
}

template <int NV, bool FULL>
__device__ __forceinline__ void load_row(const float *__restrict__ logits, int64_t t, int E4,
                                         int lane, float4 (&f)[NV])
{
    const float4 *row = reinterpret_cast<const float4 *>(logits) + t * E4;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
        const int q = lane + 32 * v;
        if (FULL || q < E4) f[v] = __ldcs(row + q);
    }
}

// The k choices of the token whose row is `cur`: lane j < k gets choice j,
// its expert id and the two parts of its softmax gate, ex / sum (the caller
// divides, for lanes j < k only).  NV: float4s per lane; FULL: E == 128*NV
// (no bounds checks); KC: k fixed at compile time (0: run-time k).
// cand_sm[wib], sel_sm[wib], key_sm[wib]: this warp's shared scratch (NW
// warps per block; key_sm holds a lane's keys, used when NV <= 4, so that
// only the few candidates are read back for the compaction).  All 32 lanes
// call it.
template <int NV> struct KeyRows { static constexpr int V = NV <= 4 ? NV : 1; };

template <int NV, bool FULL, int KC, int NW>
__device__ __forceinline__ void route_select(const float4 (&cur)[NV], int k, int E4, int lane,
                                             int wib, unsigned long long (&cand_sm)[NW][32],
                                             unsigned long long (&sel_sm)[NW][32],
                                             uint4 (&key_sm)[NW][KeyRows<NV>::V][32],
                                             int32_t &sel_idx_out, float &ex_out,
                                             float &sum_out)
{
    const uint32_t base = 4u * lane;
    uint32_t key[NV][4];
#pragma unroll
    for (int v = 0; v < NV; ++v) {
        const bool in = FULL || lane + 32 * v < E4;
        key[v][0] = in ? order_key(cur[v].x) : 0u;
        key[v][1] = in ? order_key(cur[v].y) : 0u;
        key[v][2] = in ? order_key(cur[v].z) : 0u;
        key[v][3] = in ? order_key(cur[v].w) : 0u;
    }
    uint32_t lm = 0;
#pragma unroll
    for (int v = 0; v < NV; ++v)
#pragma unroll
        for (int c = 0; c < 4; ++c) lm = max(lm, key[v][c]);

    // tau = k-th largest lane maximum: at least k logits are >= tau, so
    // every one of the top k is >= tau.  Usually few logits pass.
    uint32_t rem = lm, tau = 0;
#pragma unroll
    for (int j = 0; j < (KC ? KC : 1); ++j) {
        tau = __reduce_max_sync(FULL_MASK, rem);
        rem = (rem == tau) ? 0u : rem;
    }
    if (!KC)
        for (int j = 1; j < k; ++j) {
            tau = __reduce_max_sync(FULL_MASK, rem);
            rem = (rem == tau) ? 0u : rem;
        }
    // candidates of this lane; NV <= 4: bit 4v + c of cmask for key[v][c] >= tau
    uint32_t cmask = 0;
    int cnt = 0;
    if (NV <= 4) {
#pragma unroll
        for (int v = 0; v < KeyRows<NV>::V; ++v)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (key[v][c] >= tau) cmask |= 1u << (4 * v + c);
        cnt = __popc(cmask);
    } else {
#pragma unroll
        for (int v = 0; v < NV; ++v)
#pragma unroll
            for (int c = 0; c < 4; ++c) cnt += key[v][c] >= tau;
    }
    const int C = tau ? int(__reduce_add_sync(FULL_MASK, unsigned(cnt))) : 1 << 30;

    uint32_t sel_key = 0;
    int32_t sel_idx = 0;
    if (C <= 32) {
        // compact the candidates (lane order, then element order) ...
        int pos = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(FULL_MASK, pos, o);
            if (lane >= o) pos += u;
        }
        pos -= cnt;
        if (NV <= 4) {
            // the lane's keys go to shared memory in NV 16-byte stores, and
            // only its candidates (set bits of cmask, ~9 per token over the
            // warp) are read back: no predicated store per logit.  A lane
            // reads only what it wrote, so no barrier is needed.
#pragma unroll
            for (int v = 0; v < KeyRows<NV>::V; ++v)
                key_sm[wib][v][lane] = make_uint4(key[v][0], key[v][1], key[v][2], key[v][3]);
            uint32_t m = cmask;
            while (m) {
                const int j = __ffs(m) - 1;
                m &= m - 1;
                const int v = j >> 2, c = j & 3;
                const uint32_t kj = reinterpret_cast<const uint32_t *>(&key_sm[wib][v][lane])[c];
                cand_sm[wib][pos++] =
                    (static_cast<unsigned long long>(kj) << 32) | ~(base + 128u * v + c);
            }
        } else {
#pragma unroll
            for (int v = 0; v < NV; ++v)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (key[v][c] >= tau)
                        cand_sm[wib][pos++] = (static_cast<unsigned long long>(key[v][c]) << 32) |
                                              ~(base + 128u * v + c);
        }
        if (lane >= C) cand_sm[wib][lane] = 0ull;  // ranks below every candidate
        __syncwarp();
        // ... and rank each one against all of them, two per 16-byte load
        const unsigned long long me = cand_sm[wib][lane];
        int rank = 0;
        const int C2 = (C + 1) & ~1;
        const ulonglong2 *pairs = reinterpret_cast<const ulonglong2 *>(&cand_sm[wib][0]);
#pragma unroll 2
        for (int i = 0; i < C2; i += 2) {
            const ulonglong2 q = pairs[i >> 1];
            rank += q.x > me;
            rank += q.y > me;
        }
        if (lane < C && rank < k) sel_sm[wib][rank] = me;
        __syncwarp();
        if (lane < k) {
            const unsigned long long s = sel_sm[wib][lane];
            sel_key = uint32_t(s >> 32);
            sel_idx = int32_t(~uint32_t(s));
        }
        __syncwarp();
    } else {
        // many equal logits: k exact rounds over every logit
        for (int j = 0; j < k; ++j) {
            uint32_t mx = 0;
#pragma unroll
            for (int v = 0; v < NV; ++v)
#pragma unroll
                for (int c = 0; c < 4; ++c) mx = max(mx, key[v][c]);
            const uint32_t m = __reduce_max_sync(FULL_MASK, mx);
            // lowest expert id in this lane whose key equals the maximum
            int32_t cid = 0x7FFFFFFF;
#pragma unroll
            for (int v = NV - 1; v >= 0; --v)
#pragma unroll
                for (int c = 3; c >= 0; --c)
                    if (key[v][c] == m) cid = base + 128 * v + c;
            const int32_t gi = __reduce_min_sync(FULL_MASK, cid);
            const int32_t rel = gi - int32_t(base);  // 128*v + c only in the owning lane
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
    }

    // softmax over the chosen logits: lane j holds choice j
    const float val = key_value(sel_key);
    const float top = __shfl_sync(FULL_MASK, val, 0);
    const float ex = (lane < k) ? expf(val - top) : 0.0f;
    float sum = 0.0f;
    if (KC == 8) {
        // butterfly over lanes 0..7: every lane of the group ends with the
        // same bits (each add's operands only swap places)
        sum = ex;
        sum += __shfl_xor_sync(FULL_MASK, sum, 1);
        sum += __shfl_xor_sync(FULL_MASK, sum, 2);
        sum += __shfl_xor_sync(FULL_MASK, sum, 4);
    } else {
#pragma unroll
        for (int j = 0; j < (KC ? KC : 1); ++j) sum += __shfl_sync(FULL_MASK, ex, j);
        if (!KC)
            for (int j = 1; j < k; ++j) sum += __shfl_sync(FULL_MASK, ex, j);
    }
    sel_idx_out = sel_idx;
    ex_out = ex;
    sum_out = sum;
}

}  // namespace moe_pw
