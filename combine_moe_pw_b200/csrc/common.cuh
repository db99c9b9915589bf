// common.cuh - internal declarations and device helpers of libmoe_pw.so.
// Not part of the public ABI (include/moe_pw.h is).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "moe_pw.h"

namespace moe_pw {

constexpr unsigned FULL_MASK = 0xFFFFFFFFu;

// Everything a kernel needs to know about the batch, derived on the host
// from a validated moe_pw_config.
struct Geo {
    int64_t T;        // tokens
    int32_t E, k, D, R, L, W, P;
    int32_t mode;     // MOE_PW_POOLED / MOE_PW_RAGGED
    int64_t T_s;      // tokens per source shard (pooled), T (ragged)
    int64_t C_s, C_r; // capacities (pooled)
    int64_t n_pools;  // R*R*W (pooled), 0 (ragged)
    int64_t n_slots;  // pool rows
    // ranking (assign) decomposition
    int32_t NB;       // bins: pools per source (R*W) or experts (E)
    int32_t n_groups; // sources (R) or 1
    int64_t group_tokens;   // tokens per group
    int64_t chunk_tokens;   // tokens per chunk
    int32_t chunks_per_group;
    int32_t n_chunks;
    // expert parallelism over GPUs: this GPU is ep_g of ep_n and hosts the
    // Rn = R / ep_n logical ranks [ep_g * Rn, (ep_g + 1) * Rn) (one GPU:
    // ep_n = 1, ep_g = 0, Rn = R)
    int32_t ep_n, ep_g, Rn;
};

// Peer tables of an expert-parallel run, passed to the kernels by value.
struct EpRows {
    uint16_t *x[MOE_PW_EP_MAX_GPUS];
    int32_t *hdr[MOE_PW_EP_MAX_GPUS];
};

// Per-device attributes, cached on first use.
struct DevInfo {
    int sms;
    int smem_optin;  // max dynamic shared memory per block (opt-in)
};
int dev_info(DevInfo *out);

// Kernel launchers (asynchronous; return cudaError_t of the launch).
cudaError_t launch_route(const Geo &g, const float *logits, int32_t *idx, float *gates,
                         cudaStream_t st);
// Route and sender assignment (with the kept slots' headers) in one
// clustered launch, pooled mode on one GPU; zeroes *ctr first.
// cudaErrorNotSupported (nothing enqueued) when the batch takes the separate
// kernels: the caller then runs launch_route and launch_assign.  form:
// MOE_PW_RA_* to ask for one form (cudaErrorInvalidValue if the clustered
// launch does not fit), -1 for the default choice.
cudaError_t launch_route_assign(const Geo &g, const float *logits, int32_t *idx, float *gates,
                                int32_t *slot_map, int32_t *occ, int32_t *pool_hdr,
                                moe_pw_counters *ctr, cudaStream_t st, int form = -1);
// The form launch_route_assign takes for this batch on the current device
// (MOE_PW_RA_*; MOE_PW_RA_SEPARATE: it returns cudaErrorNotSupported).
cudaError_t route_assign_plan(const Geo &g, int *form);
// pool_hdr (optional): also write the kept slots' headers (the expert id),
// as the fused pack + bucketing launch expects.
cudaError_t launch_assign(const Geo &g, const int32_t *idx, int32_t *slot_map, int32_t *occ,
                          moe_pw_counters *ctr, void *ws, cudaStream_t st,
                          int32_t *pool_hdr = nullptr);
// ep (optional): the receive pools of every GPU of an expert-parallel run;
// rows then go to the destination's GPU, only for waves in wave_mask.
cudaError_t launch_pack(const Geo &g, const uint16_t *x, const int32_t *idx,
                        const int32_t *slot_map, const int32_t *occ, uint16_t *pool_x,
                        int32_t *pool_hdr, moe_pw_counters *ctr, cudaStream_t st,
                        const EpRows *ep = nullptr, uint32_t wave_mask = ~0u);
// Pack and receiver bucketing in one launch (one GPU, pooled mode, T > 0):
// the kept slots' headers must already be in pool_hdr (launch_assign with
// pool_hdr); the launch writes the rows, the empty slots' headers and the
// bucketing's outputs.
cudaError_t launch_pack_bucket(const Geo &g, const uint16_t *x, const int32_t *idx,
                               const int32_t *slot_map, const int32_t *occ, uint16_t *pool_x,
                               int32_t *pool_hdr, int32_t *recv_row, int32_t *bucket_slot,
                               int32_t *expert_counts, moe_pw_counters *ctr, cudaStream_t st);
// occ == nullptr: an empty slot is one whose header is -1 (expert-parallel
// receive pools, where no counts are exchanged).
cudaError_t launch_bucket(const Geo &g, const int32_t *pool_hdr, const int32_t *occ,
                          int32_t *recv_row, int32_t *bucket_slot, int32_t *expert_counts,
                          moe_pw_counters *ctr, cudaStream_t st, uint32_t wave_mask = ~0u);
// ep (optional): the return pools of every GPU; results then go to the
// source's GPU, only for waves in wave_mask.
// ctr: MOE_PW_DEVERR_TIMEOUT of the bulk-copy kernel (nullptr: the kernel
// without waits runs).
cudaError_t launch_expert(const Geo &g, const uint16_t *pool_x, const int32_t *pool_hdr,
                          const int32_t *recv_row, const float *scale, uint16_t *ret_x,
                          int32_t *ret_hdr, moe_pw_counters *ctr, cudaStream_t st,
                          const EpRows *ep = nullptr, uint32_t wave_mask = ~0u);
cudaError_t launch_combine(const Geo &g, const uint16_t *ret_x, const int32_t *ret_hdr,
                           const int32_t *slot_map, const float *gates, float *out,
                           moe_pw_counters *ctr, cudaStream_t st);

cudaError_t launch_combine_bf16(const Geo &g, const uint16_t *ret_x, const int32_t *ret_hdr,
                                const int32_t *slot_map, const float *gates, uint16_t *out,
                                moe_pw_counters *ctr, cudaStream_t st);
cudaError_t launch_combine_backward(const Geo &g, const float *dout, const uint16_t *ret_x,
                                    const int32_t *ret_hdr, const int32_t *slot_map,
                                    const int32_t *idx, const float *gates, uint16_t *d_ret,
                                    float *dgates, float *dlogits, moe_pw_counters *ctr,
                                    cudaStream_t st);

int64_t balance_ws_bytes(int64_t T, int64_t L, int32_t E);
cudaError_t launch_balance(const Geo &g, int64_t seq_len, float alpha, const float *logits,
                           const int32_t *idx, float *f, float *P, float *loss, float *dlogits,
                           int32_t accumulate, void *ws, cudaStream_t st);

cudaError_t launch_gemm(const uint16_t *A, const uint16_t *Bt, int64_t M, int32_t N, int32_t K,
                        int32_t mode, uint16_t *C, int64_t ldc, const int32_t *slot_map,
                        const int32_t *idx, int32_t topk, uint16_t *pool_x, int32_t *pool_hdr,
                        int64_t n_slots, moe_pw_counters *ctr, cudaStream_t st,
                        const uint16_t *add = nullptr);

// Workspace layout of the ranking pass.
inline int64_t align256(int64_t b) { return (b + 255) & ~int64_t(255); }
inline int64_t ws_counts_bytes(const Geo &g) { return align256(4 * int64_t(g.n_chunks) * g.NB); }
inline int64_t ws_totals_bytes(const Geo &g) { return align256(4 * int64_t(g.n_groups) * g.NB); }
inline int64_t ws_bytes(const Geo &g) { return ws_counts_bytes(g) + ws_totals_bytes(g); }

// ---------------------------------------------------------------------------
// Device helpers: mbarrier and bulk (TMA) copies, inline PTX for sm_100a.
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Make barrier initialisation and generic-proxy shared-memory writes visible
// to the async proxy (TMA) before any bulk copy uses them.
__device__ __forceinline__ void fence_init_and_proxy()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait on a barrier phase: gives up after `limit` polls (each poll
// may itself suspend for a hardware time slice).  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint32_t limit)
{
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// Global -> shared bulk copy, completion counted on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src, uint32_t bytes,
                                         uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// Shared -> global bulk copy in the calling thread's current bulk group.
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src_smem, uint32_t bytes,
                                         uint64_t policy)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(dst),
                 "r"(smem_addr(src_smem)), "r"(bytes), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until all of this thread's bulk groups have completed (writes performed).
__device__ __forceinline__ void bulk_wait_all()
{
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// L2 eviction policies for the bulk copies.
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Expert-parallel relabelling of a pool slot (32-bit: slot ids fit in int32).
// Send slot q = ((s_loc*R + d)*W + w)*C_s + c of GPU g -> the destination's
// GPU h = d / Rn and its receive slot ((s*Rn + d_loc)*W + w)*C_s + c.
__device__ __forceinline__ uint32_t ep_send_to_recv(const Geo &g, uint32_t q, int &h, int &w)
{
    const uint32_t Cs = uint32_t(g.C_s), W = uint32_t(g.W), R = uint32_t(g.R),
                   Rn = uint32_t(g.Rn);
    const uint32_t c = q % Cs, r1 = q / Cs;
    w = int(r1 % W);
    const uint32_t r2 = r1 / W;
    const uint32_t d = r2 % R, s_loc = r2 / R;
    h = int(d / Rn);
    const uint32_t d_loc = d - uint32_t(h) * Rn;
    const uint32_t s = uint32_t(g.ep_g) * Rn + s_loc;
    return ((s * Rn + d_loc) * W + uint32_t(w)) * Cs + c;
}

// Receive slot rq = ((s*Rn + d_loc)*W + w)*C_s + c of GPU g -> the source's
// GPU h = s / Rn and its send slot ((s_loc*R + d)*W + w)*C_s + c.
__device__ __forceinline__ uint32_t ep_recv_to_send(const Geo &g, uint32_t rq, int &h, int &w)
{
    const uint32_t Cs = uint32_t(g.C_s), W = uint32_t(g.W), R = uint32_t(g.R),
                   Rn = uint32_t(g.Rn);
    const uint32_t c = rq % Cs, r1 = rq / Cs;
    w = int(r1 % W);
    const uint32_t r2 = r1 / W;
    const uint32_t d_loc = r2 % Rn, s = r2 / Rn;
    h = int(s / Rn);
    const uint32_t s_loc = s - uint32_t(h) * Rn;
    const uint32_t d = uint32_t(g.ep_g) * Rn + d_loc;
    return ((s_loc * R + d) * W + uint32_t(w)) * Cs + c;
}

__device__ __forceinline__ void set_error(moe_pw_counters *ctr, int bits)
{
    atomicOr(&ctr->error, bits);
}

// Ranking bin of expert e: pooled, the pool (d, w) of its rank and wave
// within a source, (e / L) * W + (e % L) / P; ragged, the expert itself.
__device__ __forceinline__ int32_t bin_of_expert(const Geo &g, int32_t e)
{
    return g.mode == MOE_PW_POOLED ? (e / g.L) * g.W + (e % g.L) / g.P : e;
}

// Lanes of the warp holding the same bin b >= 0 as this lane (b < 0: none),
// through a per-warp array of lane masks in shared memory, zero on entry:
// each lane sets its bit in mask[b] and reads the word back.  The caller's
// lowest lane of each group (lane == __ffs(result) - 1) must set mask[b] back
// to 0, after a __syncwarp, before the next call.  One shared-memory atomic
// instead of a ballot per bit of the bin id.
__device__ __forceinline__ unsigned equal_lanes_smem(int32_t b, uint32_t *mask, int lane)
{
    if (b >= 0) atomicOr(&mask[b], 1u << lane);
    __syncwarp();
    return b >= 0 ? mask[b] : 0u;
}

// Programmatic dependent launch: a kernel launched with
// cudaLaunchAttributeProgrammaticStreamSerialization may start while the
// previous kernel in its stream is finishing; griddep_wait() returns once
// that kernel has completed and its memory is visible (at once for a normal
// launch).  Only shared-memory set-up may come before it.
__device__ __forceinline__ void griddep_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace moe_pw
