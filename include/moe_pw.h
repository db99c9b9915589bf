/*
 * moe_pw.h - C ABI of libmoe_pw.so: capacity-limited pooled-wave MoE token
 * dispatch and combine on one NVIDIA B200 (sm_100a).
 *
 * The method is the expert-parallel transport of the Marin 535B-A23B model,
 * described in "Marin 开始公开训练 535B 参数 MoE 模型" (lamjinlab blog),
 * section 二 (how the sparse model is organised):
 *   - a router picks k = 8 of E = 384 routed experts per token;
 *   - experts sit on R = 64 expert-parallel ranks, L = 6 per rank;
 *   - the sender builds one fixed pool per destination rank, not one buffer
 *     per expert, and sends it in W = 3 waves of identical shape;
 *   - the expert id travels inside the row payload, so no token counts or
 *     routing metadata are exchanged;
 *   - a sender factor 1.10 caps what one source sends one destination and a
 *     receiver factor 1.15 caps the rows one local expert accepts; assignments
 *     over either fixed buffer are dropped and the two drops are counted apart.
 * Section 四 of the same page adds that a dropped assignment does not lose
 * the token and names a dropless ragged all-to-all as an alternative; the
 * huxiu article "535B大模型“直播”训练三个月" (MoE / token dropping section) notes
 * that results come back through a second all-to-all.
 *
 * Here the R ranks are logical shards of one batch on one GPU: the exchange is
 * a relabelling of pool indices in HBM (destination d reads pool (s, d, w)
 * where source s wrote it), so nothing crosses a device boundary.
 *
 * Conventions that the pages leave open (and this library fixes):
 *   - token t belongs to source s = t / (T / R); expert e lives on rank
 *     d = e / L as local expert e % L; wave w carries local experts
 *     {P*w, ..., P*w + P - 1} (P = L / W);
 *   - top-k order is (logit descending, expert id ascending): equal logits go
 *     to the lower id (float comparison: -0.0 equals +0.0); gates are the
 *     softmax over the k chosen logits, max-subtracted (the device sums the
 *     k exponentials in a fixed order: a butterfly for k = 8, j order
 *     otherwise; gates agree with the exact softmax within 1e-6);
 *   - sender order: assignments (t, j) of a source in lexicographic order; the
 *     slot of (t, j) in pool (s, d, w) is the number of earlier ones in that
 *     pool; kept iff slot < C_s;
 *   - receiver order: per (d, w), sources ascending, then slots ascending; the
 *     row of an arrival is the number of earlier arrivals for its expert; kept
 *     iff row < C_r;
 *   - capacities C_s = ceil(cf_s% * (T/R) * k * P / (100 * E)),
 *     C_r = ceil(cf_r% * T * k / (100 * E)); a factor <= 0 is unbounded
 *     (C_s = (T/R) * min(k, P), C_r = T);
 *   - empty slots hold an all-zero row and header -1;
 *   - per-expert op (stand-in for the expert network): y = s_e * x in fp32,
 *     rounded to bf16 nearest-even; the return pools share the dispatch pools'
 *     slot ids; slots the receiver did not keep return zeros and header -1;
 *   - combine: out[t] = sum over surviving j of g_j * y_j in fp32, j
 *     ascending, one fmaf per term from +0; no renormalisation over drops.
 *
 * Data layout (all row-major, element types as named):
 *   logits  f32  [T, E]
 *   idx     i32  [T, k]          gates f32 [T, k]
 *   x       bf16 [T, D]          (raw bits as uint16_t)
 *   slot_map i32 [T, k]          flat slot id of (t, j), or -1 if sender-dropped
 *   occ     i32  pooled: [R(src), R(dst), W] rows kept per pool
 *                ragged: [E + 1] row offsets of each expert (exclusive scan)
 *   pool_x  bf16 [n_slots, D]    pooled: slot = ((s*R + d)*W + w)*C_s + c
 *   pool_hdr i32 [n_slots]       global expert id, or -1
 *   recv_row i32 [n_slots]       row of the slot in its expert bucket, or -1
 *   bucket_slot i32 [E, C_r]     slot of each bucket row, or -1 (pooled only)
 *   expert_counts i32 [2, E]     arrivals[e], then kept[e] = min(arrivals, C_r)
 *   scale   f32  [E]
 *   ret_x   bf16 [n_slots, D]    ret_hdr i32 [n_slots]
 *   out     f32  [T, D]
 * In ragged mode n_slots = T * k rows, grouped by expert (ascending), token
 * order inside an expert; slot_map holds row ids and nothing is dropped.
 *
 * Ownership: the caller allocates every buffer (device memory unless stated)
 * and keeps it alive until the stream work completes.  The library allocates
 * nothing and keeps no state between calls except a per-device cache of
 * attributes; calls are reentrant.
 *
 * Alignment: logits, x, pool_x, ret_x and out 16-byte aligned; every other
 * array 4-byte aligned; the workspace 256-byte aligned.
 *
 * Errors: every call returns MOE_PW_OK (0) or a negative code and never
 * aborts, traps or throws.  Device-side violations (an expert id out of range
 * in idx, a header outside its pool's experts, a bounded wait that ran out)
 * set counters->error; moe_pw_stats reports them as MOE_PW_EDEVICE.
 * All calls except moe_pw_plan and moe_pw_stats are asynchronous on `stream`.
 */
#ifndef MOE_PW_H
#define MOE_PW_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_PW_OK 0
#define MOE_PW_EINVAL (-1)        /* null pointer, bad config, inconsistent sizes */
#define MOE_PW_EUNSUPPORTED (-2)  /* shape or alignment this library does not handle */
#define MOE_PW_ECUDA (-3)         /* a CUDA runtime call or a launch failed */
#define MOE_PW_EDEVICE (-4)       /* a kernel flagged a violation (moe_pw_stats) */
#define MOE_PW_ENOMEM (-5)        /* buffers exceed the caller's budget (moe_pw_plan) or the
                                     built-in scratch (moe_pw_assign_noalloc) */

#define MOE_PW_POOLED 0
#define MOE_PW_RAGGED 1

/* counters->error bits */
#define MOE_PW_DEVERR_EXPERT_ID 1   /* idx entry outside [0, E) */
#define MOE_PW_DEVERR_HEADER 2      /* pool header outside its (d, w) experts */
#define MOE_PW_DEVERR_TIMEOUT 4     /* a bounded wait gave up: that launch's outputs are
                                       incomplete.  The kernel first waits, again with a
                                       bound, for the copies it has in flight; if those
                                       waits run out too, copies may still land after the
                                       kernel ends, so treat the outputs (and, to be safe,
                                       the context) as suspect and re-run the step */
#define MOE_PW_DEVERR_SLOT 8        /* slot_map entry outside [-1, n_slots) */

/* Problem description.  Limits of this library: 1 <= k <= 32, k <= E,
 * E == R * L, L == W * P, E <= 2048 (and E % 4 == 0 for moe_pw_route),
 * T % R == 0, 8 <= D <= 12288 with D % 8 == 0, R * W <= 2048. */
typedef struct moe_pw_config {
    int64_t T;            /* tokens in the batch (>= 0) */
    int32_t E;            /* routed experts */
    int32_t k;            /* experts chosen per token */
    int32_t D;            /* latent width, bf16 elements */
    int32_t R;            /* expert-parallel ranks (logical) */
    int32_t L;            /* experts per rank */
    int32_t W;            /* waves per (source, destination) */
    int32_t P;            /* experts per wave */
    int32_t cf_send_pct;  /* sender capacity factor, percent (110); <= 0 unbounded */
    int32_t cf_recv_pct;  /* receiver capacity factor, percent (115); <= 0 unbounded */
    int32_t mode;         /* MOE_PW_POOLED or MOE_PW_RAGGED */
} moe_pw_config;

/* Sizes derived from a config by moe_pw_plan.  Element counts unless "bytes". */
typedef struct moe_pw_sizes {
    int64_t C_s;            /* sender capacity per (s, d, w) pool (pooled) */
    int64_t C_r;            /* receiver capacity per expert (pooled) */
    int64_t n_pools;        /* R * R * W (pooled), 0 (ragged) */
    int64_t n_slots;        /* rows of pool_x / ret_x */
    int64_t occ_len;        /* int32 entries of occ */
    int64_t bucket_len;     /* int32 entries of bucket_slot (0 in ragged mode) */
    int64_t workspace_bytes;/* scratch for moe_pw_assign / moe_pw_dispatch */
    int64_t total_bytes;    /* every buffer of the path, logits to out */
} moe_pw_sizes;

/* Device-side counters, written by the kernels.  moe_pw_assign zeroes them.
 * Calls that may run at the same time need counters of their own. */
typedef struct moe_pw_counters {
    unsigned long long sender_dropped;
    unsigned long long receiver_dropped;
    unsigned long long kept;
    int32_t max_occ;     /* largest pool occupancy */
    int32_t max_fill;    /* largest per-expert kept count */
    int32_t error;       /* MOE_PW_DEVERR_* bits */
    int32_t work;        /* scratch: moe_pw_pack's counter of pools handed out for
                            zero-filling (reset by moe_pw_pack before its kernel) */
} moe_pw_counters;

/* Host copy of the counters, filled by moe_pw_stats. */
typedef struct moe_pw_drop_stats {
    int64_t assignments;       /* T * k */
    int64_t kept;              /* rows every expert accepted */
    int64_t sender_dropped;
    int64_t receiver_dropped;
    int32_t max_occ;
    int32_t max_fill;
    int32_t error;
    int32_t reserved;
} moe_pw_drop_stats;

/* Library version (major * 10000 + minor * 100 + patch). */
int moe_pw_version(void);

/* Text for a return code (static storage). */
const char *moe_pw_strerror(int code);

/*
 * Host-only.  Validates `cfg` and fills `out` with capacities and buffer
 * sizes.  budget_bytes > 0 makes the call fail with MOE_PW_ENOMEM when the
 * path's buffers (out->total_bytes) exceed it: the pages record a fixed
 * expert-cell design whose memory estimate failed allocation, and a caller
 * can refuse such a config before allocating.  Never touches the GPU.
 */
int moe_pw_plan(const moe_pw_config *cfg, int64_t budget_bytes, moe_pw_sizes *out);

/*
 * Route (section 二: the router picks k experts per token).  One warp per
 * token selects the k largest logits (ties to the lower id) and writes their
 * ids to idx and their softmax gates to gates.  Logits must be finite.
 */
int moe_pw_route(const moe_pw_config *cfg, const float *logits, int32_t *idx, float *gates,
                 cudaStream_t stream);

/*
 * Sender slot assignment (section 二: fixed per-destination pools, sender
 * factor).  Zeroes *counters, then writes slot_map and occ and counts sender
 * drops.  Ranks come from per-chunk histograms and a prefix scan over chunks,
 * so the result is deterministic.  Ragged mode: slot_map receives row ids and
 * occ the E + 1 expert row offsets.  workspace: device scratch of at least
 * moe_pw_sizes.workspace_bytes, 256-byte aligned; its contents on entry do
 * not matter.
 */
int moe_pw_assign(const moe_pw_config *cfg, const int32_t *idx, int32_t *slot_map,
                  int32_t *occ, moe_pw_counters *counters, void *workspace,
                  size_t workspace_bytes, cudaStream_t stream);

/*
 * Pack (section 二: expert id in the payload).  Copies each kept row x[t] into
 * its slot with TMA bulk copies through shared memory (one read of x[t], up to
 * k writes), writes the expert id into the slot header, and fills the empty
 * tail of every pool (positions >= occ) with zeros and header -1.  Ragged
 * mode: rows only, no empty slots.  A slot_map entry >= n_slots is skipped
 * and flagged in counters->error (which moe_pw_assign zeroed).  The empty
 * tails are handed out to the kernel's warps through counters->work, which
 * this call resets on `stream` before the kernel; two packs that share a
 * counters struct must not run at the same time.
 */
int moe_pw_pack(const moe_pw_config *cfg, const uint16_t *x, const int32_t *idx,
                const int32_t *slot_map, const int32_t *occ, uint16_t *pool_x,
                int32_t *pool_hdr, moe_pw_counters *counters, cudaStream_t stream);

/*
 * Exchange + receiver bucketing (section 二: receiver factor; huxiu: first
 * all-to-all).  For every (d, w) walks the pools (s, d, w), s ascending, over
 * positions c < occ, and ranks each arrival within its expert.  Writes
 * recv_row, bucket_slot (pooled; may be NULL in ragged mode) and
 * expert_counts, and adds receiver drops and kept rows to *counters.
 */
int moe_pw_bucket(const moe_pw_config *cfg, const int32_t *pool_hdr, const int32_t *occ,
                  int32_t *recv_row, int32_t *bucket_slot, int32_t *expert_counts,
                  moe_pw_counters *counters, cudaStream_t stream);

/*
 * Allocation-free moe_pw_assign.  (The pages have no counterpart: this is an
 * interface convenience of this library, not part of the method.)
 *
 * For callers that cannot allocate device memory for a workspace: a plugin
 * whose host process owns every device allocation and gives it no allocator,
 * or a latency-critical loop that must never call cudaMalloc/cudaFree, which
 * can synchronise the whole device.  Same inputs, outputs and results as
 * moe_pw_assign, but the ranking scratch is a fixed array of
 * MOE_PW_NOALLOC_SCRATCH_BYTES compiled into the library: every GPU that
 * loads the library holds it until the process exits.  This call allocates
 * nothing and calls no allocating routine.
 *   - A batch whose ranking needs more scratch than that (workspace_bytes of
 *     moe_pw_plan above the limit) is refused with MOE_PW_ENOMEM before any
 *     launch; the rack-scale batch (262,144 tokens, 64 ranks, 3 waves) needs
 *     under 1 MiB.
 *   - Every call looks up the array's device address in the current
 *     device's context (cudaGetSymbolAddress, with that device current); the
 *     first call on a device also loads the library's device code there, so
 *     make that first call before any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents; nothing in it needs to start at zero (each call writes every
 *     entry it reads).  Calls whose kernels overlap on the GPU, such as calls
 *     on two streams without ordering between them, race on the array and
 *     give wrong slots: order them on one stream or with events.
 */
#define MOE_PW_NOALLOC_SCRATCH_BYTES (4u << 20)
int moe_pw_assign_noalloc(const moe_pw_config *cfg, const int32_t *idx, int32_t *slot_map,
                          int32_t *occ, moe_pw_counters *counters, cudaStream_t stream);

/*
 * moe_pw_route followed by moe_pw_assign_headers, in one launch where the
 * batch allows (pooled mode, one GPU; moe_pw_route_assign_plan says which
 * form runs).  Outputs (idx, gates, slot_map, occ, the kept slots' headers in
 * pool_hdr, *counters zeroed and then the sender drops) equal those of the
 * two calls in either form:
 *   - MOE_PW_RA_CLUSTER (up to 256 tokens per SM): one thread-block
 *     cluster per source shard routes the shard's tokens, exchanges the
 *     per-pool counts of its blocks through distributed shared memory and
 *     ranks the choices; no global workspace is touched.  A cluster is tied
 *     to one shard, so its route work cannot spread evenly over the SMs; on
 *     larger batches that costs more than the separate kernels' fixed
 *     latency.
 *   - MOE_PW_RA_SEPARATE: the two calls (larger batches, or a shape the
 *     clustered launch does not fit: shared memory per block, or no cluster
 *     placement on this device).
 * workspace and workspace_bytes are as for moe_pw_assign.  Pooled mode only
 * (MOE_PW_EUNSUPPORTED otherwise).
 */
int moe_pw_route_assign(const moe_pw_config *cfg, const float *logits, int32_t *idx,
                        float *gates, int32_t *slot_map, int32_t *occ, int32_t *pool_hdr,
                        moe_pw_counters *counters, void *workspace, size_t workspace_bytes,
                        cudaStream_t stream);

#define MOE_PW_RA_SEPARATE 0
#define MOE_PW_RA_CLUSTER 1

/*
 * moe_pw_route_assign in the given form (MOE_PW_RA_*), or -1 for its default
 * choice: for timing the forms against one another and testing each.
 * MOE_PW_EUNSUPPORTED if the form does not fit the batch on this device
 * (nothing enqueued); MOE_PW_RA_SEPARATE always fits.
 */
int moe_pw_route_assign_form(const moe_pw_config *cfg, int32_t form, const float *logits,
                             int32_t *idx, float *gates, int32_t *slot_map, int32_t *occ,
                             int32_t *pool_hdr, moe_pw_counters *counters, void *workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/*
 * The form moe_pw_route_assign takes for this batch on the current device:
 * *form = one of MOE_PW_RA_* above.  Needs a CUDA device (occupancy queries;
 * nothing is launched).
 */
int moe_pw_route_assign_plan(const moe_pw_config *cfg, int32_t *form);

/*
 * moe_pw_assign that also writes the header (the expert id) of every slot the
 * sender kept into pool_hdr [n_slots]; the other headers are left as they
 * are.  Pooled mode only (MOE_PW_EUNSUPPORTED otherwise).  The first half of
 * the fused dispatch: moe_pw_pack_bucket then needs no headers from the pack.
 */
int moe_pw_assign_headers(const moe_pw_config *cfg, const int32_t *idx, int32_t *slot_map,
                          int32_t *occ, int32_t *pool_hdr, moe_pw_counters *counters,
                          void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * moe_pw_pack and moe_pw_bucket in one launch (pooled mode, one GPU).  The
 * bucketing reads only the occupancies and the kept slots' headers, so it
 * runs beside the row copies instead of after them: the pack's copy warp of
 * every block drives the TMA engine while the block's other warps bucket the
 * (destination, wave) items.  Precondition: pool_hdr holds the kept slots'
 * headers of this batch, written by moe_pw_assign_headers with the same
 * idx, slot_map and occ (the pack writes no headers here).  Writes pool_x
 * (kept rows; zero rows in the empty tails), the empty slots' headers (-1),
 * recv_row, bucket_slot and expert_counts, and adds receiver drops and kept
 * rows to *counters: every output equals moe_pw_pack followed by
 * moe_pw_bucket.  Ragged mode: MOE_PW_EUNSUPPORTED.  T = 0: the two calls
 * are made one after the other.  Hands the empty pool tails out through
 * counters->work, which must be 0 on entry: the assignment call before it
 * (moe_pw_assign_headers or moe_pw_route_assign) zeroes the counters, and
 * nothing else may run on these counters in between.
 */
int moe_pw_pack_bucket(const moe_pw_config *cfg, const uint16_t *x, const int32_t *idx,
                       const int32_t *slot_map, const int32_t *occ, uint16_t *pool_x,
                       int32_t *pool_hdr, int32_t *recv_row, int32_t *bucket_slot,
                       int32_t *expert_counts, moe_pw_counters *counters, cudaStream_t stream);

/*
 * moe_pw_assign, moe_pw_pack and moe_pw_bucket in one call.  Pooled mode:
 * moe_pw_assign_headers then moe_pw_pack_bucket (same outputs).
 */
int moe_pw_dispatch(const moe_pw_config *cfg, const uint16_t *x, const int32_t *idx,
                    int32_t *slot_map, int32_t *occ, uint16_t *pool_x, int32_t *pool_hdr,
                    int32_t *recv_row, int32_t *bucket_slot, int32_t *expert_counts,
                    moe_pw_counters *counters, void *workspace, size_t workspace_bytes,
                    cudaStream_t stream);

/*
 * Per-expert op and return layout (stand-in for the expert network; huxiu:
 * results return by a second all-to-all).  For every slot: if the receiver
 * kept it (recv_row >= 0), ret_x = bf16_rn(scale[e] * pool_x) and ret_hdr = e;
 * otherwise ret_x = 0 and ret_hdr = -1.  On one GPU the rows stream through
 * shared memory by bulk copies with bounded waits: a wait that gives up sets
 * MOE_PW_DEVERR_TIMEOUT in counters->error (device memory, 8-byte aligned;
 * nothing else in *counters is touched).
 */
int moe_pw_expert(const moe_pw_config *cfg, const uint16_t *pool_x, const int32_t *pool_hdr,
                  const int32_t *recv_row, const float *scale, uint16_t *ret_x,
                  int32_t *ret_hdr, moe_pw_counters *counters, cudaStream_t stream);

/*
 * Combine (section 四: a dropped assignment leaves the token, so its term is
 * simply absent).  out[t] = sum_j g_j * float(ret_x[slot_map[t][j]]) over
 * j with slot >= 0 and ret_hdr[slot] >= 0, fp32, j ascending, fmaf from +0.
 * A slot_map entry >= n_slots is skipped and flagged in counters->error.
 */
int moe_pw_combine(const moe_pw_config *cfg, const uint16_t *ret_x, const int32_t *ret_hdr,
                   const int32_t *slot_map, const float *gates, float *out,
                   moe_pw_counters *counters, cudaStream_t stream);

/*
 * moe_pw_combine with the fp32 sum rounded to bf16 nearest-even (out: bf16
 * [T, D]), the input of the up-projection (moe_pw_project with the up weights)
 * that takes the combined latent back to model width (section 二).
 */
int moe_pw_combine_bf16(const moe_pw_config *cfg, const uint16_t *ret_x, const int32_t *ret_hdr,
                        const int32_t *slot_map, const float *gates, uint16_t *out,
                        moe_pw_counters *counters, cudaStream_t stream);

/*
 * moe_pw_combine_bf16 for the tokens [first_token, first_token + n_tokens) of
 * the batch only: out (bf16 [n_tokens, D]) row i is token first_token + i.
 * Lets the combine of one block of tokens run while the up-projection of the
 * previous block is on the tensor cores (Buffers.run_routed_layer with
 * chunk_tokens), so the latent passes through a small buffer that stays in
 * L2.  MOE_PW_EINVAL if the range leaves the batch.
 */
int moe_pw_combine_bf16_rows(const moe_pw_config *cfg, const uint16_t *ret_x,
                             const int32_t *ret_hdr, const int32_t *slot_map, const float *gates,
                             int64_t first_token, int64_t n_tokens, uint16_t *out,
                             moe_pw_counters *counters, cudaStream_t stream);

/*
 * Backward of the combine.  The pages train this model ("Marin 开始公开训练 535B
 * 参数 MoE 模型", section 一) but give no backward; this is the derivative of the
 * forward definitions above.  Given dout = dL/dout (f32 [T, D]):
 *   d_ret (bf16 [n_slots, D], the gradient pool, same slot ids as ret_x):
 *     for every surviving (t, j) (slot >= 0, ret_hdr[slot] >= 0)
 *     d_ret[slot] = bf16_rn(g_j * dout[t]) with the product in fp32; every
 *     other slot is zeroed (a fixed pool, like the forward's);
 *   dgates (f32 [T, k], may be NULL): <dout[t], y_j> for surviving (t, j),
 *     else 0 (fp32, each lane's share in chunk order, then a fixed xor tree);
 *   dlogits (f32 [T, E], may be NULL): the top-k softmax backward,
 *     dlogits[t][idx[t][j]] = g_j * (dgate_j - sum_i g_i dgate_i), all other
 *     logits 0 (top-k selection is piecewise constant in the logits).
 * The stand-in expert op's backward is moe_pw_expert applied to d_ret (the
 * same scale op, its bf16 rounding passed straight through), giving d_pool.
 */
int moe_pw_combine_backward(const moe_pw_config *cfg, const float *dout, const uint16_t *ret_x,
                            const int32_t *ret_hdr, const int32_t *slot_map, const int32_t *idx,
                            const float *gates, uint16_t *d_ret, float *dgates, float *dlogits,
                            moe_pw_counters *counters, cudaStream_t stream);

/*
 * Backward of the pack: x[t] was copied into the slot of each (t, j) the
 * sender kept, so dx[t] = sum over those j of d_pool[slot] (f32 [T, D], j
 * ascending, exact fp32 adds from +0).  Slots the receiver dropped
 * (recv_row < 0) carry zero gradient and are skipped.
 */
int moe_pw_dispatch_backward(const moe_pw_config *cfg, const uint16_t *d_pool,
                             const int32_t *recv_row, const int32_t *slot_map, float *dx,
                             moe_pw_counters *counters, cudaStream_t stream);

/*
 * Latent projection on the tensor cores (section 二: the routed activations are
 * compressed from the 6144-wide model state to 3072 before the exchange and
 * projected back afterwards).  C[m][n] = bf16_rn(sum_k A[m][k] * Bt[n][k]),
 * fp32 accumulation in TMEM (tcgen05.mma, bf16 operands).  A: bf16 [M, K]
 * row-major, Bt: bf16 [N, K] row-major (one row per output column), C: bf16
 * [M, N].  K % 8 == 0, N % 8 == 0, all three 16-byte aligned.  counters
 * receives MOE_PW_DEVERR_TIMEOUT if a bounded wait gives up.  The product runs
 * on pairs of SMs (tcgen05 cta_group::2, 256 x 256 tiles) where a cluster of
 * two CTAs can be launched, else on single SMs (128 x 256 tiles); setting the
 * environment variable MOE_PW_GEMM_PAIR=0 before the first call selects the
 * single-SM kernel.  Both give bit-identical results.
 */
int moe_pw_project(const uint16_t *A, const uint16_t *Bt, uint16_t *C, int64_t M, int32_t N,
                   int32_t K, moe_pw_counters *counters, cudaStream_t stream);

/*
 * Up-projection merged with the shared-expert path (section 二: the routed
 * outputs are projected back to model width before they merge with the two
 * shared experts, which run locally on every token):
 *   C[m][n] = bf16_rn(sum_k A[m][k] * Bt[n][k] + add[m][n]),
 * the sum accumulated in fp32 (TMEM), add (bf16 [M, N], the shared path's
 * output) added in fp32 in the epilogue, one rounding to bf16.  add may be C
 * itself (in place).  Shapes, alignment and kernels as moe_pw_project.
 */
int moe_pw_project_add(const uint16_t *A, const uint16_t *Bt, const uint16_t *add, uint16_t *C,
                       int64_t M, int32_t N, int32_t K, moe_pw_counters *counters,
                       cudaStream_t stream);

/*
 * Down-projection fused with the pack: pool_x[slot] = bf16(h[t] @ w_down_t^T)
 * for every (t, j) the sender kept (slot_map from moe_pw_assign), written by
 * the GEMM epilogue directly into the pool slots, headers as in moe_pw_pack,
 * and the empty pool tails zero-filled: the same pools moe_pw_pack builds
 * from x = bf16(h @ w_down_t^T), without materialising x.
 * h: bf16 [T, model_width]; w_down_t: bf16 [D, model_width].  The tail fill
 * uses counters->work as moe_pw_pack does.
 */
int moe_pw_project_pack(const moe_pw_config *cfg, const uint16_t *h, const uint16_t *w_down_t,
                        int32_t model_width, const int32_t *idx, const int32_t *slot_map,
                        const int32_t *occ, uint16_t *pool_x, int32_t *pool_hdr,
                        moe_pw_counters *counters, cudaStream_t stream);

/*
 * Sequence-level balancing ("Marin 开始公开训练 535B 参数 MoE 模型", section 四:
 * the third remedy named for high drop rates, one that may make the experts
 * re-specialise during training; the pages give no formula).  This library's
 * reading is a per-sequence balance term of the training loss.  For each
 * sequence s of seq_len = L consecutive tokens (T % L == 0):
 *   p[t][e] = softmax over all E logits of token t
 *   f[s][e] = E / (k L) * (assignments of s to e in idx)   (1 at balance)
 *   P[s][e] = (1 / L) * sum over t in s of p[t][e]
 *   loss[s] = alpha * sum_e f[s][e] * P[s][e]               (alpha at balance)
 * and, when dlogits is not NULL, its gradient with the routing held fixed,
 *   dlogits[t][e] = alpha / L * p[t][e] * (f[s][e] - sum_i f[s][i] p[t][i]),
 * written (accumulate = 0) or added to dlogits (accumulate != 0, e.g. onto
 * the top-k softmax gradient of moe_pw_combine_backward).  logits f32 [T, E]
 * (16-byte aligned), idx i32 [T, k]; f (16-byte aligned), P f32 [T / L, E];
 * loss f32 [T / L];
 * dlogits f32 [T, E] (16-byte aligned).  Sums in fp32 in a fixed order
 * (deterministic).  workspace: at least the bytes moe_pw_seq_balance_plan
 * gives, 256-byte aligned.  E % 4 == 0.
 */
int moe_pw_seq_balance_plan(const moe_pw_config *cfg, int64_t seq_len, int64_t *workspace_bytes);
int moe_pw_seq_balance(const moe_pw_config *cfg, int64_t seq_len, float alpha,
                       const float *logits, const int32_t *idx, float *f, float *P, float *loss,
                       float *dlogits, int32_t accumulate, void *workspace,
                       size_t workspace_bytes, cudaStream_t stream);

/*
 * Drop statistics (section 二: the two kinds of drop are reported apart).
 * Copies *counters (device) to *host_out (host memory) and, when both
 * expert_counts (device, i32 [2, E] as written by moe_pw_bucket) and
 * host_expert_counts (host, i32 [2, E]) are given, the per-expert arrivals
 * and kept rows too; either may be NULL to skip that copy.  Synchronises the
 * stream.  Returns MOE_PW_EDEVICE when a kernel flagged a violation (the
 * stats are still filled).
 */
int moe_pw_stats(const moe_pw_config *cfg, const moe_pw_counters *counters,
                 const int32_t *expert_counts, moe_pw_drop_stats *host_out,
                 int32_t *host_expert_counts, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* One step from host memory to host memory.                                 */
/* ------------------------------------------------------------------------ */

/* The device arrays of one step (caller-allocated, sizes from moe_pw_plan). */
typedef struct moe_pw_device_buffers {
    float *logits;           /* f32 [T, E] */
    uint16_t *x;             /* bf16 [T, D] */
    float *scale;            /* f32 [E] */
    int32_t *idx;            /* i32 [T, k] */
    float *gates;            /* f32 [T, k] */
    int32_t *slot_map;       /* i32 [T, k] */
    int32_t *occ;            /* i32 [occ_len] */
    uint16_t *pool_x;        /* bf16 [n_slots, D] */
    int32_t *pool_hdr;       /* i32 [n_slots] */
    int32_t *recv_row;       /* i32 [n_slots] */
    int32_t *bucket_slot;    /* i32 [bucket_len] (pooled) */
    int32_t *expert_counts;  /* i32 [2, E] */
    uint16_t *ret_x;         /* bf16 [n_slots, D] */
    int32_t *ret_hdr;        /* i32 [n_slots] */
    float *out;              /* f32 [T, D] */
    moe_pw_counters *counters;
    void *workspace;
    size_t workspace_bytes;
} moe_pw_device_buffers;

/*
 * One whole step with host buffers in and out, all of it enqueued, nothing
 * waited for: on copy_in the host inputs (logits f32 [T, E], x bf16 [T, D],
 * scale f32 [E]) go to dev; compute waits for them and runs route, dispatch,
 * the per-expert op and the combine; copy_out waits for the combine and
 * brings out (f32 [T, D] into h_out) and the counters (into *h_counters)
 * back.  The three streams may be the same stream.  For the copies to run
 * beside the kernels, the host buffers must be pinned (cudaHostAlloc /
 * cudaHostRegister) and the streams distinct; then the upload of one batch,
 * the compute of the previous one and the download of the one before can
 * overlap when the caller alternates two sets of device buffers and orders
 * each set's reuse (its inputs after the compute that read them, its output
 * after the download that read it) with events on these streams.  Returns
 * once everything is enqueued; synchronise copy_out before reading h_out.
 */
int moe_pw_step_host(const moe_pw_config *cfg, const float *h_logits, const uint16_t *h_x,
                     const float *h_scale, float *h_out, moe_pw_counters *h_counters,
                     const moe_pw_device_buffers *dev, cudaStream_t compute,
                     cudaStream_t copy_in, cudaStream_t copy_out);

/* ------------------------------------------------------------------------ */
/* Expert parallelism over several GPUs.                                     */
/* ------------------------------------------------------------------------ */

/*
 * "Marin 开始公开训练 535B 参数 MoE 模型", section 二: the experts sit on a
 * 64-GPU expert-parallel domain, and the fixed pools cross GPUs in three waves
 * of identical shape with the expert id in the payload; the huxiu article's
 * JAX section adds that the exchange should overlap the expert compute.
 *
 * Here the R logical ranks are spread over n_gpus GPUs, Rn = R / n_gpus on
 * each: GPU g holds the token shards of sources s in [g*Rn, (g+1)*Rn) (global
 * tokens [g*Rn*T_s, (g+1)*Rn*T_s), T_s = T / R) and the experts of
 * destinations d in [g*Rn, (g+1)*Rn).  Capacities are those of the whole
 * batch.  On each GPU (n_slots = Rn * R * W * C_s, the same for all three
 * pool arrays):
 *   send side   slot_map / occ / ret_x / ret_hdr use the local send slot
 *               q = ((s_loc*R + d)*W + w)*C_s + c, s_loc = s - g*Rn, i.e. the
 *               single-GPU slot ids of this GPU's sources;
 *   receive     recv_x / recv_hdr / recv_row use the receive slot
 *   side        rq = ((s*Rn + d_loc)*W + w)*C_s + c, d_loc = d - g*Rn, for all
 *               R sources s;
 *   buckets     bucket_slot [Rn*L, C_r] (receive slots) and expert_counts
 *               [2, Rn*L] cover the local experts e - g*Rn*L.
 * Every array of GPU g holds exactly the single-GPU arrays' entries for its
 * sources or its destinations, relabelled as above.
 *
 * The exchange is done by the kernels themselves, over peer memory: the pack
 * stores each kept row (TMA bulk store, no multicast) and its header straight
 * into the receive pool of the destination's GPU, and zero-fills the empty
 * pool tails there; the expert op stores each result row into the return
 * pool of the source's GPU.  The peer addresses come from a table
 * (moe_pw_ep_peers): device pointers as this GPU addresses them, from
 * cudaIpcOpenMemHandle (moe_pw_ipc_open) or, for this GPU's own entry or GPUs
 * of one process, plain device pointers.
 *
 * Order across GPUs is the caller's: every GPU's pack must be complete before
 * any GPU buckets those waves, and every expert op before any combine (a
 * stream-ordered barrier, such as a one-element NCCL all-reduce after the
 * kernels, does it).  The kernels end with a system-scope fence so that their
 * peer stores are visible once the kernel has completed.
 *
 * Waves: wave_mask (bit w = wave w; (1 << W) - 1 = all) selects the waves a
 * pack, bucket or expert call handles, so wave w can be exchanged while the
 * expert op of wave w - 1 runs.  Pooled mode only.
 *
 * Only what is read crosses GPUs: an empty send slot and a slot the receiver
 * did not keep travel as their header -1 alone; their rows in the receive
 * and return pools are left as they were (the single-GPU calls write zeros
 * there).  Every consumer skips such rows by the header.
 */
#define MOE_PW_EP_MAX_GPUS 64

typedef struct moe_pw_ep {
    int32_t n_gpus;  /* GPUs sharing the R logical ranks; R % n_gpus == 0 */
    int32_t gpu;     /* this GPU's index, 0 <= gpu < n_gpus */
} moe_pw_ep;

/* Where the kernels of this GPU write: entry h is GPU h's array, as a device
 * pointer valid on this GPU (entries >= n_gpus are ignored). */
typedef struct moe_pw_ep_peers {
    uint16_t *recv_x[MOE_PW_EP_MAX_GPUS];   /* bf16 [n_slots, D] receive pools */
    int32_t *recv_hdr[MOE_PW_EP_MAX_GPUS];  /* i32 [n_slots] their headers */
    uint16_t *ret_x[MOE_PW_EP_MAX_GPUS];    /* bf16 [n_slots, D] return pools */
    int32_t *ret_hdr[MOE_PW_EP_MAX_GPUS];   /* i32 [n_slots] their headers */
} moe_pw_ep_peers;

/* Per-GPU sizes (element counts unless "bytes"). */
typedef struct moe_pw_ep_sizes {
    int64_t tokens;          /* Rn * T_s tokens on this GPU */
    int64_t first_token;     /* global index of its first token */
    int64_t C_s, C_r;        /* capacities of the whole batch */
    int64_t n_pools;         /* Rn * R * W send pools */
    int64_t n_slots;         /* rows of every pool array on this GPU */
    int64_t local_experts;   /* Rn * L */
    int64_t bucket_len;      /* local_experts * C_r */
    int64_t workspace_bytes; /* scratch for moe_pw_ep_assign */
    int64_t total_bytes;     /* every buffer of this GPU's share */
} moe_pw_ep_sizes;

/* Host-only: validates cfg (pooled mode) and ep and fills *out; with
 * budget_bytes > 0, MOE_PW_ENOMEM when out->total_bytes exceeds it. */
int moe_pw_ep_plan(const moe_pw_config *cfg, const moe_pw_ep *ep, int64_t budget_bytes,
                   moe_pw_ep_sizes *out);

/* moe_pw_route on this GPU's tokens (logits f32 [tokens, E]). */
int moe_pw_ep_route(const moe_pw_config *cfg, const moe_pw_ep *ep, const float *logits,
                    int32_t *idx, float *gates, cudaStream_t stream);

/* moe_pw_assign for this GPU's sources: slot_map [tokens, k] receives local
 * send slots, occ [Rn, R, W] the rows kept per pool.  Zeroes *counters. */
int moe_pw_ep_assign(const moe_pw_config *cfg, const moe_pw_ep *ep, const int32_t *idx,
                     int32_t *slot_map, int32_t *occ, moe_pw_counters *counters,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Pack and send (section 二: fixed per-destination pools, expert id in the
 * payload).  For every kept (t, j) whose wave is in wave_mask, the row x[t]
 * (loaded once into shared memory) is bulk-stored into the receive pool of
 * the destination's GPU (peers->recv_x[d / Rn]) at its receive slot, with the
 * expert id as its header; the empty tails (c >= occ) of this GPU's pools of
 * those waves get header -1 there (their rows are not sent).  Uses
 * counters->work like moe_pw_pack.  x bf16 [tokens, D].
 */
int moe_pw_ep_pack(const moe_pw_config *cfg, const moe_pw_ep *ep, const moe_pw_ep_peers *peers,
                   const uint16_t *x, const int32_t *idx, const int32_t *slot_map,
                   const int32_t *occ, uint32_t wave_mask, moe_pw_counters *counters,
                   cudaStream_t stream);

/*
 * Receiver bucketing (section 二: receiver factor) over this GPU's receive
 * pool, for the waves in wave_mask: per (local destination, wave), sources
 * ascending, then slots ascending; an empty slot is recognised by its header
 * -1 alone (no counts are exchanged).  Writes recv_row, bucket_slot (receive
 * slots) and expert_counts of the local experts of those waves and adds
 * receiver drops and kept rows to *counters.
 */
int moe_pw_ep_bucket(const moe_pw_config *cfg, const moe_pw_ep *ep, const int32_t *recv_hdr,
                     int32_t *recv_row, int32_t *bucket_slot, int32_t *expert_counts,
                     uint32_t wave_mask, moe_pw_counters *counters, cudaStream_t stream);

/*
 * Per-expert op and return trip (huxiu: results come back by a second
 * all-to-all).  For every receive slot of the waves in wave_mask: if the
 * receiver kept it, bf16_rn(scale[e] * row) and header e, else header -1
 * alone, stored into the return pool of the source's GPU (peers->ret_x[s /
 * Rn]) at the source's send slot.
 */
int moe_pw_ep_expert(const moe_pw_config *cfg, const moe_pw_ep *ep, const moe_pw_ep_peers *peers,
                     const uint16_t *recv_x, const int32_t *recv_hdr, const int32_t *recv_row,
                     const float *scale, uint32_t wave_mask, cudaStream_t stream);

/* moe_pw_combine on this GPU's tokens and return pool (out f32 [tokens, D]). */
int moe_pw_ep_combine(const moe_pw_config *cfg, const moe_pw_ep *ep, const uint16_t *ret_x,
                      const int32_t *ret_hdr, const int32_t *slot_map, const float *gates,
                      float *out, moe_pw_counters *counters, cudaStream_t stream);

/* moe_pw_stats for this GPU: assignments = tokens * k; sender drops of its
 * sources; receiver drops, kept rows and expert_counts ([2, Rn*L]) of its
 * experts.  Summed over the GPUs they give the whole batch's statistics. */
int moe_pw_ep_stats(const moe_pw_config *cfg, const moe_pw_ep *ep,
                    const moe_pw_counters *counters, const int32_t *expert_counts,
                    moe_pw_drop_stats *host_out, int32_t *host_expert_counts,
                    cudaStream_t stream);

/*
 * Sharing device buffers between the processes of an expert-parallel run
 * (one process per GPU).  moe_pw_ipc_export describes the allocation that
 * holds dev_ptr (cudaIpcGetMemHandle of its base) and dev_ptr's offset in it;
 * moe_pw_ipc_open maps such a description exported by another process into
 * this one (cudaIpcOpenMemHandle with peer access enabled) and returns the
 * same byte as a pointer valid on the current device; moe_pw_ipc_close
 * unmaps it (pass the pointer open returned and the same description).  A
 * process cannot open its own handles; use the pointer itself.  Host-only,
 * synchronous.
 */
typedef struct moe_pw_ipc_handle {
    unsigned char handle[64];  /* cudaIpcMemHandle_t of the allocation */
    uint64_t offset;           /* dev_ptr - allocation base */
} moe_pw_ipc_handle;

int moe_pw_ipc_export(const void *dev_ptr, moe_pw_ipc_handle *out);
int moe_pw_ipc_open(const moe_pw_ipc_handle *h, void **dev_ptr);
int moe_pw_ipc_close(void *dev_ptr, const moe_pw_ipc_handle *h);

/*
 * Self-test of failure detection (no counterpart on the pages): launches one
 * warp that waits, with the library's bounded mbarrier wait, on a barrier
 * phase that nothing completes.  After `polls` polls the wait gives up, the
 * kernel sets MOE_PW_DEVERR_TIMEOUT in counters->error and returns, and the
 * CUDA context stays usable.  Lets a caller check that timeouts surface as a
 * status instead of a hang.
 */
int moe_pw_selftest_wait_timeout(moe_pw_counters *counters, int32_t polls, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_PW_H */
