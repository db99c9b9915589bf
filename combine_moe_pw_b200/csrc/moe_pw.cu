// moe_pw.cu - the C ABI of libmoe_pw.so: argument checks, sizes, launches.
// The kernels live in route.cu, assign.cu, pack.cu, bucket.cu, expert.cu and
// combine.cu; this file owns validation and the contract of include/moe_pw.h.
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace moe_pw {

int dev_info(DevInfo *out)
{
    static std::mutex mu;
    static DevInfo cache[64];
    static bool have[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && have[dev]) {
        *out = cache[dev];
        return 0;
    }
    DevInfo di;
    if (cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return -1;
    if (cudaDeviceGetAttribute(&di.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
        cudaSuccess)
        return -1;
    if (dev >= 0 && dev < 64) {
        cache[dev] = di;
        have[dev] = true;
    }
    *out = di;
    return 0;
}

namespace {

constexpr int64_t MAX_INT32 = 0x7FFFFFFF;

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

#ifndef MOE_PW_ASSIGN_CHUNK
#define MOE_PW_ASSIGN_CHUNK 2048
#endif

// Validate a config and derive the kernel geometry.
int make_geo(const moe_pw_config *c, Geo *g)
{
    if (!c || !g) return MOE_PW_EINVAL;
    if (c->T < 0 || c->R < 1 || c->L < 1 || c->W < 1 || c->P < 1 || c->k < 1 || c->D < 1)
        return MOE_PW_EINVAL;
    if (c->mode != MOE_PW_POOLED && c->mode != MOE_PW_RAGGED) return MOE_PW_EINVAL;
    if (int64_t(c->W) * c->P != c->L) return MOE_PW_EINVAL;
    if (int64_t(c->R) * c->L != c->E) return MOE_PW_EINVAL;
    if (c->k > c->E) return MOE_PW_EINVAL;
    if (c->T % c->R != 0) return MOE_PW_EINVAL;
    if (c->k > 32 || c->E > 2048 || c->P > 32 || int64_t(c->R) * c->W > 2048)
        return MOE_PW_EUNSUPPORTED;
    if (c->D % 8 != 0 || c->D < 8 || c->D > 12288) return MOE_PW_EUNSUPPORTED;
    if (c->T * c->k > MAX_INT32) return MOE_PW_EUNSUPPORTED;

    std::memset(g, 0, sizeof(*g));
    g->T = c->T;
    g->ep_n = 1;
    g->ep_g = 0;
    g->Rn = c->R;
    g->E = c->E;
    g->k = c->k;
    g->D = c->D;
    g->R = c->R;
    g->L = c->L;
    g->W = c->W;
    g->P = c->P;
    g->mode = c->mode;
    const int64_t T_s = c->T / c->R;
    if (c->mode == MOE_PW_POOLED) {
        g->T_s = T_s;
        const int64_t kp = c->k < c->P ? c->k : c->P;
        g->C_s = c->cf_send_pct > 0
                     ? ceil_div(int64_t(c->cf_send_pct) * T_s * c->k * c->P, int64_t(100) * c->E)
                     : T_s * kp;
        g->C_r = c->cf_recv_pct > 0
                     ? ceil_div(int64_t(c->cf_recv_pct) * c->T * c->k, int64_t(100) * c->E)
                     : c->T;
        g->n_pools = int64_t(c->R) * c->R * c->W;
        if (g->C_s > MAX_INT32 || g->C_r > MAX_INT32) return MOE_PW_EUNSUPPORTED;
        g->n_slots = g->n_pools * g->C_s;
        if (g->n_slots > MAX_INT32 || int64_t(c->E) * g->C_r > (int64_t(1) << 40))
            return MOE_PW_EUNSUPPORTED;
        g->NB = c->R * c->W;
        g->n_groups = c->R;
        g->group_tokens = T_s;
    } else {
        g->T_s = c->T;
        g->n_pools = 0;
        g->n_slots = c->T * c->k;
        g->NB = c->E;
        g->n_groups = 1;
        g->group_tokens = c->T;
    }
    // ranking chunks: MOE_PW_ASSIGN_CHUNK assignments (256 tokens at k = 8),
    // never straddling a group
    int64_t ct = MOE_PW_ASSIGN_CHUNK / c->k > 0 ? MOE_PW_ASSIGN_CHUNK / c->k : 1;
    if (g->group_tokens < ct) ct = g->group_tokens > 0 ? g->group_tokens : 1;
    g->chunk_tokens = ct;
    g->chunks_per_group = int32_t(ceil_div(g->group_tokens > 0 ? g->group_tokens : 1, ct));
    const int64_t nch = int64_t(g->n_groups) * g->chunks_per_group;
    if (nch > MAX_INT32) return MOE_PW_EUNSUPPORTED;
    g->n_chunks = int32_t(nch);
    return MOE_PW_OK;
}

// The share of GPU ep->gpu in an expert-parallel run: the single-GPU
// geometry of the whole batch (capacities included), narrowed to this GPU's
// Rn sources (its tokens, send pools and send slots) and Rn destinations.
int make_geo_ep(const moe_pw_config *c, const moe_pw_ep *ep, Geo *g)
{
    int rc = make_geo(c, g);
    if (rc != MOE_PW_OK) return rc;
    if (!ep || ep->n_gpus < 1 || ep->n_gpus > MOE_PW_EP_MAX_GPUS || ep->gpu < 0 ||
        ep->gpu >= ep->n_gpus)
        return MOE_PW_EINVAL;
    if (c->mode != MOE_PW_POOLED) return MOE_PW_EUNSUPPORTED;
    if (c->R % ep->n_gpus != 0) return MOE_PW_EINVAL;
    const int32_t Rn = c->R / ep->n_gpus;
    g->ep_n = ep->n_gpus;
    g->ep_g = ep->gpu;
    g->Rn = Rn;
    g->T = int64_t(Rn) * g->T_s;
    g->n_groups = Rn;
    g->n_pools = int64_t(Rn) * c->R * c->W;
    g->n_slots = g->n_pools * g->C_s;
    g->n_chunks = Rn * g->chunks_per_group;
    return MOE_PW_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MOE_PW_OK : MOE_PW_ECUDA; }

}  // namespace
}  // namespace moe_pw

using namespace moe_pw;

extern "C" {

int moe_pw_version(void) { return 10000; }

const char *moe_pw_strerror(int code)
{
    switch (code) {
    case MOE_PW_OK: return "ok";
    case MOE_PW_EINVAL: return "invalid argument or config";
    case MOE_PW_EUNSUPPORTED: return "shape or alignment not supported by this library";
    case MOE_PW_ECUDA: return "CUDA runtime or launch error";
    case MOE_PW_EDEVICE: return "a kernel flagged a violation (see counters.error)";
    case MOE_PW_ENOMEM: return "buffers exceed the memory budget or the built-in scratch limit";
    default: return "unknown error code";
    }
}

int moe_pw_plan(const moe_pw_config *cfg, int64_t budget_bytes, moe_pw_sizes *out)
{
    if (!out) return MOE_PW_EINVAL;
    Geo g;
    const int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    std::memset(out, 0, sizeof(*out));
    const int64_t T = g.T, E = g.E, k = g.k, D = g.D;
    out->C_s = g.mode == MOE_PW_POOLED ? g.C_s : 0;
    out->C_r = g.mode == MOE_PW_POOLED ? g.C_r : 0;
    out->n_pools = g.n_pools;
    out->n_slots = g.n_slots;
    out->occ_len = g.mode == MOE_PW_POOLED ? g.n_pools : E + 1;
    out->bucket_len = g.mode == MOE_PW_POOLED ? E * g.C_r : 0;
    out->workspace_bytes = ws_bytes(g);
    const int64_t S = g.n_slots;
    out->total_bytes = 4 * T * E          // logits
                       + 8 * T * k        // idx, gates
                       + 2 * T * D        // x
                       + 4 * T * k        // slot_map
                       + 4 * out->occ_len //
                       + 2 * (2 * S * D)  // pool_x, ret_x
                       + 3 * (4 * S)      // pool_hdr, recv_row, ret_hdr
                       + 4 * out->bucket_len + 8 * E + 4 * E  // buckets, expert_counts, scale
                       + 4 * T * D        // out
                       + int64_t(sizeof(moe_pw_counters)) + out->workspace_bytes;
    if (budget_bytes > 0 && out->total_bytes > budget_bytes) return MOE_PW_ENOMEM;
    return MOE_PW_OK;
}

int moe_pw_route(const moe_pw_config *cfg, const float *logits, int32_t *idx, float *gates,
                 cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.E % 4 != 0) return MOE_PW_EUNSUPPORTED;
    if (g.T == 0) return MOE_PW_OK;
    if (!logits || !idx || !gates) return MOE_PW_EINVAL;
    if (!aligned(logits, 16) || !aligned(idx, 4) || !aligned(gates, 4)) return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_route(g, logits, idx, gates, stream));
}

int moe_pw_assign(const moe_pw_config *cfg, const int32_t *idx, int32_t *slot_map, int32_t *occ,
                  moe_pw_counters *counters, void *workspace, size_t workspace_bytes,
                  cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!counters || !occ) return MOE_PW_EINVAL;
    if (g.T > 0 && (!idx || !slot_map || !workspace)) return MOE_PW_EINVAL;
    if (g.T > 0 && int64_t(workspace_bytes) < ws_bytes(g)) return MOE_PW_EINVAL;
    if (!aligned(counters, 8) || !aligned(occ, 4) || (g.T > 0 && (!aligned(idx, 4) ||
        !aligned(slot_map, 4) || !aligned(workspace, 256))))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_assign(g, idx, slot_map, occ, counters, workspace, stream));
}

int moe_pw_pack(const moe_pw_config *cfg, const uint16_t *x, const int32_t *idx,
                const int32_t *slot_map, const int32_t *occ, uint16_t *pool_x, int32_t *pool_hdr,
                moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.n_slots == 0) return MOE_PW_OK;
    if (!x || !idx || !slot_map || !occ || !pool_x || !pool_hdr || !counters) return MOE_PW_EINVAL;
    if (!aligned(x, 16) || !aligned(pool_x, 16) || !aligned(idx, 4) || !aligned(slot_map, 4) ||
        !aligned(occ, 4) || !aligned(pool_hdr, 4) || !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_pack(g, x, idx, slot_map, occ, pool_x, pool_hdr, counters, stream));
}

int moe_pw_bucket(const moe_pw_config *cfg, const int32_t *pool_hdr, const int32_t *occ,
                  int32_t *recv_row, int32_t *bucket_slot, int32_t *expert_counts,
                  moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!counters || !expert_counts) return MOE_PW_EINVAL;
    if (g.T > 0) {
        if (!pool_hdr || !occ || !recv_row) return MOE_PW_EINVAL;
        if (g.mode == MOE_PW_POOLED && !bucket_slot) return MOE_PW_EINVAL;
    }
    if (!aligned(counters, 8) || !aligned(expert_counts, 4)) return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_bucket(g, pool_hdr, occ, recv_row, bucket_slot, expert_counts, counters,
                                 stream));
}

int moe_pw_assign_headers(const moe_pw_config *cfg, const int32_t *idx, int32_t *slot_map,
                          int32_t *occ, int32_t *pool_hdr, moe_pw_counters *counters,
                          void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.mode != MOE_PW_POOLED) return MOE_PW_EUNSUPPORTED;
    if (!counters || !occ) return MOE_PW_EINVAL;
    if (g.T > 0 && (!idx || !slot_map || !workspace || !pool_hdr)) return MOE_PW_EINVAL;
    if (g.T > 0 && int64_t(workspace_bytes) < ws_bytes(g)) return MOE_PW_EINVAL;
    if (!aligned(counters, 8) || !aligned(occ, 4) || (g.T > 0 && (!aligned(idx, 4) ||
        !aligned(slot_map, 4) || !aligned(pool_hdr, 4) || !aligned(workspace, 256))))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_assign(g, idx, slot_map, occ, counters, workspace, stream, pool_hdr));
}

int moe_pw_route_assign_form(const moe_pw_config *cfg, int32_t form, const float *logits,
                             int32_t *idx, float *gates, int32_t *slot_map, int32_t *occ,
                             int32_t *pool_hdr, moe_pw_counters *counters, void *workspace,
                             size_t workspace_bytes, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.mode != MOE_PW_POOLED || g.E % 4 != 0) return MOE_PW_EUNSUPPORTED;
    if (form < -1 || form > MOE_PW_RA_CLUSTER) return MOE_PW_EINVAL;
    if (!counters || !occ) return MOE_PW_EINVAL;
    if (g.T > 0 && (!logits || !idx || !gates || !slot_map || !pool_hdr || !workspace))
        return MOE_PW_EINVAL;
    if (g.T > 0 && int64_t(workspace_bytes) < ws_bytes(g)) return MOE_PW_EINVAL;
    if (!aligned(counters, 8) || !aligned(occ, 4) ||
        (g.T > 0 && (!aligned(logits, 16) || !aligned(idx, 4) || !aligned(gates, 4) ||
                     !aligned(slot_map, 4) || !aligned(pool_hdr, 4) ||
                     !aligned(workspace, 256))))
        return MOE_PW_EUNSUPPORTED;
    if (g.T > 0 && form != MOE_PW_RA_SEPARATE) {
        const cudaError_t e = launch_route_assign(g, logits, idx, gates, slot_map, occ, pool_hdr,
                                                  counters, stream, form);
        if (e == cudaErrorInvalidValue) return MOE_PW_EUNSUPPORTED;  // the form does not fit
        if (e != cudaErrorNotSupported) return cuda_rc(e);
    }
    rc = moe_pw_route(cfg, logits, idx, gates, stream);
    if (rc != MOE_PW_OK) return rc;
    return moe_pw_assign_headers(cfg, idx, slot_map, occ, pool_hdr, counters, workspace,
                                 workspace_bytes, stream);
}

int moe_pw_route_assign(const moe_pw_config *cfg, const float *logits, int32_t *idx,
                        float *gates, int32_t *slot_map, int32_t *occ, int32_t *pool_hdr,
                        moe_pw_counters *counters, void *workspace, size_t workspace_bytes,
                        cudaStream_t stream)
{
    return moe_pw_route_assign_form(cfg, -1, logits, idx, gates, slot_map, occ, pool_hdr,
                                    counters, workspace, workspace_bytes, stream);
}

int moe_pw_route_assign_plan(const moe_pw_config *cfg, int32_t *form)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!form) return MOE_PW_EINVAL;
    int f = MOE_PW_RA_SEPARATE;
    const cudaError_t e = route_assign_plan(g, &f);
    *form = f;
    return cuda_rc(e);
}

int moe_pw_pack_bucket(const moe_pw_config *cfg, const uint16_t *x, const int32_t *idx,
                       const int32_t *slot_map, const int32_t *occ, uint16_t *pool_x,
                       int32_t *pool_hdr, int32_t *recv_row, int32_t *bucket_slot,
                       int32_t *expert_counts, moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.mode != MOE_PW_POOLED) return MOE_PW_EUNSUPPORTED;
    if (g.T == 0) {
        rc = moe_pw_pack(cfg, x, idx, slot_map, occ, pool_x, pool_hdr, counters, stream);
        if (rc != MOE_PW_OK) return rc;
        return moe_pw_bucket(cfg, pool_hdr, occ, recv_row, bucket_slot, expert_counts, counters,
                             stream);
    }
    if (!x || !idx || !slot_map || !occ || !pool_x || !pool_hdr || !recv_row || !bucket_slot ||
        !expert_counts || !counters)
        return MOE_PW_EINVAL;
    if (!aligned(x, 16) || !aligned(pool_x, 16) || !aligned(idx, 4) || !aligned(slot_map, 4) ||
        !aligned(occ, 4) || !aligned(pool_hdr, 4) || !aligned(recv_row, 4) ||
        !aligned(bucket_slot, 4) || !aligned(expert_counts, 4) || !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_pack_bucket(g, x, idx, slot_map, occ, pool_x, pool_hdr, recv_row,
                                      bucket_slot, expert_counts, counters, stream));
}

int moe_pw_dispatch(const moe_pw_config *cfg, const uint16_t *x, const int32_t *idx,
                    int32_t *slot_map, int32_t *occ, uint16_t *pool_x, int32_t *pool_hdr,
                    int32_t *recv_row, int32_t *bucket_slot, int32_t *expert_counts,
                    moe_pw_counters *counters, void *workspace, size_t workspace_bytes,
                    cudaStream_t stream)
{
    if (cfg && cfg->mode == MOE_PW_POOLED) {
        // the bucketing runs beside the row copies (same outputs)
        int rc = moe_pw_assign_headers(cfg, idx, slot_map, occ, pool_hdr, counters, workspace,
                                       workspace_bytes, stream);
        if (rc != MOE_PW_OK) return rc;
        return moe_pw_pack_bucket(cfg, x, idx, slot_map, occ, pool_x, pool_hdr, recv_row,
                                  bucket_slot, expert_counts, counters, stream);
    }
    int rc = moe_pw_assign(cfg, idx, slot_map, occ, counters, workspace, workspace_bytes, stream);
    if (rc != MOE_PW_OK) return rc;
    rc = moe_pw_pack(cfg, x, idx, slot_map, occ, pool_x, pool_hdr, counters, stream);
    if (rc != MOE_PW_OK) return rc;
    return moe_pw_bucket(cfg, pool_hdr, occ, recv_row, bucket_slot, expert_counts, counters,
                         stream);
}

int moe_pw_expert(const moe_pw_config *cfg, const uint16_t *pool_x, const int32_t *pool_hdr,
                  const int32_t *recv_row, const float *scale, uint16_t *ret_x, int32_t *ret_hdr,
                  moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.n_slots == 0) return MOE_PW_OK;
    if (!pool_x || !pool_hdr || !recv_row || !scale || !ret_x || !ret_hdr || !counters)
        return MOE_PW_EINVAL;
    if (!aligned(pool_x, 16) || !aligned(ret_x, 16) || !aligned(pool_hdr, 4) ||
        !aligned(recv_row, 4) || !aligned(scale, 4) || !aligned(ret_hdr, 4) ||
        !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_expert(g, pool_x, pool_hdr, recv_row, scale, ret_x, ret_hdr, counters,
                                 stream));
}

int moe_pw_combine(const moe_pw_config *cfg, const uint16_t *ret_x, const int32_t *ret_hdr,
                   const int32_t *slot_map, const float *gates, float *out,
                   moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.T == 0) return MOE_PW_OK;
    if (!ret_x || !ret_hdr || !slot_map || !gates || !out || !counters) return MOE_PW_EINVAL;
    if (!aligned(ret_x, 16) || !aligned(out, 16) || !aligned(ret_hdr, 4) ||
        !aligned(slot_map, 4) || !aligned(gates, 4) || !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_combine(g, ret_x, ret_hdr, slot_map, gates, out, counters, stream));
}

int moe_pw_combine_bf16(const moe_pw_config *cfg, const uint16_t *ret_x, const int32_t *ret_hdr,
                        const int32_t *slot_map, const float *gates, uint16_t *out,
                        moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.T == 0) return MOE_PW_OK;
    if (!ret_x || !ret_hdr || !slot_map || !gates || !out || !counters) return MOE_PW_EINVAL;
    if (!aligned(ret_x, 16) || !aligned(out, 16) || !aligned(ret_hdr, 4) ||
        !aligned(slot_map, 4) || !aligned(gates, 4) || !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_combine_bf16(g, ret_x, ret_hdr, slot_map, gates, out, counters, stream));
}

int moe_pw_combine_bf16_rows(const moe_pw_config *cfg, const uint16_t *ret_x,
                             const int32_t *ret_hdr, const int32_t *slot_map, const float *gates,
                             int64_t first_token, int64_t n_tokens, uint16_t *out,
                             moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (first_token < 0 || n_tokens < 0 || first_token + n_tokens > g.T) return MOE_PW_EINVAL;
    if (n_tokens == 0) return MOE_PW_OK;
    if (!ret_x || !ret_hdr || !slot_map || !gates || !out || !counters) return MOE_PW_EINVAL;
    if (!aligned(ret_x, 16) || !aligned(out, 16) || !aligned(ret_hdr, 4) ||
        !aligned(slot_map, 4) || !aligned(gates, 4) || !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    // the same kernel on the token range: the pool (and its slot ids) is the
    // whole batch's, only the tokens are narrowed
    Geo rows = g;
    rows.T = n_tokens;
    return cuda_rc(launch_combine_bf16(rows, ret_x, ret_hdr, slot_map + first_token * g.k,
                                       gates + first_token * g.k, out, counters, stream));
}

int moe_pw_combine_backward(const moe_pw_config *cfg, const float *dout, const uint16_t *ret_x,
                            const int32_t *ret_hdr, const int32_t *slot_map, const int32_t *idx,
                            const float *gates, uint16_t *d_ret, float *dgates, float *dlogits,
                            moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.T == 0 && g.n_slots == 0) return MOE_PW_OK;
    if (!ret_hdr || !d_ret || !counters) return MOE_PW_EINVAL;
    if (g.T > 0 && (!dout || !ret_x || !slot_map || !idx || !gates)) return MOE_PW_EINVAL;
    if (!aligned(d_ret, 16) || !aligned(ret_hdr, 4) || !aligned(counters, 8) ||
        (g.T > 0 && (!aligned(dout, 16) || !aligned(ret_x, 16) || !aligned(slot_map, 4) ||
                     !aligned(idx, 4) || !aligned(gates, 4))) ||
        (dgates && !aligned(dgates, 4)) || (dlogits && !aligned(dlogits, 4)))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_combine_backward(g, dout, ret_x, ret_hdr, slot_map, idx, gates, d_ret,
                                           dgates, dlogits, counters, stream));
}

int moe_pw_dispatch_backward(const moe_pw_config *cfg, const uint16_t *d_pool,
                             const int32_t *recv_row, const int32_t *slot_map, float *dx,
                             moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.T == 0) return MOE_PW_OK;
    if (!d_pool || !recv_row || !slot_map || !dx || !counters) return MOE_PW_EINVAL;
    if (!aligned(d_pool, 16) || !aligned(dx, 16) || !aligned(recv_row, 4) ||
        !aligned(slot_map, 4) || !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    // the combine kernel with unit gates; recv_row >= 0 marks the slots whose
    // gradient rows are live (the others were zeroed by the expert backward)
    return cuda_rc(launch_combine(g, d_pool, recv_row, slot_map, nullptr, dx, counters, stream));
}

int moe_pw_project(const uint16_t *A, const uint16_t *Bt, uint16_t *C, int64_t M, int32_t N,
                   int32_t K, moe_pw_counters *counters, cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 1 || M > MAX_INT32) return MOE_PW_EINVAL;
    if (M == 0 || N == 0) return MOE_PW_OK;
    if (!A || !Bt || !C || !counters) return MOE_PW_EINVAL;
    if (K % 8 != 0 || N % 8 != 0) return MOE_PW_EUNSUPPORTED;
    if (!aligned(A, 16) || !aligned(Bt, 16) || !aligned(C, 16) || !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_gemm(A, Bt, M, N, K, 0, C, N, nullptr, nullptr, 0, nullptr, nullptr, 0,
                               counters, stream));
}

int moe_pw_project_add(const uint16_t *A, const uint16_t *Bt, const uint16_t *add, uint16_t *C,
                       int64_t M, int32_t N, int32_t K, moe_pw_counters *counters,
                       cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 1 || M > MAX_INT32) return MOE_PW_EINVAL;
    if (M == 0 || N == 0) return MOE_PW_OK;
    if (!A || !Bt || !add || !C || !counters) return MOE_PW_EINVAL;
    if (K % 8 != 0 || N % 8 != 0) return MOE_PW_EUNSUPPORTED;
    if (!aligned(A, 16) || !aligned(Bt, 16) || !aligned(add, 16) || !aligned(C, 16) ||
        !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_gemm(A, Bt, M, N, K, 0, C, N, nullptr, nullptr, 0, nullptr, nullptr, 0,
                               counters, stream, add));
}

int moe_pw_project_pack(const moe_pw_config *cfg, const uint16_t *h, const uint16_t *w_down_t,
                        int32_t model_width, const int32_t *idx, const int32_t *slot_map,
                        const int32_t *occ, uint16_t *pool_x, int32_t *pool_hdr,
                        moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (model_width < 8 || model_width % 8 != 0) return MOE_PW_EUNSUPPORTED;
    if (g.n_slots == 0) return MOE_PW_OK;
    if (!h || !w_down_t || !idx || !slot_map || !occ || !pool_x || !pool_hdr || !counters)
        return MOE_PW_EINVAL;
    if (!aligned(h, 16) || !aligned(w_down_t, 16) || !aligned(pool_x, 16) || !aligned(idx, 4) ||
        !aligned(slot_map, 4) || !aligned(occ, 4) || !aligned(pool_hdr, 4) ||
        !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    // rows of the kept slots straight from the GEMM epilogue ...
    cudaError_t e = launch_gemm(h, w_down_t, g.T, g.D, model_width, 1, nullptr, 0, slot_map, idx,
                                g.k, pool_x, pool_hdr, g.n_slots, counters, stream);
    if (e != cudaSuccess) return MOE_PW_ECUDA;
    // ... and the empty pool tails zero-filled by the pack kernel's second phase
    if (g.mode == MOE_PW_POOLED) {
        Geo tails = g;
        tails.T = 0;
        e = launch_pack(tails, nullptr, idx, slot_map, occ, pool_x, pool_hdr, counters, stream);
    }
    return cuda_rc(e);
}

int moe_pw_seq_balance_plan(const moe_pw_config *cfg, int64_t seq_len, int64_t *workspace_bytes)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!workspace_bytes || seq_len < 1 || g.T % seq_len != 0) return MOE_PW_EINVAL;
    *workspace_bytes = balance_ws_bytes(g.T, seq_len, g.E);
    return MOE_PW_OK;
}

int moe_pw_seq_balance(const moe_pw_config *cfg, int64_t seq_len, float alpha,
                       const float *logits, const int32_t *idx, float *f, float *P, float *loss,
                       float *dlogits, int32_t accumulate, void *workspace,
                       size_t workspace_bytes, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (seq_len < 1 || g.T % seq_len != 0) return MOE_PW_EINVAL;
    if (g.E % 4 != 0) return MOE_PW_EUNSUPPORTED;
    if (g.T == 0) return MOE_PW_OK;
    if (!logits || !idx || !f || !P || !loss || !workspace) return MOE_PW_EINVAL;
    if (int64_t(workspace_bytes) < balance_ws_bytes(g.T, seq_len, g.E)) return MOE_PW_EINVAL;
    if (!aligned(logits, 16) || !aligned(idx, 4) || !aligned(f, 16) || !aligned(P, 4) ||
        !aligned(loss, 4) || !aligned(workspace, 256) || (dlogits && !aligned(dlogits, 16)))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_balance(g, seq_len, alpha, logits, idx, f, P, loss, dlogits, accumulate,
                                  workspace, stream));
}

int moe_pw_stats(const moe_pw_config *cfg, const moe_pw_counters *counters,
                 const int32_t *expert_counts, moe_pw_drop_stats *host_out,
                 int32_t *host_expert_counts, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!counters || !host_out) return MOE_PW_EINVAL;
    moe_pw_counters c;
    if (cudaMemcpyAsync(&c, counters, sizeof(c), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return MOE_PW_ECUDA;
    if (expert_counts && host_expert_counts &&
        cudaMemcpyAsync(host_expert_counts, expert_counts, sizeof(int32_t) * 2 * size_t(g.E),
                        cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return MOE_PW_ECUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_PW_ECUDA;
    host_out->assignments = g.T * g.k;
    host_out->kept = int64_t(c.kept);
    host_out->sender_dropped = int64_t(c.sender_dropped);
    host_out->receiver_dropped = int64_t(c.receiver_dropped);
    host_out->max_occ = c.max_occ;
    host_out->max_fill = c.max_fill;
    host_out->error = c.error;
    host_out->reserved = 0;
    return c.error != 0 ? MOE_PW_EDEVICE : MOE_PW_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of moe_pw_assign.
//
// Some callers cannot hand this library a workspace: a plugin whose host
// process owns all device memory and exposes no allocator to it, or a
// latency-critical loop that must never call cudaMalloc/cudaFree (both can
// synchronise the whole device).  For them, moe_pw_assign_noalloc keeps the
// ranking scratch in a fixed array compiled into the library instead.
// ---------------------------------------------------------------------------

namespace moe_pw {
namespace {

// Fixed scratch of the allocation-free assign: 4 MiB on every device that
// loads this library, held until the process exits.
constexpr size_t NOALLOC_SCRATCH_BYTES = MOE_PW_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current device's context.  In
// host code the symbol's name is only a host-side handle, so the address is
// looked up (cudaGetSymbolAddress, with the target device current) on every
// call rather than cached: a cached address would outlive a cudaDeviceReset
// or belong to another context made current on the same device.  The lookup
// allocates nothing; the first one on a device also loads this library's
// device code there.
int noalloc_scratch(void **out)
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MOE_PW_ECUDA;
    *out = p;
    return MOE_PW_OK;
}

}  // namespace
}  // namespace moe_pw

extern "C" int moe_pw_assign_noalloc(const moe_pw_config *cfg, const int32_t *idx,
                                     int32_t *slot_map, int32_t *occ, moe_pw_counters *counters,
                                     cudaStream_t stream)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!counters || !occ) return MOE_PW_EINVAL;
    if (g.T > 0 && (!idx || !slot_map)) return MOE_PW_EINVAL;
    if (ws_bytes(g) > int64_t(NOALLOC_SCRATCH_BYTES)) return MOE_PW_ENOMEM;
    if (!aligned(counters, 8) || !aligned(occ, 4) ||
        (g.T > 0 && (!aligned(idx, 4) || !aligned(slot_map, 4))))
        return MOE_PW_EUNSUPPORTED;
    void *scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch)) != MOE_PW_OK) return rc;
    return cuda_rc(launch_assign(g, idx, slot_map, occ, counters, scratch, stream));
}

// ---------------------------------------------------------------------------
// Self-test of the bounded wait every mbarrier wait in this library uses.
// ---------------------------------------------------------------------------

namespace moe_pw {
namespace {

// One warp waits on a phase of an mbarrier that nothing ever completes; the
// wait gives up after `polls` polls and the kernel records the timeout.
__global__ void selftest_wait_kernel(moe_pw_counters *ctr, uint32_t polls)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) mbar_init(&bar, 1);
    fence_init_and_proxy();
    __syncwarp();
    const bool done = mbar_wait_bounded(&bar, 0u, polls);
    if (!__all_sync(FULL_MASK, done) && threadIdx.x == 0) set_error(ctr, MOE_PW_DEVERR_TIMEOUT);
}

}  // namespace
}  // namespace moe_pw

extern "C" int moe_pw_selftest_wait_timeout(moe_pw_counters *counters, int32_t polls,
                                            cudaStream_t stream)
{
    if (!counters || polls < 1) return MOE_PW_EINVAL;
    if (!aligned(counters, 8)) return MOE_PW_EUNSUPPORTED;
    selftest_wait_kernel<<<1, 32, 0, stream>>>(counters, uint32_t(polls));
    return cuda_rc(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// One step from host memory to host memory.
// ---------------------------------------------------------------------------

namespace moe_pw {
namespace {

// Make `waiter` wait for the work enqueued so far on `signaller` (a one-shot
// event, released as soon as it is recorded: CUDA keeps it alive until the
// wait is resolved).  Nothing to do when the two are the same stream.
cudaError_t order(cudaStream_t signaller, cudaStream_t waiter)
{
    if (signaller == waiter) return cudaSuccess;
    cudaEvent_t ev;
    cudaError_t e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
    e = cudaEventRecord(ev, signaller);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(waiter, ev, 0);
    const cudaError_t d = cudaEventDestroy(ev);
    return e != cudaSuccess ? e : d;
}

}  // namespace
}  // namespace moe_pw

extern "C" int moe_pw_step_host(const moe_pw_config *cfg, const float *h_logits,
                                const uint16_t *h_x, const float *h_scale, float *h_out,
                                moe_pw_counters *h_counters, const moe_pw_device_buffers *dev,
                                cudaStream_t compute, cudaStream_t copy_in,
                                cudaStream_t copy_out)
{
    Geo g;
    int rc = make_geo(cfg, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!dev || !h_scale || !h_counters || !dev->scale || !dev->counters) return MOE_PW_EINVAL;
    if (g.T > 0 && (!h_logits || !h_x || !h_out || !dev->logits || !dev->x || !dev->out))
        return MOE_PW_EINVAL;
    const size_t T = size_t(g.T), E = size_t(g.E), D = size_t(g.D);
    // inputs up
    if (T > 0) {
        if (cudaMemcpyAsync(dev->logits, h_logits, 4 * T * E, cudaMemcpyHostToDevice, copy_in) !=
                cudaSuccess ||
            cudaMemcpyAsync(dev->x, h_x, 2 * T * D, cudaMemcpyHostToDevice, copy_in) !=
                cudaSuccess)
            return MOE_PW_ECUDA;
    }
    if (cudaMemcpyAsync(dev->scale, h_scale, 4 * E, cudaMemcpyHostToDevice, copy_in) !=
        cudaSuccess)
        return MOE_PW_ECUDA;
    if (order(copy_in, compute) != cudaSuccess) return MOE_PW_ECUDA;
    // the path, every step in this library's kernels
    if (g.mode == MOE_PW_POOLED) {
        if ((rc = moe_pw_route_assign(cfg, dev->logits, dev->idx, dev->gates, dev->slot_map,
                                      dev->occ, dev->pool_hdr, dev->counters, dev->workspace,
                                      dev->workspace_bytes, compute)) != MOE_PW_OK)
            return rc;
        if ((rc = moe_pw_pack_bucket(cfg, dev->x, dev->idx, dev->slot_map, dev->occ, dev->pool_x,
                                     dev->pool_hdr, dev->recv_row, dev->bucket_slot,
                                     dev->expert_counts, dev->counters, compute)) != MOE_PW_OK)
            return rc;
    } else {
        if ((rc = moe_pw_route(cfg, dev->logits, dev->idx, dev->gates, compute)) != MOE_PW_OK)
            return rc;
        if ((rc = moe_pw_dispatch(cfg, dev->x, dev->idx, dev->slot_map, dev->occ, dev->pool_x,
                                  dev->pool_hdr, dev->recv_row, dev->bucket_slot,
                                  dev->expert_counts, dev->counters, dev->workspace,
                                  dev->workspace_bytes, compute)) != MOE_PW_OK)
            return rc;
    }
    if ((rc = moe_pw_expert(cfg, dev->pool_x, dev->pool_hdr, dev->recv_row, dev->scale,
                            dev->ret_x, dev->ret_hdr, dev->counters, compute)) != MOE_PW_OK)
        return rc;
    if ((rc = moe_pw_combine(cfg, dev->ret_x, dev->ret_hdr, dev->slot_map, dev->gates, dev->out,
                             dev->counters, compute)) != MOE_PW_OK)
        return rc;
    // result down
    if (order(compute, copy_out) != cudaSuccess) return MOE_PW_ECUDA;
    if (T > 0 &&
        cudaMemcpyAsync(h_out, dev->out, 4 * T * D, cudaMemcpyDeviceToHost, copy_out) != cudaSuccess)
        return MOE_PW_ECUDA;
    if (cudaMemcpyAsync(h_counters, dev->counters, sizeof(moe_pw_counters), cudaMemcpyDeviceToHost,
                        copy_out) != cudaSuccess)
        return MOE_PW_ECUDA;
    return MOE_PW_OK;
}

// ---------------------------------------------------------------------------
// Expert parallelism over several GPUs: the same kernels on each GPU's share,
// with the pack and the expert op storing into peer GPUs' pools.
// ---------------------------------------------------------------------------

namespace moe_pw {
namespace {

// Copy the receive (or return) column of the caller's peer table; every entry
// of the run's GPUs must be set and aligned.
int ep_rows(const Geo &g, uint16_t *const *x, int32_t *const *hdr, EpRows *out)
{
    std::memset(out, 0, sizeof(*out));
    for (int h = 0; h < g.ep_n; ++h) {
        if (!x[h] || !hdr[h]) return MOE_PW_EINVAL;
        if (!aligned(x[h], 16) || !aligned(hdr[h], 4)) return MOE_PW_EUNSUPPORTED;
        out->x[h] = x[h];
        out->hdr[h] = hdr[h];
    }
    return MOE_PW_OK;
}

uint32_t wave_bits(const Geo &g, uint32_t mask) { return mask & ((1u << g.W) - 1u); }

}  // namespace
}  // namespace moe_pw

extern "C" {

int moe_pw_ep_plan(const moe_pw_config *cfg, const moe_pw_ep *ep, int64_t budget_bytes,
                   moe_pw_ep_sizes *out)
{
    if (!out) return MOE_PW_EINVAL;
    Geo g;
    const int rc = make_geo_ep(cfg, ep, &g);
    if (rc != MOE_PW_OK) return rc;
    std::memset(out, 0, sizeof(*out));
    const int64_t T = g.T, E = g.E, k = g.k, D = g.D, S = g.n_slots;
    const int64_t El = int64_t(g.Rn) * g.L;
    out->tokens = T;
    out->first_token = int64_t(g.ep_g) * T;
    out->C_s = g.C_s;
    out->C_r = g.C_r;
    out->n_pools = g.n_pools;
    out->n_slots = S;
    out->local_experts = El;
    out->bucket_len = El * g.C_r;
    out->workspace_bytes = ws_bytes(g);
    out->total_bytes = 4 * T * E + 8 * T * k + 2 * T * D + 4 * T * k  // logits .. slot_map
                       + 4 * g.n_pools                                 // occ
                       + 2 * (2 * S * D) + 3 * (4 * S) + 4 * S         // recv / ret pools + headers
                       + 4 * out->bucket_len + 8 * El + 4 * E           // buckets, counts, scale
                       + 4 * T * D                                      // out
                       + int64_t(sizeof(moe_pw_counters)) + out->workspace_bytes;
    if (budget_bytes > 0 && out->total_bytes > budget_bytes) return MOE_PW_ENOMEM;
    return MOE_PW_OK;
}

int moe_pw_ep_route(const moe_pw_config *cfg, const moe_pw_ep *ep, const float *logits,
                    int32_t *idx, float *gates, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo_ep(cfg, ep, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.E % 4 != 0) return MOE_PW_EUNSUPPORTED;
    if (g.T == 0) return MOE_PW_OK;
    if (!logits || !idx || !gates) return MOE_PW_EINVAL;
    if (!aligned(logits, 16) || !aligned(idx, 4) || !aligned(gates, 4)) return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_route(g, logits, idx, gates, stream));
}

int moe_pw_ep_assign(const moe_pw_config *cfg, const moe_pw_ep *ep, const int32_t *idx,
                     int32_t *slot_map, int32_t *occ, moe_pw_counters *counters,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo_ep(cfg, ep, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!counters || !occ) return MOE_PW_EINVAL;
    if (g.T > 0 && (!idx || !slot_map || !workspace)) return MOE_PW_EINVAL;
    if (g.T > 0 && int64_t(workspace_bytes) < ws_bytes(g)) return MOE_PW_EINVAL;
    if (!aligned(counters, 8) || !aligned(occ, 4) || (g.T > 0 && (!aligned(idx, 4) ||
        !aligned(slot_map, 4) || !aligned(workspace, 256))))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_assign(g, idx, slot_map, occ, counters, workspace, stream));
}

int moe_pw_ep_pack(const moe_pw_config *cfg, const moe_pw_ep *ep, const moe_pw_ep_peers *peers,
                   const uint16_t *x, const int32_t *idx, const int32_t *slot_map,
                   const int32_t *occ, uint32_t wave_mask, moe_pw_counters *counters,
                   cudaStream_t stream)
{
    Geo g;
    int rc = make_geo_ep(cfg, ep, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!peers) return MOE_PW_EINVAL;
    if (g.n_slots == 0 || wave_bits(g, wave_mask) == 0) return MOE_PW_OK;
    if (!x || !idx || !slot_map || !occ || !counters) return MOE_PW_EINVAL;
    if (!aligned(x, 16) || !aligned(idx, 4) || !aligned(slot_map, 4) || !aligned(occ, 4) ||
        !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    EpRows rows;
    if ((rc = ep_rows(g, peers->recv_x, peers->recv_hdr, &rows)) != MOE_PW_OK) return rc;
    return cuda_rc(launch_pack(g, x, idx, slot_map, occ, nullptr, nullptr, counters, stream,
                               &rows, wave_bits(g, wave_mask)));
}

int moe_pw_ep_bucket(const moe_pw_config *cfg, const moe_pw_ep *ep, const int32_t *recv_hdr,
                     int32_t *recv_row, int32_t *bucket_slot, int32_t *expert_counts,
                     uint32_t wave_mask, moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo_ep(cfg, ep, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!counters || !expert_counts) return MOE_PW_EINVAL;
    if (g.n_slots > 0 && (!recv_hdr || !recv_row || !bucket_slot)) return MOE_PW_EINVAL;
    if (!aligned(counters, 8) || !aligned(expert_counts, 4) || !aligned(recv_hdr, 4) ||
        !aligned(recv_row, 4) || !aligned(bucket_slot, 4))
        return MOE_PW_EUNSUPPORTED;
    if (wave_bits(g, wave_mask) == 0) return MOE_PW_OK;
    return cuda_rc(launch_bucket(g, recv_hdr, nullptr, recv_row, bucket_slot, expert_counts,
                                 counters, stream, wave_bits(g, wave_mask)));
}

int moe_pw_ep_expert(const moe_pw_config *cfg, const moe_pw_ep *ep, const moe_pw_ep_peers *peers,
                     const uint16_t *recv_x, const int32_t *recv_hdr, const int32_t *recv_row,
                     const float *scale, uint32_t wave_mask, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo_ep(cfg, ep, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!peers) return MOE_PW_EINVAL;
    if (g.n_slots == 0 || wave_bits(g, wave_mask) == 0) return MOE_PW_OK;
    if (!recv_x || !recv_hdr || !recv_row || !scale) return MOE_PW_EINVAL;
    if (!aligned(recv_x, 16) || !aligned(recv_hdr, 4) || !aligned(recv_row, 4) ||
        !aligned(scale, 4))
        return MOE_PW_EUNSUPPORTED;
    EpRows rows;
    if ((rc = ep_rows(g, peers->ret_x, peers->ret_hdr, &rows)) != MOE_PW_OK) return rc;
    return cuda_rc(launch_expert(g, recv_x, recv_hdr, recv_row, scale, nullptr, nullptr, nullptr,
                                 stream,
                                 &rows, wave_bits(g, wave_mask)));
}

int moe_pw_ep_combine(const moe_pw_config *cfg, const moe_pw_ep *ep, const uint16_t *ret_x,
                      const int32_t *ret_hdr, const int32_t *slot_map, const float *gates,
                      float *out, moe_pw_counters *counters, cudaStream_t stream)
{
    Geo g;
    int rc = make_geo_ep(cfg, ep, &g);
    if (rc != MOE_PW_OK) return rc;
    if (g.T == 0) return MOE_PW_OK;
    if (!ret_x || !ret_hdr || !slot_map || !gates || !out || !counters) return MOE_PW_EINVAL;
    if (!aligned(ret_x, 16) || !aligned(out, 16) || !aligned(ret_hdr, 4) ||
        !aligned(slot_map, 4) || !aligned(gates, 4) || !aligned(counters, 8))
        return MOE_PW_EUNSUPPORTED;
    return cuda_rc(launch_combine(g, ret_x, ret_hdr, slot_map, gates, out, counters, stream));
}

int moe_pw_ep_stats(const moe_pw_config *cfg, const moe_pw_ep *ep,
                    const moe_pw_counters *counters, const int32_t *expert_counts,
                    moe_pw_drop_stats *host_out, int32_t *host_expert_counts,
                    cudaStream_t stream)
{
    Geo g;
    int rc = make_geo_ep(cfg, ep, &g);
    if (rc != MOE_PW_OK) return rc;
    if (!counters || !host_out) return MOE_PW_EINVAL;
    moe_pw_counters c;
    if (cudaMemcpyAsync(&c, counters, sizeof(c), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return MOE_PW_ECUDA;
    const size_t el = size_t(g.Rn) * g.L;
    if (expert_counts && host_expert_counts &&
        cudaMemcpyAsync(host_expert_counts, expert_counts, sizeof(int32_t) * 2 * el,
                        cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return MOE_PW_ECUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_PW_ECUDA;
    host_out->assignments = g.T * g.k;
    host_out->kept = int64_t(c.kept);
    host_out->sender_dropped = int64_t(c.sender_dropped);
    host_out->receiver_dropped = int64_t(c.receiver_dropped);
    host_out->max_occ = c.max_occ;
    host_out->max_fill = c.max_fill;
    host_out->error = c.error;
    host_out->reserved = 0;
    return c.error != 0 ? MOE_PW_EDEVICE : MOE_PW_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Buffer sharing between the processes of an expert-parallel run.
// ---------------------------------------------------------------------------

namespace moe_pw {
namespace {

// cuMemGetAddressRange from the driver, fetched through the runtime (the
// library links only the runtime): the base of the allocation holding a
// device pointer, which cudaIpcGetMemHandle describes.
typedef int (*mem_range_fn)(unsigned long long *, size_t *, unsigned long long);

mem_range_fn mem_range()
{
    static mem_range_fn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return mem_range_fn(nullptr);
        return reinterpret_cast<mem_range_fn>(p);
    }();
    return fn;
}

}  // namespace
}  // namespace moe_pw

extern "C" {

int moe_pw_ipc_export(const void *dev_ptr, moe_pw_ipc_handle *out)
{
    if (!dev_ptr || !out) return MOE_PW_EINVAL;
    static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(out->handle), "IPC handle size");
    const mem_range_fn range = mem_range();
    if (!range) return MOE_PW_ECUDA;
    unsigned long long base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<unsigned long long>(dev_ptr)) != 0)
        return MOE_PW_ECUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess)
        return MOE_PW_ECUDA;
    std::memcpy(out->handle, &h, sizeof(h));
    out->offset = reinterpret_cast<unsigned long long>(dev_ptr) - base;
    return MOE_PW_OK;
}

int moe_pw_ipc_open(const moe_pw_ipc_handle *h, void **dev_ptr)
{
    if (!h || !dev_ptr) return MOE_PW_EINVAL;
    cudaIpcMemHandle_t ch;
    std::memcpy(&ch, h->handle, sizeof(ch));
    void *base = nullptr;
    if (cudaIpcOpenMemHandle(&base, ch, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
        return MOE_PW_ECUDA;
    *dev_ptr = static_cast<char *>(base) + h->offset;
    return MOE_PW_OK;
}

int moe_pw_ipc_close(void *dev_ptr, const moe_pw_ipc_handle *h)
{
    if (!dev_ptr || !h) return MOE_PW_EINVAL;
    return cuda_rc(cudaIpcCloseMemHandle(static_cast<char *>(dev_ptr) - h->offset));
}

}  // extern "C"
