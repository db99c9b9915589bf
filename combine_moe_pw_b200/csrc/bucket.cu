// bucket.cu - exchange (index relabel) + receiver bucketing.
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 二: the 1.15 receiver factor
// caps the rows a local expert accepts; overflow is dropped and counted apart
// from sender drops.  The all-to-all gives destination d the pools (s, d, w);
// on one GPU destination d simply reads them where source s wrote them.
//
// Pooled: one block per (d, w), the item worker of bucket_body.cuh over all
// of the block's threads.  Ragged: rows are already grouped by expert; row r
// of expert e is r - off[e].
#include "bucket_body.cuh"

namespace moe_pw {

namespace {

constexpr int BK_THREADS = 512;

__global__ void __launch_bounds__(BK_THREADS, 2) bucket_pooled(BucketArgs p)
{
    extern __shared__ __align__(16) int32_t sm[];
    const int dw = blockIdx.x;
    const int w = dw % p.g.W;
    if (!((p.wave_mask >> w) & 1u)) return;
    bucket_item<BK_THREADS, 0, false>(p, dw, threadIdx.x, sm);
}

__global__ void bucket_ragged(BucketArgs p)
{
    const int64_t n = p.g.n_slots;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t q = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; q < n; q += stride) {
        const int32_t e = p.pool_hdr[q];
        int32_t row = -1;
        if (e >= 0 && e < p.g.E)
            row = int32_t(q - p.occ[e]);
        else
            set_error(p.ctr, MOE_PW_DEVERR_HEADER);
        p.recv_row[q] = row;
    }
    for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < p.g.E; e += stride) {
        const int32_t cnt = p.occ[e + 1] - p.occ[e];
        p.expert_counts[e] = cnt;
        p.expert_counts[p.g.E + e] = cnt;
        atomicMax(&p.ctr->max_fill, cnt);
        atomicAdd(&p.ctr->kept, (unsigned long long)cnt);
    }
}

}  // namespace

cudaError_t launch_bucket(const Geo &g, const int32_t *pool_hdr, const int32_t *occ,
                          int32_t *recv_row, int32_t *bucket_slot, int32_t *expert_counts,
                          moe_pw_counters *ctr, cudaStream_t st, uint32_t wave_mask)
{
    BucketArgs p;
    p.pool_hdr = pool_hdr;
    p.occ = occ;
    p.recv_row = recv_row;
    p.bucket_slot = bucket_slot;
    p.expert_counts = expert_counts;
    p.ctr = ctr;
    p.g = g;
    p.wave_mask = wave_mask;
    p.hdr_out = nullptr;
    if (g.T == 0 && g.ep_n == 1)
        return cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * 2 * g.E, st);
    if (g.mode == MOE_PW_POOLED) {
        const size_t smem = bucket_smem_bytes(BK_THREADS, g.P);
        const cudaError_t aerr = cudaFuncSetAttribute(
            bucket_pooled, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (aerr != cudaSuccess) return aerr;
        bucket_pooled<<<g.Rn * g.W, BK_THREADS, smem, st>>>(p);
    } else {
        DevInfo di;
        if (dev_info(&di) != 0) return cudaErrorUnknown;
        int64_t blocks = (g.n_slots + 255) / 256;
        if (blocks > int64_t(di.sms) * 8) blocks = int64_t(di.sms) * 8;
        bucket_ragged<<<unsigned(blocks), 256, 0, st>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace moe_pw
