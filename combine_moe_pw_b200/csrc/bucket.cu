// bucket.cu - exchange (index relabel) + receiver bucketing.
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 二: the 1.15 receiver factor
// caps the rows a local expert accepts; overflow is dropped and counted apart
// from sender drops.  The all-to-all gives destination d the pools (s, d, w);
// on one GPU destination d simply reads them where source s wrote them.
//
// Pooled: one block per (d, w).  The block walks positions q = s * C_s + c
// (sources ascending, slots ascending) 1024 at a time; an arrival's row in its
// expert bucket is the number of earlier arrivals with the same header, found
// with one ballot per local expert, a block-wide scan of the warp counts and a
// running total per expert.  Positions c >= occ are empty.
// Ragged: rows are already grouped by expert; row r of expert e is r - off[e].
#include "common.cuh"

namespace moe_pw {

namespace {

struct BucketArgs {
    const int32_t *pool_hdr;
    const int32_t *occ;
    int32_t *recv_row;
    int32_t *bucket_slot;
    int32_t *expert_counts;
    moe_pw_counters *ctr;
    Geo g;
};

// Dynamic shared memory: wcnt[P][32] warp counts, run[P] running totals, tot[P].
__global__ void __launch_bounds__(1024) bucket_pooled(BucketArgs p)
{
    extern __shared__ int32_t sm[];
    const int P = p.g.P;
    int32_t *wcnt = sm;
    int32_t *run = sm + 32 * P;
    int32_t *tot = run + P;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int dw = blockIdx.x;
    const int d = dw / p.g.W, w = dw - d * p.g.W;
    const int32_t e0 = d * p.g.L + w * p.g.P;
    const int64_t C_s = p.g.C_s, C_r = p.g.C_r;
    const int64_t npos = int64_t(p.g.R) * C_s;
    for (int i = threadIdx.x; i < P; i += blockDim.x) run[i] = 0;
    __syncthreads();

    for (int64_t base = 0; base < npos; base += blockDim.x) {
        const int64_t q = base + threadIdx.x;
        int64_t slot = -1;
        int pe = -1;
        if (q < npos) {
            const int64_t s = q / C_s, c = q - s * C_s;
            const int64_t pool = (s * p.g.R + d) * p.g.W + w;
            slot = pool * C_s + c;
            if (c < p.occ[pool]) {
                const int32_t e = p.pool_hdr[slot];
                pe = e - e0;
                if (pe < 0 || pe >= P) {
                    pe = -1;
                    set_error(p.ctr, MOE_PW_DEVERR_HEADER);
                }
            }
        }
        int32_t pre = 0;
        for (int pp = 0; pp < P; ++pp) {
            const unsigned bal = __ballot_sync(FULL_MASK, pe == pp);
            if (pe == pp) pre = __popc(bal & lanemask_lt());
            if (lane == 0) wcnt[pp * 32 + warp] = __popc(bal);
        }
        __syncthreads();
        if (warp == 0) {
            const int nw = blockDim.x >> 5;
            for (int pp = 0; pp < P; ++pp) {
                const int32_t v = lane < nw ? wcnt[pp * 32 + lane] : 0;
                int32_t inc = v;
                for (int o = 1; o < 32; o <<= 1) {
                    const int32_t u = __shfl_up_sync(FULL_MASK, inc, o);
                    if (lane >= o) inc += u;
                }
                if (lane < nw) wcnt[pp * 32 + lane] = inc - v;
                if (lane == 31) tot[pp] = inc;
            }
        }
        __syncthreads();
        if (slot >= 0) {
            int32_t row = -1;
            if (pe >= 0) {
                const int64_t r = int64_t(run[pe]) + wcnt[pe * 32 + warp] + pre;
                if (r < C_r) {
                    row = int32_t(r);
                    p.bucket_slot[int64_t(e0 + pe) * C_r + r] = int32_t(slot);
                }
            }
            p.recv_row[slot] = row;
        }
        __syncthreads();
        if (threadIdx.x < P) run[threadIdx.x] += tot[threadIdx.x];
        __syncthreads();
    }

    for (int pp = 0; pp < P; ++pp) {
        const int32_t arrivals = run[pp];
        const int64_t kept = arrivals < C_r ? arrivals : C_r;
        const int32_t e = e0 + pp;
        for (int64_t r = kept + threadIdx.x; r < C_r; r += blockDim.x)
            p.bucket_slot[int64_t(e) * C_r + r] = -1;
        if (threadIdx.x == 0) {
            p.expert_counts[e] = arrivals;
            p.expert_counts[p.g.E + e] = int32_t(kept);
            if (arrivals > kept)
                atomicAdd(&p.ctr->receiver_dropped, (unsigned long long)(arrivals - kept));
            atomicAdd(&p.ctr->kept, (unsigned long long)kept);
            atomicMax(&p.ctr->max_fill, int32_t(kept));
        }
    }
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
                          moe_pw_counters *ctr, cudaStream_t st)
{
    BucketArgs p;
    p.pool_hdr = pool_hdr;
    p.occ = occ;
    p.recv_row = recv_row;
    p.bucket_slot = bucket_slot;
    p.expert_counts = expert_counts;
    p.ctr = ctr;
    p.g = g;
    if (g.T == 0) return cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * 2 * g.E, st);
    if (g.mode == MOE_PW_POOLED) {
        const size_t smem = sizeof(int32_t) * (32 * size_t(g.P) + 2 * size_t(g.P));
        bucket_pooled<<<g.R * g.W, 1024, smem, st>>>(p);
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
