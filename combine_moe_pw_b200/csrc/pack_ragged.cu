// pack_ragged.cu - the dropless mode's pack, in the order its rows are stored.
//
// "Marin 开始公开训练 535B 参数 MoE 模型", section 四, lists a dropless ragged
// all-to-all as the alternative to capacity drops: every assignment gets a row,
// the rows grouped by expert (ascending) and in token order inside an expert.
//
// Sweeping the tokens (pack.cu) reads each x row once and stores it to its k
// rows, but the stores in flight then spread over every expert's region of
// the T*k-row array.  Here the rows are written in their own order instead,
// block by block: the tokens are cut into blocks of about 24 MB of x, and
// within block b the rows go out expert by expert (the run of expert e's rows
// whose tokens fall in block b is contiguous), so the stores in flight cover a
// few neighbouring runs.  Each row is loaded from x[t] with a TMA bulk copy;
// the block's x rows are used k times while the block is being written, and
// stay in L2 meanwhile (x is read from HBM about once).
//
// Inputs this needs besides the pack's own:
//   - the row -> token map, written by ragged_tokens_kernel into pool_hdr
//     (each row's header slot holds its token until the row is copied, then
//     the expert id), from slot_map;
//   - per block, where each expert's run starts: occ[e] (the expert's first
//     row) + the assignment pass's chunk base of the block's first chunk for
//     e (the workspace of moe_pw_assign, unchanged since), and the exclusive
//     prefix over experts of the runs' lengths (ragged_runs_kernel).
// Work: warp g takes pieces g, g + G, ... of 32 consecutive rows of the
// block-major order; a piece never straddles a block.  Each piece's rows are
// found lane-parallel (binary search over the block's run prefix in shared
// memory) and queued; a ring of row stages keeps loads and stores in flight as
// in pack.cu.
#include <cstring>

#include "common.cuh"

namespace moe_pw {

namespace {

constexpr uint32_t RG_WAIT_LIMIT = 1u << 24;
constexpr int RG_LAG = 12;          // store groups left in flight before a refill
constexpr int RG_MAX_STAGES = 32;
constexpr int RG_QUEUE = 64;         // queued rows per warp (>= stages + one piece)

struct RaggedPack {
    const uint16_t *x;
    const int32_t *slot_map;
    const int32_t *occ;      // [E + 1] first row of each expert
    const int32_t *bases;    // [n_chunks][E] chunk bases from the assignment pass
    int32_t *seq;            // [n_blocks][E + 1] run prefix within each block
    uint16_t *pool_x;
    int32_t *pool_hdr;
    moe_pw_counters *ctr;
    int64_t T;
    int64_t n_rows;          // T * k
    int32_t k, D, E;
    int32_t stages;
    uint32_t rowbytes;
    int32_t chunk_tokens;    // tokens per assignment chunk
    int32_t cpb;             // chunks per block
    int32_t n_chunks, n_blocks;
    int64_t block_tokens;    // cpb * chunk_tokens
};

__device__ __forceinline__ int64_t block_rows(const RaggedPack &p, int64_t b)
{
    const int64_t t0 = b * p.block_tokens;
    const int64_t t1 = t0 + p.block_tokens < p.T ? t0 + p.block_tokens : p.T;
    return (t1 - t0) * p.k;
}

// row -> token, into the header array (overwritten by the expert id later)
__global__ void ragged_tokens_kernel(RaggedPack p)
{
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t a = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; a < p.n_rows; a += stride) {
        const int32_t row = p.slot_map[a];
        if (row < 0 || row >= p.n_rows)
            set_error(p.ctr, MOE_PW_DEVERR_SLOT);
        else
            p.pool_hdr[row] = int32_t(a / p.k);
    }
}

// seq[b][e] = rows of experts < e among block b's tokens; seq[b][E] = all
__global__ void __launch_bounds__(1024) ragged_runs_kernel(RaggedPack p)
{
    __shared__ int32_t wsum[33];
    const int b = blockIdx.x;
    const int E = p.E;
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = threadIdx.x * per;
    const int32_t *cur = p.bases + int64_t(b) * p.cpb * E;
    const bool last = (b + 1) * p.cpb >= p.n_chunks;
    const int32_t *nxt = p.bases + int64_t(b + 1) * p.cpb * E;
    int32_t local = 0;
    for (int e = e0; e < e0 + per && e < E; ++e) {
        const int32_t end = last ? p.occ[e + 1] - p.occ[e] : nxt[e];
        local += end - cur[e];
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t incl = local;
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(FULL_MASK, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        const int32_t v = lane < nw ? wsum[lane] : 0;
        int32_t inc = v;
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(FULL_MASK, inc, o);
            if (lane >= o) inc += u;
        }
        if (lane < nw) wsum[lane] = inc - v;
        if (lane == nw - 1) wsum[32] = inc;
    }
    __syncthreads();
    int32_t run = wsum[warp] + incl - local;
    int32_t *out = p.seq + int64_t(b) * (E + 1);
    for (int e = e0; e < e0 + per && e < E; ++e) {
        out[e] = run;
        const int32_t end = last ? p.occ[e + 1] - p.occ[e] : nxt[e];
        run += end - cur[e];
    }
    if (threadIdx.x == 0) out[E] = wsum[32];
}

__global__ void __launch_bounds__(32) pack_ragged_kernel(RaggedPack p)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x & 31;
    const int NS = p.stages;
    const uint32_t rb = p.rowbytes;
    const int E = p.E;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem);                       // [NS]
    int32_t *q_row = reinterpret_cast<int32_t *>(smem + RG_MAX_STAGES * 8);  // [RG_QUEUE]
    int32_t *q_tok = q_row + RG_QUEUE;
    int32_t *q_exp = q_tok + RG_QUEUE;
    int32_t *seq_sm = q_exp + RG_QUEUE;                                       // [E + 1]
    int32_t *base_sm = seq_sm + E + 1;                                        // [E]
    const size_t meta = size_t(RG_MAX_STAGES) * 8 + 3 * RG_QUEUE * 4 + (2 * size_t(E) + 1) * 4;
    unsigned char *buf = smem + ((meta + 127) & ~size_t(127));

    if (lane == 0)
        for (int s = 0; s < NS; ++s) mbar_init(&bar[s], 1);
    fence_init_and_proxy();
    __syncwarp();

    const uint64_t pol_x = policy_evict_normal();
    const uint64_t pol_pool = policy_evict_first();
    const int64_t D = p.D;
    const int64_t gw = blockIdx.x, GW = gridDim.x;
    const int64_t full_rows = int64_t(p.block_tokens) * p.k;
    const int64_t ppb = (full_rows + 31) / 32;  // pieces per full block
    const int64_t last_rows = block_rows(p, p.n_blocks - 1);
    const int64_t n_pieces = int64_t(p.n_blocks - 1) * ppb + (last_rows + 31) / 32;

    int64_t piece = gw;      // next piece to queue
    int64_t cached_b = -1;   // block whose runs are in shared memory
    int64_t tail = 0;        // rows queued so far (stream positions)

    // queue the next piece's rows (lane l: row 32 * j + l of block b)
    auto enqueue = [&]() -> bool {
        if (piece >= n_pieces) return false;
        const int64_t b = piece / ppb, j = piece - b * ppb;
        piece += GW;
        if (b != cached_b) {
            __syncwarp();
            const int32_t *sq = p.seq + b * (E + 1);
            const int32_t *bs = p.bases + b * p.cpb * int64_t(E);
            for (int e = lane; e <= E; e += 32) {
                seq_sm[e] = sq[e];
                if (e < E) base_sm[e] = bs[e];
            }
            cached_b = b;
            __syncwarp();
        }
        const int64_t rows_b = b == p.n_blocks - 1 ? last_rows : full_rows;
        const int64_t q = 32 * j + lane;
        const int nv = int(rows_b - 32 * j < 32 ? rows_b - 32 * j : 32);
        int32_t row = -1, tok = -1, e = -1;
        if (lane < nv) {
            // the run holding position q: the last e with seq[e] <= q
            int lo = 0, hi = E;  // seq[lo] <= q < seq[hi]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (seq_sm[mid] <= q) lo = mid; else hi = mid;
            }
            e = lo;
            row = p.occ[e] + base_sm[e] + int32_t(q - seq_sm[e]);
            if (row < 0 || row >= p.n_rows) {
                set_error(p.ctr, MOE_PW_DEVERR_SLOT);
                row = -1;
            } else {
                tok = p.pool_hdr[row];
                if (tok < 0 || tok >= p.T) {
                    set_error(p.ctr, MOE_PW_DEVERR_SLOT);
                    row = -1;
                }
            }
        }
        if (lane < nv) {
            const int slot = int((tail + lane) % RG_QUEUE);
            q_row[slot] = row;
            q_tok[slot] = tok;
            q_exp[slot] = e;
        }
        tail += nv;
        __syncwarp();
        return true;
    };

    auto issue_load = [&](int64_t i) {
        const int s = int(i % NS);
        const int slot = int(i % RG_QUEUE);
        mbar_arrive_expect_tx(&bar[s], rb);
        const int32_t tok = q_row[slot] >= 0 ? q_tok[slot] : 0;  // a skipped row still fills its stage
        bulk_g2s(buf + size_t(s) * rb, p.x + int64_t(tok) * D, rb, &bar[s], pol_x);
    };

    // fill the ring
    while (tail < NS && enqueue()) {}
    if (lane == 0)
        for (int64_t i = 0; i < tail && i < NS; ++i) issue_load(i);
    bool ok = true;
    for (int64_t i = 0; i < tail; ++i) {
        // keep the queue one piece ahead of the refill position
        const int64_t ii = i - RG_LAG + NS;
        while (ii >= tail && tail - i < RG_QUEUE - 32 && enqueue()) {}
        const int s = int(i % NS);
        const uint32_t parity = uint32_t((i / NS) & 1);
        const bool landed = mbar_wait_bounded(&bar[s], parity, RG_WAIT_LIMIT);
        if (!__all_sync(FULL_MASK, landed)) {
            // stop taking rows; wait (bounded) for the loads still in flight
            ok = false;
            const int64_t last = i < RG_LAG ? (tail < NS ? tail : NS) - 1
                                            : (i - 1 - RG_LAG + NS < tail ? i - 1 - RG_LAG + NS
                                                                         : tail - 1);
            for (int64_t jj = i; jj <= last; ++jj)
                mbar_wait_bounded(&bar[jj % NS], uint32_t((jj / NS) & 1), RG_WAIT_LIMIT / NS);
            break;
        }
        if (lane == 0) {
            const int slot = int(i % RG_QUEUE);
            const int32_t row = q_row[slot];
            if (row >= 0) {
                bulk_s2g(p.pool_x + int64_t(row) * D, buf + size_t(s) * rb, rb, pol_pool);
                p.pool_hdr[row] = q_exp[slot];
            }
        }
        bulk_commit();
        if (i >= RG_LAG) {
            bulk_wait_read<RG_LAG>();
            __syncwarp();
            if (lane == 0 && ii < tail) issue_load(ii);
        }
    }
    if (!ok && lane == 0) set_error(p.ctr, MOE_PW_DEVERR_TIMEOUT);
    bulk_wait_all();
}

}  // namespace

cudaError_t launch_pack_ragged(const Geo &g, const uint16_t *x, const int32_t *slot_map,
                               const int32_t *occ, uint16_t *pool_x, int32_t *pool_hdr,
                               moe_pw_counters *ctr, void *ws, cudaStream_t st)
{
    if (g.T == 0) return cudaSuccess;
    DevInfo di;
    if (dev_info(&di) != 0) return cudaErrorUnknown;
    RaggedPack p;
    std::memset(&p, 0, sizeof(p));
    p.x = x;
    p.slot_map = slot_map;
    p.occ = occ;
    p.bases = static_cast<const int32_t *>(ws);  // the assignment pass's chunk bases
    p.seq = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + ws_counts_bytes(g) +
                                        ws_totals_bytes(g));
    p.pool_x = pool_x;
    p.pool_hdr = pool_hdr;
    p.ctr = ctr;
    p.T = g.T;
    p.n_rows = g.T * g.k;
    p.k = g.k;
    p.D = g.D;
    p.E = g.E;
    p.rowbytes = uint32_t(g.D) * 2u;
    p.chunk_tokens = int32_t(g.chunk_tokens);
    const int64_t cpb = ragged_chunks_per_block(g);
    p.cpb = int32_t(cpb);
    p.n_chunks = g.n_chunks;
    p.n_blocks = int32_t((g.n_chunks + cpb - 1) / cpb);
    p.block_tokens = cpb * g.chunk_tokens;

    const size_t meta = size_t(RG_MAX_STAGES) * 8 + 3 * RG_QUEUE * 4 + (2 * size_t(g.E) + 1) * 4;
    const size_t head = (meta + 127) & ~size_t(127);
    int stages = int((size_t(di.smem_optin) - 1024 - head) / p.rowbytes);
    if (stages > RG_MAX_STAGES) stages = RG_MAX_STAGES;
    if (stages < RG_LAG + 2) return cudaErrorNotSupported;
    p.stages = stages;
    const size_t smem = head + size_t(stages) * p.rowbytes;

    cudaError_t err;
    int64_t blocks = (p.n_rows + 255) / 256;
    if (blocks > int64_t(di.sms) * 8) blocks = int64_t(di.sms) * 8;
    ragged_tokens_kernel<<<unsigned(blocks), 256, 0, st>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    ragged_runs_kernel<<<p.n_blocks, 1024, 0, st>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if ((err = cudaFuncSetAttribute(pack_ragged_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    int(smem))) != cudaSuccess)
        return err;
    const int64_t pieces = (p.n_rows + 31) / 32 + p.n_blocks;
    int64_t grid = di.sms;
    if (grid > pieces) grid = pieces;
    pack_ragged_kernel<<<unsigned(grid), 32, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace moe_pw
