/*
 * oracle.c - plain, slow, single-threaded CPU definition of capacity-limited
 * pooled-wave MoE token dispatch and combine.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's CPU
 * baseline may load this.  It shares no source, header, table or helper with
 * the CUDA library, and it never reads anything the CUDA library computed.
 *
 * Sources (pages):
 *   [P1-2] "Marin 开始公开训练 535B 参数 MoE 模型" (lamjinlab blog), section 二
 *          (how the sparse model is organised): 384 routed experts, router picks
 *          8 per token; 64-GPU expert-parallel domain with 6 experts per GPU;
 *          one fixed pool per destination GPU instead of per-expert buffers;
 *          three consecutive waves of identical shape; the expert id travels in
 *          the activation payload so no counts or routing metadata are sent;
 *          sender capacity factor 1.10 per source->destination, receiver factor
 *          1.15 per local expert; assignments over either buffer are dropped and
 *          the two kinds of drop are reported apart.
 *   [P1-4] same page, section 四: a dropped assignment does not remove the token
 *          (shared experts still see it); a dropless ragged all-to-all is listed
 *          as an alternative.
 *   [P2-a2a] "535B大模型“直播”训练三个月" (huxiu), MoE/token-dropping section:
 *          one all-to-all sends tokens to experts, a second brings results back.
 *
 * Where the pages are silent the plainest reading is taken; each one is marked
 * READING below.  Floating point: the softmax gates and the combine are formed
 * in double (the pages fix no precision).  The per-expert op y = s_e * x is
 * rounded to bf16, a discrete decision, so its product is taken in fp32, the
 * precision the device kernel decides it in, and then rounded to nearest even.
 *
 * Build: gcc -O2 -fPIC -shared -ffp-contract=off (no FMA contraction, IEEE
 * single/double on x86-64 SSE2).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Geometry of one batch as the oracle sees it. */
typedef struct {
    int64_t T;    /* tokens supplied                                         */
    int64_t T_s;  /* tokens per source shard; sources present = T / T_s      */
    int32_t R;    /* expert-parallel ranks = destinations                    */
    int32_t L;    /* experts per rank                                        */
    int32_t W;    /* waves                                                   */
    int32_t P;    /* experts per wave, L == W * P                            */
    int32_t E;    /* routed experts, E == R * L                              */
    int32_t k;    /* experts chosen per token                                */
    int32_t D;    /* latent width (bf16 elements)                            */
    int32_t pad;
    int64_t C_s;  /* sender capacity per (source, destination, wave) pool    */
    int64_t C_r;  /* receiver capacity per expert                            */
} orc_geom;

/* ------------------------------------------------------------------------ */
/* Capacities.                                                               */
/* ------------------------------------------------------------------------ */

/*
 * [P1-2] fixes the factors (1.10 sender, 1.15 receiver) but not what they
 * multiply.  READING: "expected" is the mean load under uniform routing and
 * the product is rounded up.
 *   sender   : one (source, destination, wave) pool carries P of the E experts
 *              for T_s tokens with k choices each -> T_s*k*P/E rows expected.
 *   receiver : one expert over the whole batch -> T*k/E rows expected.
 * Factors are given in integer percent so the product is exact:
 *   C = ceil(pct * num / (100 * den)).
 * pct <= 0 means unbounded: the largest load that can occur, T_s*min(k,P)
 * for a pool and T for an expert, so nothing is ever dropped.
 */
static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int orc_capacity(int64_t T, int64_t T_s, int32_t E, int32_t k, int32_t P,
                 int32_t cf_send_pct, int32_t cf_recv_pct,
                 int64_t *C_s, int64_t *C_r)
{
    if (T < 0 || T_s <= 0 || E <= 0 || k <= 0 || P <= 0) return -1;
    if (cf_send_pct > 0)
        *C_s = ceil_div((int64_t)cf_send_pct * T_s * k * P, (int64_t)100 * E);
    else
        *C_s = T_s * (k < P ? k : P);
    if (cf_recv_pct > 0)
        *C_r = ceil_div((int64_t)cf_recv_pct * T * k, (int64_t)100 * E);
    else
        *C_r = T;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Route: top-k of the router logits and softmax gates.                      */
/* ------------------------------------------------------------------------ */

/*
 * [P1-2] the router picks k (=8) of E (=384) experts per token.
 * READING: the k largest logits, ordered by value descending; equal values go
 * to the lower expert index (float comparison, so -0.0 and +0.0 are equal).
 * Selection by k passes of "largest not yet chosen".
 * Gates: softmax over the k chosen logits, max-subtracted, terms summed in
 * j order (READING: the pages do not say how gates are formed).
 */
void orc_route(const orc_geom *g, const float *logits, int32_t *idx, double *gates)
{
    const int32_t E = g->E, k = g->k;
    char *chosen = (char *)malloc((size_t)E);
    double *ex = (double *)malloc(sizeof(double) * (size_t)k);
    for (int64_t t = 0; t < g->T; ++t) {
        const float *l = logits + t * E;
        memset(chosen, 0, (size_t)E);
        for (int32_t j = 0; j < k; ++j) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (chosen[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict: lower index keeps ties */
            }
            chosen[best] = 1;
            idx[t * k + j] = best;
        }
        const double top = (double)l[idx[t * k]];
        double den = 0.0;
        for (int32_t j = 0; j < k; ++j) {
            ex[j] = exp((double)l[idx[t * k + j]] - top);
            den += ex[j];
        }
        for (int32_t j = 0; j < k; ++j) gates[t * k + j] = ex[j] / den;
    }
    free(chosen);
    free(ex);
}

/* ------------------------------------------------------------------------ */
/* Placement of an expert.                                                   */
/* ------------------------------------------------------------------------ */

/*
 * [P1-2] 6 experts per destination GPU, three waves of identical shape.
 * READING: experts are placed contiguously (d = e / L, local = e % L) and wave
 * w carries local experts {P*w, ..., P*w + P - 1}.
 */
static void place(const orc_geom *g, int32_t e, int32_t *d, int32_t *w)
{
    *d = e / g->L;
    *w = (e % g->L) / g->P;
}

/* Flat slot id of (source s, destination d, wave w, position c). */
static int64_t slot_id(const orc_geom *g, int64_t s, int32_t d, int32_t w, int64_t c)
{
    return ((s * g->R + d) * g->W + w) * g->C_s + c;
}

/* ------------------------------------------------------------------------ */
/* Sender slot assignment (pooled).                                          */
/* ------------------------------------------------------------------------ */

/*
 * [P1-2] one fixed pool per (source, destination) per wave; the sender factor
 * caps what one source sends to one destination; overflow is dropped.
 * READING: token t belongs to source s = t / T_s; within a source the
 * assignments (t, j) are taken in lexicographic order; an assignment's slot in
 * pool (s, d, w) is the number of earlier assignments of that source in the
 * same pool; it is kept when that number is below C_s and dropped otherwise.
 *
 * Outputs: slot_map[t*k+j] = flat slot or -1; occ[(s*R+d)*W+w] = rows kept
 * in the pool; slot_tok[slot] = token in the slot or -1.  Returns the number
 * of sender drops.
 */
int64_t orc_assign_pooled(const orc_geom *g, const int32_t *idx, int32_t *slot_map,
                          int32_t *occ, int32_t *slot_tok)
{
    const int64_t n_src = g->T / g->T_s;
    const int64_t n_pool = n_src * g->R * g->W;
    int64_t *count = (int64_t *)calloc((size_t)n_pool, sizeof(int64_t));
    for (int64_t q = 0; q < n_pool * g->C_s; ++q) slot_tok[q] = -1;
    int64_t dropped = 0;
    for (int64_t t = 0; t < g->T; ++t) {
        const int64_t s = t / g->T_s;
        for (int32_t j = 0; j < g->k; ++j) {
            int32_t d, w;
            place(g, idx[t * g->k + j], &d, &w);
            const int64_t p = (s * g->R + d) * g->W + w;
            const int64_t rank = count[p]++;
            if (rank < g->C_s) {
                const int64_t slot = slot_id(g, s, d, w, rank);
                slot_map[t * g->k + j] = (int32_t)slot;
                slot_tok[slot] = (int32_t)t;
            } else {
                slot_map[t * g->k + j] = -1;
                ++dropped;
            }
        }
    }
    for (int64_t p = 0; p < n_pool; ++p)
        occ[p] = (int32_t)(count[p] < g->C_s ? count[p] : g->C_s);
    free(count);
    return dropped;
}

/* ------------------------------------------------------------------------ */
/* Pack.                                                                     */
/* ------------------------------------------------------------------------ */

/*
 * [P1-2] the expert id is packed with the activation so the receiver needs no
 * separate counts.  Every kept (t, j) copies row x[t] bit for bit into its slot
 * and writes the global expert id into the slot's header.  READING: an empty
 * slot holds an all-zero row and header -1.
 */
void orc_pack(const orc_geom *g, int64_t n_slots, const uint16_t *x, const int32_t *idx,
              const int32_t *slot_map, uint16_t *pool_x, int32_t *pool_hdr)
{
    const int64_t D = g->D;
    for (int64_t q = 0; q < n_slots; ++q) {
        pool_hdr[q] = -1;
        for (int64_t i = 0; i < D; ++i) pool_x[q * D + i] = 0;
    }
    for (int64_t t = 0; t < g->T; ++t) {
        for (int32_t j = 0; j < g->k; ++j) {
            const int64_t slot = slot_map[t * g->k + j];
            if (slot < 0) continue;
            for (int64_t i = 0; i < D; ++i) pool_x[slot * D + i] = x[t * D + i];
            pool_hdr[slot] = idx[t * g->k + j];
        }
    }
}

/* The header half of the pack alone (same definition, rows left out), for
 * batches whose pools are too large to materialise on the host. */
void orc_pack_headers(const orc_geom *g, int64_t n_slots, const int32_t *idx,
                      const int32_t *slot_map, int32_t *pool_hdr)
{
    for (int64_t q = 0; q < n_slots; ++q) pool_hdr[q] = -1;
    for (int64_t t = 0; t < g->T; ++t)
        for (int32_t j = 0; j < g->k; ++j) {
            const int64_t slot = slot_map[t * g->k + j];
            if (slot >= 0) pool_hdr[slot] = idx[t * g->k + j];
        }
}

/* ------------------------------------------------------------------------ */
/* Exchange + receiver bucketing (pooled).                                   */
/* ------------------------------------------------------------------------ */

/*
 * The all-to-all hands destination d the pools (s, d, w) of every source s
 * ([P1-2], [P2-a2a]); here it is only a change of index: the receiver reads
 * pool (s, d, w) where the sender wrote it.
 *
 * [P1-2] the receiver factor caps the rows one local expert accepts; overflow
 * is dropped and counted apart from sender drops.
 * READING: for each (d, w) the receiver walks sources s = 0..n_src-1 and, in
 * each pool, positions c = 0..occ-1; the expert id comes from the header; an
 * arrival is kept when fewer than C_r earlier arrivals for that expert exist.
 *
 * Outputs: recv_row[slot] = row in the expert's bucket, or -1 (dropped or
 * empty); bucket_slot[e*C_r + r] = slot of row r of expert e, or -1;
 * arrivals[e], bucket_cnt[e] = min(arrivals, C_r).  Returns receiver drops.
 */
int64_t orc_bucket(const orc_geom *g, const int32_t *pool_hdr, const int32_t *occ,
                   int32_t *recv_row, int32_t *bucket_slot, int32_t *arrivals,
                   int32_t *bucket_cnt)
{
    const int64_t n_src = g->T / g->T_s;
    const int64_t n_slots = n_src * g->R * g->W * g->C_s;
    for (int64_t q = 0; q < n_slots; ++q) recv_row[q] = -1;
    for (int64_t q = 0; q < (int64_t)g->E * g->C_r; ++q) bucket_slot[q] = -1;
    for (int32_t e = 0; e < g->E; ++e) arrivals[e] = 0;
    int64_t dropped = 0;
    for (int32_t d = 0; d < g->R; ++d) {
        for (int32_t w = 0; w < g->W; ++w) {
            for (int64_t s = 0; s < n_src; ++s) {
                const int32_t filled = occ[(s * g->R + d) * g->W + w];
                for (int64_t c = 0; c < filled; ++c) {
                    const int64_t slot = slot_id(g, s, d, w, c);
                    const int32_t e = pool_hdr[slot];
                    const int64_t r = arrivals[e]++;
                    if (r < g->C_r) {
                        recv_row[slot] = (int32_t)r;
                        bucket_slot[(int64_t)e * g->C_r + r] = (int32_t)slot;
                    } else {
                        ++dropped;
                    }
                }
            }
        }
    }
    for (int32_t e = 0; e < g->E; ++e)
        bucket_cnt[e] = (int32_t)(arrivals[e] < g->C_r ? arrivals[e] : g->C_r);
    return dropped;
}

/*
 * [P1-2] the drops are reported apart; what the receivers accepted is the sum
 * of the bucket fills.  With the two drop counts it accounts for every one of
 * the T*k assignments.
 */
int64_t orc_kept(const orc_geom *g, const int32_t *bucket_cnt)
{
    int64_t kept = 0;
    for (int32_t e = 0; e < g->E; ++e) kept += bucket_cnt[e];
    return kept;
}

/* ------------------------------------------------------------------------ */
/* Dropless ragged mode.                                                     */
/* ------------------------------------------------------------------------ */

/*
 * [P1-4] lists a dropless ragged all-to-all (variable-size per-expert buffers,
 * the design [P1-2] calls awkward for memory) as the alternative.
 * READING: row counts cnt[e] = number of (t, j) with idx = e; rows of expert e
 * start at off[e], the exclusive prefix sum of cnt over e; inside an expert the
 * rows follow token order.  Nothing is dropped.
 * Outputs: slot_map[t*k+j] = row; row_off[e] (E+1 entries); row_cnt[e];
 * slot_tok[row] = token.
 */
void orc_assign_ragged(const orc_geom *g, const int32_t *idx, int32_t *slot_map,
                       int32_t *row_off, int32_t *row_cnt, int32_t *slot_tok)
{
    const int32_t E = g->E, k = g->k;
    for (int32_t e = 0; e < E; ++e) row_cnt[e] = 0;
    for (int64_t a = 0; a < g->T * k; ++a) row_cnt[idx[a]]++;
    row_off[0] = 0;
    for (int32_t e = 0; e < E; ++e) row_off[e + 1] = row_off[e] + row_cnt[e];
    int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    for (int32_t e = 0; e < E; ++e) next[e] = row_off[e];
    for (int64_t t = 0; t < g->T; ++t) {
        for (int32_t j = 0; j < k; ++j) {
            const int32_t e = idx[t * k + j];
            const int32_t row = next[e]++;
            slot_map[t * k + j] = row;
            slot_tok[row] = (int32_t)t;
        }
    }
    free(next);
}

/*
 * Receiver side of the dropless mode ([P1-4]: every row reaches its expert,
 * nothing is capped).  Like the pooled receiver, the rows are walked in the
 * order they arrive (row 0 .. n_rows-1) and each one takes the next free row
 * of its expert's bucket: recv_row[q] = number of earlier rows whose header
 * names the same expert.  Rows with header -1 (none in a complete batch) get
 * -1.  arrivals[e] = bucket_cnt[e] = rows of expert e (no receiver cap).
 */
void orc_bucket_ragged(const orc_geom *g, int64_t n_rows, const int32_t *row_hdr,
                       int32_t *recv_row, int32_t *arrivals, int32_t *bucket_cnt)
{
    for (int32_t e = 0; e < g->E; ++e) arrivals[e] = 0;
    for (int64_t q = 0; q < n_rows; ++q) {
        const int32_t e = row_hdr[q];
        if (e < 0) {
            recv_row[q] = -1;
            continue;
        }
        recv_row[q] = arrivals[e]++;
    }
    for (int32_t e = 0; e < g->E; ++e) bucket_cnt[e] = arrivals[e];
}

/* ------------------------------------------------------------------------ */
/* Per-expert op and return layout.                                          */
/* ------------------------------------------------------------------------ */

static float bf16_to_f32(uint16_t h)
{
    union { uint32_t u; float f; } v;
    v.u = (uint32_t)h << 16;
    return v.f;
}

/* Round fp32 to bf16, nearest even (finite values): add 0x7FFF plus the lowest
 * kept bit, then truncate. */
static uint16_t f32_to_bf16_rne(float f)
{
    union { float f; uint32_t u; } v;
    v.f = f;
    return (uint16_t)((v.u + 0x7FFFu + ((v.u >> 16) & 1u)) >> 16);
}

/*
 * Stand-in for the expert network (the pages' experts need trained weights):
 * y = s_e * x, product in fp32, rounded to bf16 (READING).  The return pools
 * have the dispatch pools' geometry and slot ids ([P2-a2a]: results travel
 * back by a second all-to-all).  Rows that the receiver kept are scaled; every
 * other slot holds zeros and header -1 (READING).
 *
 * Pooled: the kept rows are bucket_slot[e*C_r + r] for r < bucket_cnt[e].
 */
void orc_expert_pooled(const orc_geom *g, int64_t n_slots, const uint16_t *pool_x,
                       const int32_t *bucket_slot, const int32_t *bucket_cnt,
                       const float *scale, uint16_t *ret_x, int32_t *ret_hdr)
{
    const int64_t D = g->D;
    for (int64_t q = 0; q < n_slots; ++q) {
        ret_hdr[q] = -1;
        for (int64_t i = 0; i < D; ++i) ret_x[q * D + i] = 0;
    }
    for (int32_t e = 0; e < g->E; ++e) {
        for (int64_t r = 0; r < bucket_cnt[e]; ++r) {
            const int64_t slot = bucket_slot[(int64_t)e * g->C_r + r];
            for (int64_t i = 0; i < D; ++i) {
                const float prod = scale[e] * bf16_to_f32(pool_x[slot * D + i]);
                ret_x[slot * D + i] = f32_to_bf16_rne(prod);
            }
            ret_hdr[slot] = e;
        }
    }
}

/* Ragged: every row is kept; row r belongs to expert row_hdr[r]. */
void orc_expert_ragged(const orc_geom *g, int64_t n_rows, const uint16_t *rows,
                       const int32_t *row_hdr, const float *scale, uint16_t *ret_x,
                       int32_t *ret_hdr)
{
    const int64_t D = g->D;
    for (int64_t q = 0; q < n_rows; ++q) {
        const int32_t e = row_hdr[q];
        for (int64_t i = 0; i < D; ++i) {
            const float prod = scale[e] * bf16_to_f32(rows[q * D + i]);
            ret_x[q * D + i] = f32_to_bf16_rne(prod);
        }
        ret_hdr[q] = e;
    }
}

/* ------------------------------------------------------------------------ */
/* Combine.                                                                  */
/* ------------------------------------------------------------------------ */

/*
 * out[t] = sum over j of g_j * y_j, where y_j is the returned row of (t, j);
 * terms of dropped assignments (no slot, or the receiver dropped the row:
 * header -1) are left out and the surviving gates are not renormalised
 * ([P1-4]: a dropped assignment leaves the token to the shared experts).
 * Summed in double, j ascending, starting from 0.
 */
void orc_combine(const orc_geom *g, const uint16_t *ret_x, const int32_t *ret_hdr,
                 const int32_t *slot_map, const double *gates, double *out)
{
    const int64_t D = g->D;
    for (int64_t t = 0; t < g->T; ++t) {
        double *o = out + t * D;
        for (int64_t i = 0; i < D; ++i) o[i] = 0.0;
        for (int32_t j = 0; j < g->k; ++j) {
            const int64_t slot = slot_map[t * g->k + j];
            if (slot < 0 || ret_hdr[slot] < 0) continue;
            const double gj = gates[t * g->k + j];
            for (int64_t i = 0; i < D; ++i) o[i] += gj * (double)bf16_to_f32(ret_x[slot * D + i]);
        }
    }
}

/*
 * The same combine for a list of tokens only, with the pack and the expert op
 * written out per token: row (t, j) reaches its slot unchanged, so the returned
 * row is bf16(s_e * x[t]) when the slot survived both capacity checks
 * (slot >= 0 and recv_row[slot] >= 0) and absent otherwise.  Also returns, per
 * element, sum_j g_j * |y_j| (the scale the combine error is measured against).
 */
void orc_combine_tokens(const orc_geom *g, const uint16_t *x, const int32_t *idx,
                        const double *gates, const int32_t *slot_map,
                        const int32_t *recv_row, const float *scale,
                        const int64_t *tokens, int64_t n_tokens, double *out, double *mag)
{
    const int64_t D = g->D;
    for (int64_t n = 0; n < n_tokens; ++n) {
        const int64_t t = tokens[n];
        double *o = out + n * D, *m = mag + n * D;
        for (int64_t i = 0; i < D; ++i) o[i] = m[i] = 0.0;
        for (int32_t j = 0; j < g->k; ++j) {
            const int64_t slot = slot_map[t * g->k + j];
            if (slot < 0 || recv_row[slot] < 0) continue;
            const int32_t e = idx[t * g->k + j];
            const double gj = gates[t * g->k + j];
            for (int64_t i = 0; i < D; ++i) {
                const float prod = scale[e] * bf16_to_f32(x[t * D + i]);
                const double y = (double)bf16_to_f32(f32_to_bf16_rne(prod));
                o[i] += gj * y;
                m[i] += gj * fabs(y);
            }
        }
    }
}

/* Per-element scale of the full combine: mag[t][i] = sum_j g_j * |y_j|. */
void orc_combine_mag(const orc_geom *g, const uint16_t *ret_x, const int32_t *ret_hdr,
                     const int32_t *slot_map, const double *gates, double *mag)
{
    const int64_t D = g->D;
    for (int64_t t = 0; t < g->T; ++t) {
        double *m = mag + t * D;
        for (int64_t i = 0; i < D; ++i) m[i] = 0.0;
        for (int32_t j = 0; j < g->k; ++j) {
            const int64_t slot = slot_map[t * g->k + j];
            if (slot < 0 || ret_hdr[slot] < 0) continue;
            const double gj = gates[t * g->k + j];
            for (int64_t i = 0; i < D; ++i) m[i] += gj * fabs((double)bf16_to_f32(ret_x[slot * D + i]));
        }
    }
}

/* The oracle's own bf16 rounding, exposed so a test can hold it against a library. */
void orc_bf16_round(const float *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}

void orc_expert_product(const float *s, const uint16_t *x, uint16_t *y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) y[i] = f32_to_bf16_rne(s[i] * bf16_to_f32(x[i]));
}

/* ------------------------------------------------------------------------ */
/* Backward of combine and dispatch.                                         */
/* ------------------------------------------------------------------------ */

/*
 * The pages train this model ("Marin 开始公开训练 535B 参数 MoE 模型", section 一),
 * so the path also needs its gradient.  The pages describe no backward; these
 * are the derivatives of the forward definitions above (READING: gradients
 * travel in the same fixed pools, bf16 like the forward payload).
 *
 * Given dout = dL/dout [T, D] (fp32):
 *   surviving (t, j) (slot >= 0 and ret_hdr[slot] >= 0):
 *     d_ret[slot] = bf16(g_j * dout[t])   product in fp32 (it decides a bf16
 *                                         code), gate rounded to fp32 first
 *     dgate[t][j] = <dout[t], y_j>        y_j = returned row, in double
 *   every other slot of d_ret: zero (a fixed pool, like the forward)
 *   dgate of a dropped (t, j): 0
 *   softmax over the chosen logits: dl_j = g_j * (dgate_j - sum_i g_i dgate_i),
 *   dlogits[t][idx[t][j]] = dl_j, every other logit 0 (top-k is piecewise
 *   constant in the logits).
 */
void orc_combine_backward(const orc_geom *g, int64_t n_slots, const float *dout,
                          const uint16_t *ret_x, const int32_t *ret_hdr, const int32_t *slot_map,
                          const int32_t *idx, const double *gates, uint16_t *d_ret,
                          double *dgate, double *dlogits)
{
    const int64_t D = g->D;
    const int32_t k = g->k, E = g->E;
    for (int64_t q = 0; q < n_slots * D; ++q) d_ret[q] = 0;
    for (int64_t t = 0; t < g->T; ++t) {
        const float *dt = dout + t * D;
        double *dl = dlogits + t * E;
        for (int32_t e = 0; e < E; ++e) dl[e] = 0.0;
        double weighted = 0.0;
        for (int32_t j = 0; j < k; ++j) {
            const int64_t slot = slot_map[t * k + j];
            double dg = 0.0;
            if (slot >= 0 && ret_hdr[slot] >= 0) {
                const float gj = (float)gates[t * k + j];
                for (int64_t i = 0; i < D; ++i) {
                    d_ret[slot * D + i] = f32_to_bf16_rne(gj * dt[i]);
                    dg += (double)dt[i] * (double)bf16_to_f32(ret_x[slot * D + i]);
                }
            }
            dgate[t * k + j] = dg;
            weighted += gates[t * k + j] * dg;
        }
        for (int32_t j = 0; j < k; ++j)
            dl[idx[t * k + j]] = gates[t * k + j] * (dgate[t * k + j] - weighted);
    }
}

/*
 * Pack transpose: x[t] was copied into the slot of every (t, j) the sender
 * kept, so dx[t] = sum over those j of d_pool[slot], in double.  Slots the
 * receiver dropped carry a zero gradient (the expert op's backward writes
 * zeros there), so they are left out.
 */
void orc_dispatch_backward(const orc_geom *g, const uint16_t *d_pool, const int32_t *recv_row,
                           const int32_t *slot_map, double *dx)
{
    const int64_t D = g->D;
    for (int64_t t = 0; t < g->T; ++t) {
        double *o = dx + t * D;
        for (int64_t i = 0; i < D; ++i) o[i] = 0.0;
        for (int32_t j = 0; j < g->k; ++j) {
            const int64_t slot = slot_map[t * g->k + j];
            if (slot < 0 || recv_row[slot] < 0) continue;
            for (int64_t i = 0; i < D; ++i) o[i] += (double)bf16_to_f32(d_pool[slot * D + i]);
        }
    }
}

/*
 * The whole backward for a list of tokens only (the same definitions,
 * written per token for batches whose pools are too large for the host):
 * for each listed token t and each j it survived with (slot >= 0 and
 * recv_row[slot] >= 0), y_j = bf16(s_e * x[t]) and
 *   d_ret row  = bf16(g_j * dout[t])            (fp32 product, gate in fp32)
 *   dgate_j    = <dout[t], y_j>                  (double)
 *   d_pool row = bf16(s_e * d_ret row)           (expert op backward)
 *   dx[t]      = sum_j d_pool row                (double)
 * and dlogits row t as in orc_combine_backward.  Outputs are per listed token:
 * d_ret_rows [n, k, D] (zero for dropped j), dgate [n, k], dlogits [n, E],
 * dx [n, D].
 */
void orc_backward_tokens(const orc_geom *g, const uint16_t *x, const int32_t *idx,
                         const double *gates, const int32_t *slot_map, const int32_t *recv_row,
                         const float *scale, const float *dout, const int64_t *tokens,
                         int64_t n_tokens, uint16_t *d_ret_rows, double *dgate, double *dlogits,
                         double *dx)
{
    const int64_t D = g->D;
    const int32_t k = g->k, E = g->E;
    for (int64_t n = 0; n < n_tokens; ++n) {
        const int64_t t = tokens[n];
        const float *dt = dout + t * D;
        double *o = dx + n * D, *dl = dlogits + n * E;
        for (int64_t i = 0; i < D; ++i) o[i] = 0.0;
        for (int32_t e = 0; e < E; ++e) dl[e] = 0.0;
        double weighted = 0.0;
        for (int32_t j = 0; j < k; ++j) {
            uint16_t *gr = d_ret_rows + (n * k + j) * D;
            const int64_t slot = slot_map[t * k + j];
            double dg = 0.0;
            if (slot >= 0 && recv_row[slot] >= 0) {
                const int32_t e = idx[t * k + j];
                const float gj = (float)gates[t * k + j];
                for (int64_t i = 0; i < D; ++i) {
                    const float y = bf16_to_f32(f32_to_bf16_rne(scale[e] * bf16_to_f32(x[t * D + i])));
                    dg += (double)dt[i] * (double)y;
                    gr[i] = f32_to_bf16_rne(gj * dt[i]);
                    o[i] += (double)bf16_to_f32(f32_to_bf16_rne(scale[e] * bf16_to_f32(gr[i])));
                }
            } else {
                for (int64_t i = 0; i < D; ++i) gr[i] = 0;
            }
            dgate[n * k + j] = dg;
            weighted += gates[t * k + j] * dg;
        }
        for (int32_t j = 0; j < k; ++j)
            dl[idx[t * k + j]] = gates[t * k + j] * (dgate[n * k + j] - weighted);
    }
}

/* ------------------------------------------------------------------------ */
/* Latent projections.                                                       */
/* ------------------------------------------------------------------------ */

/*
 * "Marin 开始公开训练 535B 参数 MoE 模型", section 二: before the routed
 * activations cross GPUs a latent projection halves their width (6144 ->
 * 3072), and the outputs are projected back before they meet the shared
 * experts.  READING: a plain matrix product with bf16 operands,
 *   C[m][n] = bf16( sum_k A[m][k] * Bt[n][k] ),
 * the sum in double, rounded to fp32 and then to bf16 nearest-even (the
 * device accumulates in fp32).  Bt is stored row n = output column n.
 * The merge with the shared path (same passage: routed outputs, back at model
 * width, meet the shared experts' output) is READ as a plain sum: with add
 * (bf16 [M, N], the shared path's output) given,
 *   C[m][n] = bf16( sum_k A[m][k] * Bt[n][k] + add[m][n] ),
 * again formed in double and rounded once through fp32.
 * Also returns, per element, the exact value and sum_k |A[m][k] * Bt[n][k]|
 * plus |add[m][n]| (the accumulation error is measured against it).
 */
void orc_project(const uint16_t *A, const uint16_t *Bt, int64_t M, int64_t N, int64_t K,
                 const uint16_t *add, uint16_t *C, double *Cexact, double *mag)
{
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, am = 0.0;
            for (int64_t kk = 0; kk < K; ++kk) {
                const double p = (double)bf16_to_f32(A[m * K + kk]) * (double)bf16_to_f32(Bt[n * K + kk]);
                acc += p;
                am += fabs(p);
            }
            if (add) {
                const double s = (double)bf16_to_f32(add[m * N + n]);
                acc += s;
                am += fabs(s);
            }
            C[m * N + n] = f32_to_bf16_rne((float)acc);
            if (Cexact) Cexact[m * N + n] = acc;
            if (mag) mag[m * N + n] = am;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Sequence-level balancing.                                                 */
/* ------------------------------------------------------------------------ */

/*
 * "Marin 开始公开训练 535B 参数 MoE 模型", section 四: if drops stay too high,
 * one remedy is sequence-level balancing, which "may force the experts to
 * re-specialise during training".  The pages give no formula.  READING: a
 * balance term of the training loss computed per sequence, the product of
 * how often each expert is chosen and how much router probability it gets,
 * within one sequence:
 *   p[t][e]  = softmax over all E logits of token t
 *   f[s][e]  = E / (k * L) * #{ t in s, j : idx[t][j] == e }
 *   P[s][e]  = 1 / L * sum over t in s of p[t][e]
 *   loss[s]  = alpha * sum_e f[s][e] * P[s][e]
 * with L = seq_len tokens per sequence (T % L == 0).  Perfect balance
 * (f = 1 for every expert) gives loss = alpha whatever the probabilities.
 * The gradient treats f as constant (the top-k choice is piecewise constant
 * in the logits):
 *   dlogits[t][e] = alpha / L * p[t][e] * (f[s][e] - sum_i f[s][i] * p[t][i]).
 * All in double.  f, P: [T / L, E]; loss: [T / L]; dlogits [T, E] may be NULL.
 */
void orc_seq_balance(const orc_geom *g, int64_t seq_len, double alpha, const float *logits,
                     const int32_t *idx, double *f, double *P, double *loss, double *dlogits)
{
    const int32_t E = g->E, k = g->k;
    const int64_t n_seq = g->T / seq_len;
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    for (int64_t s = 0; s < n_seq; ++s) {
        double *fs = f + s * E, *Ps = P + s * E;
        for (int32_t e = 0; e < E; ++e) fs[e] = Ps[e] = 0.0;
        for (int64_t t = s * seq_len; t < (s + 1) * seq_len; ++t) {
            for (int32_t j = 0; j < k; ++j) fs[idx[t * k + j]] += 1.0;
            const float *l = logits + t * E;
            double mx = l[0];
            for (int32_t e = 1; e < E; ++e) if (l[e] > mx) mx = l[e];
            double den = 0.0;
            for (int32_t e = 0; e < E; ++e) den += exp((double)l[e] - mx);
            for (int32_t e = 0; e < E; ++e) Ps[e] += exp((double)l[e] - mx) / den;
        }
        double acc = 0.0;
        for (int32_t e = 0; e < E; ++e) {
            fs[e] *= (double)E / ((double)k * (double)seq_len);
            Ps[e] /= (double)seq_len;
            acc += fs[e] * Ps[e];
        }
        loss[s] = alpha * acc;
        if (!dlogits) continue;
        for (int64_t t = s * seq_len; t < (s + 1) * seq_len; ++t) {
            const float *l = logits + t * E;
            double mx = l[0];
            for (int32_t e = 1; e < E; ++e) if (l[e] > mx) mx = l[e];
            double den = 0.0;
            for (int32_t e = 0; e < E; ++e) den += exp((double)l[e] - mx);
            double dot = 0.0;
            for (int32_t e = 0; e < E; ++e) {
                p[e] = exp((double)l[e] - mx) / den;
                dot += fs[e] * p[e];
            }
            for (int32_t e = 0; e < E; ++e)
                dlogits[t * E + e] = alpha / (double)seq_len * p[e] * (fs[e] - dot);
        }
    }
    free(p);
}
