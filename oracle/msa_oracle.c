/*
 * msa_oracle.c -- plain CPU oracle for the MiniMax Sparse Attention (MSA) forward path and its
 * backward (gradients of the main branch, KL training signal of the index branch).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or load this file;
 * only the tests, the package's smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes is the method's plain definition, in double precision, with no blocking,
 * fusion or reordering beyond the definition:
 *
 *  (1) Index Branch (MSA explainer "MiniMax Sparse Attention", Figure 1 and section 05-1;
 *      paper abstract): for query row i and GQA group r, score every visible key j <= i with
 *      s_j = q_idx[i,r] . k_idx[j,r]; max-pool the scores over each B_k-token KV block; pick
 *      the Top-k blocks per (i, r) on the raw scores (softmax keeps the order, so no exp is
 *      needed), always keeping the local block floor(i/B_k), which counts toward k.
 *      Readings where the pages are silent: ties go to the lower block index; a block b is
 *      visible iff b*B_k <= i; the selected set is emitted ascending, padded with -1; its size
 *      is min(k, floor(i/B_k)+1).
 *  (2) KV->Q inversion (explainer section 05-2, "KV-outer" paragraph): for every (r, b) the
 *      ascending list of query rows i whose set contains b, each entry i*k + slot where slot is
 *      the rank of b in i's ascending set.
 *  (3) Main Branch (explainer sections 02 and 05-2; abstract "exact block-sparse attention"):
 *      exact softmax attention of head h (group r = floor(h/G), adjacent heads share a KV head,
 *      explainer section 01) over the tokens T = {j <= i : j in a selected block}, logits
 *      q_h . k_j / sqrt(d_h); out = sum_j p_j v_j; lse = max + log(sum exp(. - max)) in the
 *      units of the scaled logits.
 *  (4) Decode: (1)+(3) for the single query at position len-1 of each cached sequence.
 *  (5) Main Branch backward: the gradient of (3) in q, k and v with the selected sets fixed.
 *  (6) Index Branch KL alignment loss (explainer section 03) and its gradient in q_idx, k_idx.
 *  (7) FP8 main branch: E4M3 quantisation of q, k, v per row and (3) on the dequantised values.
 *
 * Inputs are bf16 bit patterns widened exactly to double. All sums are in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static inline double bf16_to_double(uint16_t x)
{
    uint32_t u = (uint32_t)x << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static void set_threads(int n_threads)
{
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
}

int msa_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------------------------------- */
/* (1) Index Branch: score, block max-pool, Top-k with the forced local block.               */
/* ---------------------------------------------------------------------------------------- */

typedef struct {
    double score;
    int32_t block;
} scored_block;

/* Sort order of the Top-k: larger pooled score first; equal scores, lower block first. */
static int by_score_then_block(const void* a, const void* b)
{
    const scored_block* x = (const scored_block*)a;
    const scored_block* y = (const scored_block*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->block > y->block) - (x->block < y->block);
}

static int ascending_int(const void* a, const void* b)
{
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/*
 * Selection for one query row of one group.
 *   qrow : d_idx bf16 values of q_idx[i, r]
 *   kseq : k_idx of the sequence, element (j, r, d) at kseq[(j*H_kv + r)*d_idx + d]
 *   i    : query position
 *   sel  : k outputs
 *   work : scratch of at least floor(i/B_k) entries
 */
static void select_one(const uint16_t* qrow, const uint16_t* kseq, int64_t i, int r, int H_kv, int d_idx,
                       int B_k, int k, int32_t* sel, scored_block* work)
{
    const int64_t local = i / B_k;          /* the forced local block */
    const int64_t n_candidates = local;     /* blocks 0 .. local-1 are fully visible */
    double q[512];
    for (int d = 0; d < d_idx; ++d) q[d] = bf16_to_double(qrow[d]);

    for (int64_t b = 0; b < n_candidates; ++b) {
        double best = -INFINITY;
        for (int64_t j = b * B_k; j < (b + 1) * B_k; ++j) {
            const uint16_t* kr = kseq + ((size_t)j * H_kv + r) * d_idx;
            double s = 0.0;
            for (int d = 0; d < d_idx; ++d) s += q[d] * bf16_to_double(kr[d]);
            if (s > best) best = s; /* block max pooling */
        }
        work[b].score = best;
        work[b].block = (int32_t)b;
    }
    qsort(work, (size_t)n_candidates, sizeof(scored_block), by_score_then_block);

    int n = 0;
    const int64_t take = n_candidates < (int64_t)(k - 1) ? n_candidates : (int64_t)(k - 1);
    for (int64_t t = 0; t < take; ++t) sel[n++] = work[t].block;
    sel[n++] = (int32_t)local;
    qsort(sel, (size_t)n, sizeof(int32_t), ascending_int);
    for (int t = n; t < k; ++t) sel[t] = -1;
}

/*
 * Selections for a set of query rows of one sequence.
 *   q_idx : [n_rows, H_kv, d_idx] bf16, the index queries of the requested rows (gathered)
 *   rows  : [n_rows] positions i (each < N)
 *   k_idx : [N, H_kv, d_idx] bf16
 *   sel   : [n_rows, H_kv, k] int32 out
 * Returns 0, or -1 on bad arguments.
 */
int msa_oracle_select_rows(const uint16_t* q_idx, const int64_t* rows, int64_t n_rows, const uint16_t* k_idx,
                           int64_t N, int H_kv, int d_idx, int B_k, int k, int32_t* sel, int n_threads)
{
    if (!q_idx || !rows || !k_idx || !sel || N < 1 || H_kv < 1 || d_idx < 1 || d_idx > 512 || B_k < 1 || k < 1)
        return -1;
    for (int64_t t = 0; t < n_rows; ++t)
        if (rows[t] < 0 || rows[t] >= N) return -1;
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        scored_block* work = (scored_block*)malloc(sizeof(scored_block) * (size_t)(N / B_k + 1));
        if (!work) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (int64_t t = 0; t < n_rows; ++t)
            for (int r = 0; r < H_kv; ++r)
                if (work)
                    select_one(q_idx + ((size_t)t * H_kv + r) * d_idx, k_idx, rows[t], r, H_kv, d_idx, B_k, k,
                               sel + ((size_t)t * H_kv + r) * k, work);
        free(work);
    }
    return err;
}

/* ---------------------------------------------------------------------------------------- */
/* (2) KV -> Q inversion.                                                                     */
/* ---------------------------------------------------------------------------------------- */

/*
 *   block_idx : [H_kv, N, k] int32, ascending, -1 padded
 *   offsets   : [H_kv, nb+1] int64 out, CSR row pointers per group (offsets[r][0] = 0)
 *   entries   : [H_kv, N*k] int32 out, entries of group r start at entries + r*N*k
 * For each (r, b) the entries are the rows i (ascending) whose set holds b, encoded i*k + slot.
 * Returns 0, or -1 on an out-of-range block id.
 */
int msa_oracle_kv2q(const int32_t* block_idx, int64_t N, int H_kv, int B_k, int k, int64_t* offsets,
                    int32_t* entries)
{
    const int64_t nb = (N + B_k - 1) / B_k;
    for (int r = 0; r < H_kv; ++r) {
        const int32_t* sel = block_idx + (size_t)r * N * k;
        int64_t* off = offsets + (size_t)r * (nb + 1);
        int32_t* ent = entries + (size_t)r * N * k;
        for (int64_t b = 0; b <= nb; ++b) off[b] = 0;
        for (int64_t i = 0; i < N; ++i)
            for (int s = 0; s < k; ++s) {
                int32_t b = sel[i * k + s];
                if (b < 0) continue;
                if (b >= nb) return -1;
                off[b + 1] += 1;
            }
        for (int64_t b = 0; b < nb; ++b) off[b + 1] += off[b];
        int64_t* fill = (int64_t*)malloc(sizeof(int64_t) * (size_t)nb);
        if (!fill) return -1;
        for (int64_t b = 0; b < nb; ++b) fill[b] = off[b];
        for (int64_t i = 0; i < N; ++i) /* ascending i keeps each list sorted by row */
            for (int s = 0; s < k; ++s) {
                int32_t b = sel[i * k + s];
                if (b < 0) continue;
                ent[fill[b]++] = (int32_t)(i * k + s);
            }
        free(fill);
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------- */
/* (3) Main Branch: exact softmax attention over the selected blocks' visible tokens.        */
/* ---------------------------------------------------------------------------------------- */

/*
 * One (row, head).
 *   qh   : d_h bf16, q[i, h]
 *   kseq, vseq : [*, H_kv, d_h] bf16 of the sequence
 *   sel  : k block ids of (i, r), -1 padded
 *   out  : d_h doubles; *lse out
 *   logits : scratch of k*B_k doubles
 */
static void attend_one(const uint16_t* qh, const uint16_t* kseq, const uint16_t* vseq, int64_t i, int r, int H_kv,
                       int d_h, int B_k, int k, const int32_t* sel, double* out, double* lse, double* logits)
{
    const double scale = 1.0 / sqrt((double)d_h);
    double q[512];
    for (int d = 0; d < d_h; ++d) q[d] = bf16_to_double(qh[d]);

    /* logits over T, in the order of the selected blocks */
    int64_t n = 0;
    double m = -INFINITY;
    for (int s = 0; s < k; ++s) {
        int32_t b = sel[s];
        if (b < 0) continue;
        for (int64_t j = (int64_t)b * B_k; j < ((int64_t)b + 1) * B_k && j <= i; ++j) {
            const uint16_t* kr = kseq + ((size_t)j * H_kv + r) * d_h;
            double dot = 0.0;
            for (int d = 0; d < d_h; ++d) dot += q[d] * bf16_to_double(kr[d]);
            logits[n] = dot * scale;
            if (logits[n] > m) m = logits[n];
            ++n;
        }
    }
    double z = 0.0;
    for (int d = 0; d < d_h; ++d) out[d] = 0.0;
    n = 0;
    for (int s = 0; s < k; ++s) {
        int32_t b = sel[s];
        if (b < 0) continue;
        for (int64_t j = (int64_t)b * B_k; j < ((int64_t)b + 1) * B_k && j <= i; ++j) {
            double p = exp(logits[n++] - m);
            z += p;
            const uint16_t* vr = vseq + ((size_t)j * H_kv + r) * d_h;
            for (int d = 0; d < d_h; ++d) out[d] += p * bf16_to_double(vr[d]);
        }
    }
    for (int d = 0; d < d_h; ++d) out[d] /= z;
    *lse = m + log(z);
}

/*
 *   q    : [n_rows, H_q, d_h] bf16, the requested rows' queries (gathered)
 *   rows : [n_rows] positions
 *   kk, v: [N, H_kv, d_h] bf16
 *   sel  : [n_rows, H_kv, k] int32 (from msa_oracle_select_rows)
 *   out  : [n_rows, H_q, d_h] double; lse : [n_rows, H_q] double
 */
int msa_oracle_attend_rows(const uint16_t* q, const int64_t* rows, int64_t n_rows, const uint16_t* kk,
                           const uint16_t* v, int64_t N, int H_q, int H_kv, int d_h, int B_k, int k,
                           const int32_t* sel, double* out, double* lse, int n_threads)
{
    if (!q || !rows || !kk || !v || !sel || !out || !lse || H_kv < 1 || H_q % H_kv || d_h < 1 || d_h > 512)
        return -1;
    for (int64_t t = 0; t < n_rows; ++t)
        if (rows[t] < 0 || rows[t] >= N) return -1;
    const int G = H_q / H_kv;
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        double* logits = (double*)malloc(sizeof(double) * (size_t)k * B_k);
        if (!logits) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (int64_t t = 0; t < n_rows; ++t)
            for (int h = 0; h < H_q; ++h)
                if (logits) {
                    const int r = h / G;
                    attend_one(q + ((size_t)t * H_q + h) * d_h, kk, v, rows[t], r, H_kv, d_h, B_k, k,
                               sel + ((size_t)t * H_kv + r) * k, out + ((size_t)t * H_q + h) * d_h,
                               lse + (size_t)t * H_q + h, logits);
                }
        free(logits);
    }
    return err;
}

/* ---------------------------------------------------------------------------------------- */
/* (4) Decode: one query per cached sequence, at position len-1.                              */
/* ---------------------------------------------------------------------------------------- */

/*
 *   q      : [B, H_q, d_h] bf16;  q_idx : [B, H_kv, d_idx] bf16
 *   k_cache, v_cache : [B, L_max, H_kv, d_h] bf16;  k_idx_cache : [B, L_max, H_kv, d_idx] bf16
 *   lens   : [B] int32, 1 <= len <= L_max (the cache holds the current token)
 *   out    : [B, H_q, d_h] double; lse : [B, H_q] double; sel : [B, H_kv, k] int32
 */
int msa_oracle_decode(const uint16_t* q, const uint16_t* q_idx, const uint16_t* k_cache, const uint16_t* v_cache,
                      const uint16_t* k_idx_cache, const int32_t* lens, int B, int64_t L_max, int H_q, int H_kv,
                      int d_h, int d_idx, int B_k, int k, double* out, double* lse, int32_t* sel, int n_threads)
{
    for (int beta = 0; beta < B; ++beta)
        if (lens[beta] < 1 || lens[beta] > L_max) return -1;
    for (int beta = 0; beta < B; ++beta) {
        const int64_t row = lens[beta] - 1;
        const size_t kv_off = (size_t)beta * L_max * H_kv * d_h;
        const size_t ki_off = (size_t)beta * L_max * H_kv * d_idx;
        int rc = msa_oracle_select_rows(q_idx + (size_t)beta * H_kv * d_idx, &row, 1, k_idx_cache + ki_off,
                                        lens[beta], H_kv, d_idx, B_k, k, sel + (size_t)beta * H_kv * k, n_threads);
        if (rc) return rc;
        rc = msa_oracle_attend_rows(q + (size_t)beta * H_q * d_h, &row, 1, k_cache + kv_off, v_cache + kv_off,
                                    lens[beta], H_q, H_kv, d_h, B_k, k, sel + (size_t)beta * H_kv * k,
                                    out + (size_t)beta * H_q * d_h, lse + (size_t)beta * H_q, n_threads);
        if (rc) return rc;
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------- */
/* (5) Main Branch backward: the gradient of (3) with the selected sets held fixed.          */
/* ---------------------------------------------------------------------------------------- */
/*
 * The Top-k selection is not differentiable (explainer section 03), so the language-model loss
 * reaches q, k and v only through the exact softmax attention over T(i, r) of (3). For one
 * (row i, head h) with p_j = exp(q.k_j*scale - lse), out = sum_j p_j v_j and upstream dout:
 *   D      = dout . out
 *   ds_j   = p_j * (dout . v_j - D)          (softmax Jacobian applied to dout . v_j)
 *   dq_i  += scale * sum_j ds_j k_j
 *   dk_j  += scale * ds_j q_i
 *   dv_j  += p_j dout
 * lse and out are recomputed here from q, k, v (the forward pass stores them; the backward of
 * the explainer's kernels reads them back, section 05-2, "LSE fusion" paragraph).
 */

/* logits and weights of (i, h) over T in the order of the selected blocks; returns |T|.
 * tok[n] = key position of logits[n]. */
static int64_t probs_one(const double* q, const uint16_t* kseq, int64_t i, int r, int H_kv, int d_h, int B_k, int k,
                         const int32_t* sel, double* p, int64_t* tok)
{
    const double scale = 1.0 / sqrt((double)d_h);
    int64_t n = 0;
    double m = -INFINITY;
    for (int s = 0; s < k; ++s) {
        int32_t b = sel[s];
        if (b < 0) continue;
        for (int64_t j = (int64_t)b * B_k; j < ((int64_t)b + 1) * B_k && j <= i; ++j) {
            const uint16_t* kr = kseq + ((size_t)j * H_kv + r) * d_h;
            double dot = 0.0;
            for (int d = 0; d < d_h; ++d) dot += q[d] * bf16_to_double(kr[d]);
            p[n] = dot * scale;
            tok[n] = j;
            if (p[n] > m) m = p[n];
            ++n;
        }
    }
    double z = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        p[t] = exp(p[t] - m);
        z += p[t];
    }
    for (int64_t t = 0; t < n; ++t) p[t] /= z;
    return n;
}

/* ds_j of (i, h) over T (in place of p), given p and dout; returns D = dout . out. */
static double dscores_one(const double* dout, const uint16_t* vseq, int r, int H_kv, int d_h, int64_t n,
                          const int64_t* tok, const double* p, double* ds)
{
    double out[512];
    for (int d = 0; d < d_h; ++d) out[d] = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        const uint16_t* vr = vseq + ((size_t)tok[t] * H_kv + r) * d_h;
        for (int d = 0; d < d_h; ++d) out[d] += p[t] * bf16_to_double(vr[d]);
    }
    double D = 0.0;
    for (int d = 0; d < d_h; ++d) D += dout[d] * out[d];
    for (int64_t t = 0; t < n; ++t) {
        const uint16_t* vr = vseq + ((size_t)tok[t] * H_kv + r) * d_h;
        double dp = 0.0;
        for (int d = 0; d < d_h; ++d) dp += dout[d] * bf16_to_double(vr[d]);
        ds[t] = p[t] * (dp - D);
    }
    return D;
}

/*
 * dq of requested rows.
 *   q, dout : [n_rows, H_q, d_h] bf16, gathered for the requested rows
 *   rows    : [n_rows] positions;  kk, v : [N, H_kv, d_h] bf16
 *   sel     : [n_rows, H_kv, k] int32 selections of the rows
 *   dq      : [n_rows, H_q, d_h] double
 */
int msa_oracle_backward_dq_rows(const uint16_t* q, const uint16_t* dout, const int64_t* rows, int64_t n_rows,
                                const uint16_t* kk, const uint16_t* v, int64_t N, int H_q, int H_kv, int d_h,
                                int B_k, int k, const int32_t* sel, double* dq, int n_threads)
{
    if (!q || !dout || !rows || !kk || !v || !sel || !dq || H_kv < 1 || H_q % H_kv || d_h < 1 || d_h > 512)
        return -1;
    for (int64_t t = 0; t < n_rows; ++t)
        if (rows[t] < 0 || rows[t] >= N) return -1;
    const int G = H_q / H_kv;
    const double scale = 1.0 / sqrt((double)d_h);
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)k * B_k);
        double* ds = (double*)malloc(sizeof(double) * (size_t)k * B_k);
        int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * (size_t)k * B_k);
        const int ok = p && ds && tok;
        if (!ok) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (int64_t t = 0; t < n_rows; ++t)
            for (int h = 0; h < H_q; ++h)
                if (ok) {
                    const int r = h / G;
                    double qd[512], dod[512];
                    for (int d = 0; d < d_h; ++d) {
                        qd[d] = bf16_to_double(q[((size_t)t * H_q + h) * d_h + d]);
                        dod[d] = bf16_to_double(dout[((size_t)t * H_q + h) * d_h + d]);
                    }
                    const int32_t* s_r = sel + ((size_t)t * H_kv + r) * k;
                    const int64_t n = probs_one(qd, kk, rows[t], r, H_kv, d_h, B_k, k, s_r, p, tok);
                    dscores_one(dod, v, r, H_kv, d_h, n, tok, p, ds);
                    double* g = dq + ((size_t)t * H_q + h) * d_h;
                    for (int d = 0; d < d_h; ++d) g[d] = 0.0;
                    for (int64_t u = 0; u < n; ++u) {
                        const uint16_t* kr = kk + ((size_t)tok[u] * H_kv + r) * d_h;
                        for (int d = 0; d < d_h; ++d) g[d] += scale * ds[u] * bf16_to_double(kr[d]);
                    }
                }
        free(p);
        free(ds);
        free(tok);
    }
    return err;
}

/* does (i, r) select block b? */
static int selects(const int32_t* s_ir, int k, int32_t b)
{
    for (int s = 0; s < k; ++s)
        if (s_ir[s] == b) return 1;
    return 0;
}

/*
 * dk and dv of whole KV blocks: for each requested (group r, block b), every row i whose set
 * contains b and every head h of group r contribute to the keys j <= i of block b.
 *   q, dout : [N, H_q, d_h] bf16 (all rows);  kk, v : [N, H_kv, d_h] bf16
 *   sel     : [N, H_kv, k] int32 selections of all rows
 *   pairs   : [n_pairs, 2] (r, b)
 *   dk, dv  : [n_pairs, B_k, d_h] double (rows past N are zero)
 */
int msa_oracle_backward_dkv_blocks(const uint16_t* q, const uint16_t* dout, const uint16_t* kk, const uint16_t* v,
                                   int64_t N, int H_q, int H_kv, int d_h, int B_k, int k, const int32_t* sel,
                                   const int32_t* pairs, int64_t n_pairs, double* dk, double* dv, int n_threads)
{
    if (!q || !dout || !kk || !v || !sel || !pairs || !dk || !dv || H_kv < 1 || H_q % H_kv || d_h < 1 ||
        d_h > 512)
        return -1;
    const int64_t nb = (N + B_k - 1) / B_k;
    for (int64_t t = 0; t < n_pairs; ++t)
        if (pairs[2 * t] < 0 || pairs[2 * t] >= H_kv || pairs[2 * t + 1] < 0 || pairs[2 * t + 1] >= nb) return -1;
    const int G = H_q / H_kv;
    const double scale = 1.0 / sqrt((double)d_h);
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)k * B_k);
        double* ds = (double*)malloc(sizeof(double) * (size_t)k * B_k);
        int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * (size_t)k * B_k);
        const int ok = p && ds && tok;
        if (!ok) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < n_pairs; ++t) {
            if (!ok) continue;
            const int r = pairs[2 * t];
            const int32_t b = pairs[2 * t + 1];
            double* gk = dk + (size_t)t * B_k * d_h;
            double* gv = dv + (size_t)t * B_k * d_h;
            for (int64_t x = 0; x < (int64_t)B_k * d_h; ++x) gk[x] = gv[x] = 0.0;
            for (int64_t i = (int64_t)b * B_k; i < N; ++i) {
                const int32_t* s_ir = sel + ((size_t)i * H_kv + r) * k;
                if (!selects(s_ir, k, b)) continue;
                for (int h = r * G; h < (r + 1) * G; ++h) {
                    double qd[512], dod[512];
                    for (int d = 0; d < d_h; ++d) {
                        qd[d] = bf16_to_double(q[((size_t)i * H_q + h) * d_h + d]);
                        dod[d] = bf16_to_double(dout[((size_t)i * H_q + h) * d_h + d]);
                    }
                    const int64_t n = probs_one(qd, kk, i, r, H_kv, d_h, B_k, k, s_ir, p, tok);
                    dscores_one(dod, v, r, H_kv, d_h, n, tok, p, ds);
                    for (int64_t u = 0; u < n; ++u) {
                        if (tok[u] / B_k != b) continue;
                        const int64_t jj = tok[u] - (int64_t)b * B_k;
                        for (int d = 0; d < d_h; ++d) {
                            gk[jj * d_h + d] += scale * ds[u] * qd[d];
                            gv[jj * d_h + d] += p[u] * dod[d];
                        }
                    }
                }
            }
        }
        free(p);
        free(ds);
        free(tok);
    }
    return err;
}

/* ---------------------------------------------------------------------------------------- */
/* (6) Index Branch training signal: the KL alignment loss and its gradient.                 */
/* ---------------------------------------------------------------------------------------- */
/*
 * Explainer section 03 ("KL Loss"): for query i and group r, over the token set T(i, r) of the
 * selected blocks,
 *   student  P_idx_j = softmax_T(s_idx)_j,   s_idx_j = q_idx[i,r] . k_idx[j,r]   (the index score
 *            of (1), unscaled: the pages give the index score no scale)
 *   teacher  P_j = (1/G) sum_{h in group r} p_{h,j}     (the G heads' attention weights of (3),
 *            averaged as probabilities)
 *   KL(i, r) = sum_j P_j (log P_j - log P_idx_j)
 * The loss averages KL over positions and groups; the teacher is stop-gradient, so the gradient
 * reaches only the index projections: dKL/ds_idx_j = P_idx_j - P_j, hence
 *   dq_idx[i,r] += w * sum_j (P_idx_j - P_j) k_idx[j,r]
 *   dk_idx[j,r] += w * (P_idx_j - P_j) q_idx[i,r]
 * with w the caller's weight (1 / (rows * H_kv) for the mean).
 */

/* teacher weights P over T of (i, r) into P[0..n), with tok[]; student log-weights into lq[]. */
static int64_t kl_dists(const uint16_t* q_i /*[H_q, d_h]*/, const uint16_t* qidx_ir, const uint16_t* kk,
                        const uint16_t* k_idx, int64_t i, int r, int H_q, int H_kv, int d_h, int d_idx, int B_k, int k,
                        const int32_t* s_ir, double* P, double* lq, double* p, int64_t* tok)
{
    const int G = H_q / H_kv;
    int64_t n = 0;
    for (int h = r * G; h < (r + 1) * G; ++h) {
        double qd[512];
        for (int d = 0; d < d_h; ++d) qd[d] = bf16_to_double(q_i[(size_t)h * d_h + d]);
        n = probs_one(qd, kk, i, r, H_kv, d_h, B_k, k, s_ir, p, tok);
        for (int64_t t = 0; t < n; ++t) P[t] = (h == r * G ? 0.0 : P[t]) + p[t] / G;
    }
    double m = -INFINITY;
    for (int64_t t = 0; t < n; ++t) {
        const uint16_t* kr = k_idx + ((size_t)tok[t] * H_kv + r) * d_idx;
        double s = 0.0;
        for (int d = 0; d < d_idx; ++d) s += bf16_to_double(qidx_ir[d]) * bf16_to_double(kr[d]);
        lq[t] = s;
        if (s > m) m = s;
    }
    double z = 0.0;
    for (int64_t t = 0; t < n; ++t) z += exp(lq[t] - m);
    const double lz = m + log(z);
    for (int64_t t = 0; t < n; ++t) lq[t] -= lz;
    return n;
}

/*
 * KL(i, r) and dq_idx of requested rows.
 *   q      : [n_rows, H_q, d_h] bf16;  q_idx : [n_rows, H_kv, d_idx] bf16 (gathered rows)
 *   kk     : [N, H_kv, d_h] bf16;      k_idx : [N, H_kv, d_idx] bf16
 *   sel    : [n_rows, H_kv, k] int32
 *   kl     : [n_rows, H_kv] double;    dq_idx : [n_rows, H_kv, d_idx] double (scaled by w)
 */
int msa_oracle_kl_rows(const uint16_t* q, const uint16_t* q_idx, const int64_t* rows, int64_t n_rows,
                       const uint16_t* kk, const uint16_t* k_idx, int64_t N, int H_q, int H_kv, int d_h, int d_idx,
                       int B_k, int k, const int32_t* sel, double w, double* kl, double* dq_idx, int n_threads)
{
    if (!q || !q_idx || !rows || !kk || !k_idx || !sel || !kl || !dq_idx || H_kv < 1 || H_q % H_kv || d_h < 1 ||
        d_h > 512 || d_idx < 1)
        return -1;
    for (int64_t t = 0; t < n_rows; ++t)
        if (rows[t] < 0 || rows[t] >= N) return -1;
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        const size_t cap = (size_t)k * B_k;
        double* P = (double*)malloc(sizeof(double) * cap);
        double* lq = (double*)malloc(sizeof(double) * cap);
        double* p = (double*)malloc(sizeof(double) * cap);
        int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * cap);
        const int ok = P && lq && p && tok;
        if (!ok) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (int64_t t = 0; t < n_rows; ++t)
            for (int r = 0; r < H_kv; ++r)
                if (ok) {
                    const uint16_t* qi = q_idx + ((size_t)t * H_kv + r) * d_idx;
                    const int64_t n = kl_dists(q + (size_t)t * H_q * d_h, qi, kk, k_idx, rows[t], r, H_q, H_kv, d_h,
                                               d_idx, B_k, k, sel + ((size_t)t * H_kv + r) * k, P, lq, p, tok);
                    double acc = 0.0;
                    double* g = dq_idx + ((size_t)t * H_kv + r) * d_idx;
                    for (int d = 0; d < d_idx; ++d) g[d] = 0.0;
                    for (int64_t u = 0; u < n; ++u) {
                        acc += P[u] * (log(P[u]) - lq[u]);
                        const double gs = w * (exp(lq[u]) - P[u]);
                        const uint16_t* kr = k_idx + ((size_t)tok[u] * H_kv + r) * d_idx;
                        for (int d = 0; d < d_idx; ++d) g[d] += gs * bf16_to_double(kr[d]);
                    }
                    kl[(size_t)t * H_kv + r] = acc;
                }
        free(P);
        free(lq);
        free(p);
        free(tok);
    }
    return err;
}

/*
 * dk_idx of whole KV blocks: every row i whose set of group r contains b contributes to the keys
 * j <= i of block b.
 *   q : [N, H_q, d_h], q_idx : [N, H_kv, d_idx], kk : [N, H_kv, d_h], k_idx : [N, H_kv, d_idx] (bf16)
 *   sel : [N, H_kv, k] int32;  pairs : [n_pairs, 2] (r, b)
 *   dk_idx : [n_pairs, B_k, d_idx] double (scaled by w; rows past N are zero)
 */
int msa_oracle_kl_dk_idx_blocks(const uint16_t* q, const uint16_t* q_idx, const uint16_t* kk, const uint16_t* k_idx,
                                int64_t N, int H_q, int H_kv, int d_h, int d_idx, int B_k, int k, const int32_t* sel,
                                const int32_t* pairs, int64_t n_pairs, double w, double* dk_idx, int n_threads)
{
    if (!q || !q_idx || !kk || !k_idx || !sel || !pairs || !dk_idx || H_kv < 1 || H_q % H_kv || d_h < 1 ||
        d_h > 512 || d_idx < 1)
        return -1;
    const int64_t nb = (N + B_k - 1) / B_k;
    for (int64_t t = 0; t < n_pairs; ++t)
        if (pairs[2 * t] < 0 || pairs[2 * t] >= H_kv || pairs[2 * t + 1] < 0 || pairs[2 * t + 1] >= nb) return -1;
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        const size_t cap = (size_t)k * B_k;
        double* P = (double*)malloc(sizeof(double) * cap);
        double* lq = (double*)malloc(sizeof(double) * cap);
        double* p = (double*)malloc(sizeof(double) * cap);
        int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * cap);
        const int ok = P && lq && p && tok;
        if (!ok) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < n_pairs; ++t) {
            if (!ok) continue;
            const int r = pairs[2 * t];
            const int32_t b = pairs[2 * t + 1];
            double* g = dk_idx + (size_t)t * B_k * d_idx;
            for (int64_t x = 0; x < (int64_t)B_k * d_idx; ++x) g[x] = 0.0;
            for (int64_t i = (int64_t)b * B_k; i < N; ++i) {
                const int32_t* s_ir = sel + ((size_t)i * H_kv + r) * k;
                if (!selects(s_ir, k, b)) continue;
                const uint16_t* qi = q_idx + ((size_t)i * H_kv + r) * d_idx;
                const int64_t n = kl_dists(q + (size_t)i * H_q * d_h, qi, kk, k_idx, i, r, H_q, H_kv, d_h, d_idx, B_k,
                                           k, s_ir, P, lq, p, tok);
                for (int64_t u = 0; u < n; ++u) {
                    if (tok[u] / B_k != b) continue;
                    const int64_t jj = tok[u] - (int64_t)b * B_k;
                    const double gs = w * (exp(lq[u]) - P[u]);
                    for (int d = 0; d < d_idx; ++d) g[jj * d_idx + d] += gs * bf16_to_double(qi[d]);
                }
            }
        }
        free(P);
        free(lq);
        free(p);
        free(tok);
    }
    return err;
}

/* ---------------------------------------------------------------------------------------- */
/* (7) FP8 main branch: OCP E4M3 quantisation and attention over the dequantised values.      */
/* ---------------------------------------------------------------------------------------- */
/*
 * The blog page's kernel paragraph says the kernels were tuned on FP8 tensor cores but gives no
 * quantisation. Reading: q, k and v are quantised to E4M3 (1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, subnormals, no infinities, largest finite 448, S.1111.111 is NaN) row by row,
 * one scale per (token, head) row = amax / 448, round to nearest with ties to the even code,
 * saturating at 448; the main branch (3) then runs on the dequantised values code * scale.
 */

double msa_oracle_e4m3_decode(uint8_t c)
{
    if ((c & 0x7F) == 0x7F) return NAN; /* S.1111.111 */
    const int e = (c >> 3) & 15, m = c & 7;
    const double v = e == 0 ? ldexp((double)m, -9)         /* subnormal: m/8 * 2^-6 */
                            : ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return (c & 0x80) ? -v : v;
}

/* nearest finite E4M3 value by search over the 127 non-negative finite codes (0x00..0x7E, which
 * decode in increasing order); ties go to the code with an even mantissa; |x| >= 448 saturates */
uint8_t msa_oracle_e4m3_encode(double x)
{
    const uint8_t sign = signbit(x) ? 0x80 : 0;
    const double a = fabs(x);
    uint8_t best = 0;
    for (int c = 1; c <= 0x7E; ++c) {
        const double dc = fabs(msa_oracle_e4m3_decode((uint8_t)c) - a);
        const double db = fabs(msa_oracle_e4m3_decode(best) - a);
        if (dc < db || (dc == db && (c & 1) == 0)) best = (uint8_t)c;
    }
    return sign | best;
}

/*
 *   x      : [rows, cols] bf16
 *   codes  : [rows, cols] E4M3 codes;  scales : [rows] (amax / 448; 1 for an all-zero row)
 */
int msa_oracle_quantize_e4m3_rows(const uint16_t* x, int64_t rows, int cols, uint8_t* codes, double* scales)
{
    if (!x || !codes || !scales || rows < 0 || cols < 1) return -1;
    /* rows are independent: one row per iteration, any thread */
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double amax = 0.0;
        for (int c = 0; c < cols; ++c) {
            const double v = fabs(bf16_to_double(x[r * cols + c]));
            if (v > amax) amax = v;
        }
        const double scale = amax > 0.0 ? amax / 448.0 : 1.0;
        scales[r] = scale;
        for (int c = 0; c < cols; ++c) codes[r * cols + c] = msa_oracle_e4m3_encode(bf16_to_double(x[r * cols + c]) / scale);
    }
    return 0;
}

/* (3) for one (i, h) on double inputs (the dequantised rows) */
static void attend_one_f64(const double* q, const double* kseq, const double* vseq, int64_t i, int r, int H_kv,
                           int d_h, int B_k, int k, const int32_t* sel, double* out, double* lse, double* logits)
{
    const double scale = 1.0 / sqrt((double)d_h);
    int64_t n = 0;
    double m = -INFINITY;
    for (int s = 0; s < k; ++s) {
        const int32_t b = sel[s];
        if (b < 0) continue;
        for (int64_t j = (int64_t)b * B_k; j < ((int64_t)b + 1) * B_k && j <= i; ++j) {
            const double* kr = kseq + ((size_t)j * H_kv + r) * d_h;
            double dot = 0.0;
            for (int d = 0; d < d_h; ++d) dot += q[d] * kr[d];
            logits[n] = dot * scale;
            if (logits[n] > m) m = logits[n];
            ++n;
        }
    }
    double z = 0.0;
    for (int d = 0; d < d_h; ++d) out[d] = 0.0;
    n = 0;
    for (int s = 0; s < k; ++s) {
        const int32_t b = sel[s];
        if (b < 0) continue;
        for (int64_t j = (int64_t)b * B_k; j < ((int64_t)b + 1) * B_k && j <= i; ++j) {
            const double p = exp(logits[n++] - m);
            z += p;
            const double* vr = vseq + ((size_t)j * H_kv + r) * d_h;
            for (int d = 0; d < d_h; ++d) out[d] += p * vr[d];
        }
    }
    for (int d = 0; d < d_h; ++d) out[d] /= z;
    *lse = m + log(z);
}

/*
 * (3) on E4M3 inputs: value = code * scale of its row.
 *   qc, qs : [n_rows, H_q, d_h] codes, [n_rows, H_q] scales of the requested rows (gathered)
 *   kc, ks, vc, vs : [N, H_kv, d_h] codes, [N, H_kv] scales
 *   sel    : [n_rows, H_kv, k];  out : [n_rows, H_q, d_h] double;  lse : [n_rows, H_q] double
 */
int msa_oracle_attend_rows_e4m3(const uint8_t* qc, const double* qs, const int64_t* rows, int64_t n_rows,
                                const uint8_t* kc, const double* ks, const uint8_t* vc, const double* vs, int64_t N,
                                int H_q, int H_kv, int d_h, int B_k, int k, const int32_t* sel, double* out,
                                double* lse, int n_threads)
{
    if (!qc || !qs || !rows || !kc || !ks || !vc || !vs || !sel || !out || !lse || H_kv < 1 || H_q % H_kv ||
        d_h < 1 || d_h > 512)
        return -1;
    for (int64_t t = 0; t < n_rows; ++t)
        if (rows[t] < 0 || rows[t] >= N) return -1;
    const int G = H_q / H_kv;
    double* kd = (double*)malloc(sizeof(double) * (size_t)N * H_kv * d_h);
    double* vd = (double*)malloc(sizeof(double) * (size_t)N * H_kv * d_h);
    if (!kd || !vd) {
        free(kd);
        free(vd);
        return -1;
    }
    for (int64_t x = 0; x < N * H_kv; ++x)
        for (int d = 0; d < d_h; ++d) {
            kd[x * d_h + d] = msa_oracle_e4m3_decode(kc[x * d_h + d]) * ks[x];
            vd[x * d_h + d] = msa_oracle_e4m3_decode(vc[x * d_h + d]) * vs[x];
        }
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        double* logits = (double*)malloc(sizeof(double) * (size_t)k * B_k);
        if (!logits) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (int64_t t = 0; t < n_rows; ++t)
            for (int h = 0; h < H_q; ++h)
                if (logits) {
                    double qd[512];
                    const size_t qh = (size_t)t * H_q + h;
                    for (int d = 0; d < d_h; ++d) qd[d] = msa_oracle_e4m3_decode(qc[qh * d_h + d]) * qs[qh];
                    const int r = h / G;
                    attend_one_f64(qd, kd, vd, rows[t], r, H_kv, d_h, B_k, k, sel + ((size_t)t * H_kv + r) * k,
                                   out + qh * d_h, lse + qh, logits);
                }
        free(logits);
    }
    free(kd);
    free(vd);
    return err;
}
