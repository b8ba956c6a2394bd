/*
 * infllmv2_oracle.c -- plain, slow fp64 CPU oracle of the InfLLM v2 sparse-attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg may load this file's library.  It shares no code, header, table or helper with the CUDA library
 * (trainable_block_sparse_v2_b200/csrc); neither side includes or links the other.
 *
 * What it computes, step by step, in the order the method states it (sources are the MiniCPM4 pages):
 *
 *   1. semantic kernels: the mean of K over a window of kernel_size keys, advanced by kernel_stride,
 *      per KV head, rounded once to bf16 (the storage format of the kernel cache)
 *        -- "Tsinghua & ModelBest: MiniCPM4 technical details" (QbitAI), section "Model architecture:
 *           InfLLM v2", item 1 (each context block is made of several fine-grained semantic kernels);
 *           window 32 / stride 16 are workload constants, the pages give no sizes.
 *   2. block relevance: for a query token and head, the max over the kernels of a block of the
 *      query-kernel score, where scores are softmax-normalised over all visible kernels (LogSumExp)
 *        -- same section, item 1 (max over the block's kernels) and item 3 (LogSumExp).
 *   3. GQA sharing: the heads of one GQA group share one block set, so the per-head normalised maxima
 *      are pooled (summed) over the group's heads
 *        -- same section, item 2 (query heads of a GQA group share the same context blocks).
 *   4. top-k selection, always keeping the initial blocks and the local blocks; ties go to the lower
 *      block index; dense attention when the context is short (n <= dense_len)
 *        -- same article, the InfLLM v2 overview (only the top few blocks take part; short sequences
 *           keep the original dense attention), and "MiniCPM 4.0 launch article" (senqingzn.com),
 *           section 1 "efficient architecture" (dense/sparse gear shift).
 *   5. causal attention over the keys of the selected blocks only, plus, for tree verification, the
 *      draft tokens whose bit is set in the node's bit-packed ancestor mask
 *        -- QbitAI article, section "speculative sampling, quantisation and long text", long-context
 *           bullet (local attention mask with bit packing for tree drafts).
 *   6. the draft model's sliding-window attention: the last `window` keys of the context
 *        -- the same bullet (sliding-window attention for the draft model; no window size given).
 *   7. the gradients of step 5's attention with respect to q, K and V for a fixed selection (training)
 *        -- "Model architecture: InfLLM v2", item 3 (operators for training as well as inference); the
 *           derivative of step 5's definition, the pages give no formula.
 *   8. the gradient of step 1 (the semantic kernels) with respect to K: the adjoint of the window mean,
 *      the bf16 rounding taken as the identity -- same item 3; the derivative of step 1's definition.
 *
 * Every floating-point step is fp64; inputs are bf16 bit patterns widened exactly.  Rows are
 * independent, so the only parallelism is an OpenMP loop over (sequence, token, group) rows; there is
 * no tiling, fusion or reordering beyond the definition.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - kernel rounding to bf16 at storage; kernel visibility = complete windows only;
 *   - membership OVERLAP (window intersects block) by default, CONTAINED (window inside block) as an option;
 *   - group pooling = sum over the group's heads of exp(max_j z_h(j) - LSE_h);
 *   - LSE is computed exactly (the pages' "estimation" is not defined there);
 *   - forced blocks = blocks [0, init) and the `local` blocks ending at the query's own block, not
 *     counted against k; the output set is sorted ascending and padded with -1.
 *
 * Parity pins (tests/test_oracle_pins.py): hand-worked two-block example, closed forms of the window
 * mean, special cases that reduce to library softmax attention / average pooling, and invariants; the
 * backward (item 7) against central differences of the forward, library autograd on the dense case,
 * the one-key closed form and the sum rules of the softmax Jacobian; the kernel backward (item 8) against
 * the forward by the adjoint identity on keys whose window means are exact in bf16.
 * The pages' "efficient LogSumExp estimation" is not defined there (parity unpinned): params.lse_stride > 1
 * selects one reading of it, the LSE from every s-th visible kernel times s, pinned only to its special cases
 * (s = 1 is exact; the closed form on equal scores).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ----------------------------------------------------------------------------------------------- */
/* bf16 <-> fp64                                                                                    */
/* ----------------------------------------------------------------------------------------------- */

static double bf16_bits_to_f64(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round an fp64 value to the nearest bf16 (8 significant bits, ties to even), in one rounding step. */
static uint16_t f64_to_bf16_bits_rne(double x)
{
    if (x != x) return 0x7FC0u;
    uint16_t sign = (x < 0.0 || (x == 0.0 && signbit(x))) ? 0x8000u : 0u;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    double r;
    const double min_normal = ldexp(1.0, -126);
    if (a < min_normal) {
        /* bf16 subnormals are multiples of 2^-133 */
        r = nearbyint(a / ldexp(1.0, -133)) * ldexp(1.0, -133);
    } else {
        int e;
        double m = frexp(a, &e);            /* a = m * 2^e, m in [0.5, 1) */
        r = ldexp(nearbyint(m * 256.0), e - 8); /* 8 significant bits, round half to even */
    }
    if (r > 3.3895313892515355e38) return (uint16_t)(sign | 0x7F80u);
    float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

uint16_t orc_round_bf16(double x) { return f64_to_bf16_bits_rne(x); }

/* ----------------------------------------------------------------------------------------------- */
/* parameters                                                                                       */
/* ----------------------------------------------------------------------------------------------- */

typedef struct {
    int block_size;     /* bs: keys per context block */
    int kernel_size;    /* ks: keys per semantic-kernel window */
    int kernel_stride;  /* kst: distance between consecutive windows */
    int topk;           /* k: blocks chosen by score, besides the forced ones */
    int init_blocks;    /* blocks [0, init) are always kept */
    int local_blocks;   /* the `local` blocks ending at the query's own block are always kept */
    int dense_len;      /* a query whose context n <= dense_len attends densely */
    int membership;     /* 0 = OVERLAP (window intersects block), 1 = CONTAINED (window inside block) */
    double scale;       /* softmax scale for both kernel scoring and attention */
    int lse_stride;     /* 0 or 1: exact LSE; s > 1: the estimate log(s * sum over every s-th visible kernel) */
} orc_params;

/* number of complete kernel windows over the first n keys */
static long nk_of(long n, const orc_params* p)
{
    if (n < p->kernel_size) return 0;
    return (n - p->kernel_size) / p->kernel_stride + 1;
}

long orc_num_kernels(long n, int kernel_size, int kernel_stride)
{
    if (n < kernel_size) return 0;
    return (n - kernel_size) / kernel_stride + 1;
}

/* ----------------------------------------------------------------------------------------------- */
/* step 1: semantic kernels                                                                         */
/* ----------------------------------------------------------------------------------------------- */

/*
 * K: [B, Lcap, Hkv, d] bf16 bits.  For each sequence b, the kernels j in [nk(old_len[b]), nk(new_len[b]))
 * are written: kern[b, g, j, :] = bf16_rne( (1/ks) * sum_{i = j*kst}^{j*kst+ks-1} K[b, i, g, :] ).
 * kern: [B, Hkv, nk_cap, d].  Returns 0, or -1 when a kernel index would reach nk_cap or a length
 * exceeds Lcap.
 */
int orc_kernel_pool(const uint16_t* K, int B, int Lcap, int Hkv, int d, const int32_t* old_len,
                    const int32_t* new_len, int kernel_size, int kernel_stride, uint16_t* kern, int nk_cap)
{
    orc_params p;
    memset(&p, 0, sizeof p);
    p.kernel_size = kernel_size;
    p.kernel_stride = kernel_stride;
    for (int b = 0; b < B; ++b) {
        if (new_len[b] > Lcap || old_len[b] < 0 || old_len[b] > new_len[b]) return -1;
        if (nk_of(new_len[b], &p) > nk_cap) return -1;
    }
    for (int b = 0; b < B; ++b) {
        long j0 = nk_of(old_len[b], &p), j1 = nk_of(new_len[b], &p);
        for (int g = 0; g < Hkv; ++g) {
            for (long j = j0; j < j1; ++j) {
                for (int c = 0; c < d; ++c) {
                    double s = 0.0;
                    for (long i = j * kernel_stride; i < j * kernel_stride + kernel_size; ++i)
                        s += bf16_bits_to_f64(K[(((size_t)b * Lcap + i) * Hkv + g) * d + c]);
                    kern[(((size_t)b * Hkv + g) * nk_cap + j) * d + c] = f64_to_bf16_bits_rne(s / kernel_size);
                }
            }
        }
    }
    return 0;
}

/* ----------------------------------------------------------------------------------------------- */
/* step 2-3: group block scores                                                                     */
/* ----------------------------------------------------------------------------------------------- */

/* kernel j belongs to block blk under the chosen membership rule */
static int kernel_in_block(long j, long blk, const orc_params* p)
{
    long w0 = j * p->kernel_stride, w1 = w0 + p->kernel_size; /* window [w0, w1) */
    long b0 = blk * p->block_size, b1 = b0 + p->block_size;   /* block  [b0, b1) */
    if (p->membership == 1) return w0 >= b0 && w1 <= b1;
    return w0 < b1 && w1 > b0;
}

/*
 * Scores for one query row (b, t) and one KV group g.
 *   q: [B, T, Hq, d]; kern: [B, Hkv, nk_cap, d]; n = q_ctx[b*T + t] = number of context keys the query
 *   sees (its own position + 1 for ordinary queries, the prefix length for tree-draft queries).
 *   Writes S[0..c] (c = (n-1)/bs) into S_row and LSE_h for the group's heads into lse_heads.
 */
static void group_scores_row(const uint16_t* q, int T, int Hq, int Hkv, int d, const uint16_t* kern,
                             int nk_cap, const orc_params* p, int b, int t, int g, long n,
                             double* S_row, double* lse_heads, double* zbuf)
{
    const int G = Hq / Hkv;
    const long nkv = nk_of(n, p);         /* visible kernels: complete windows inside [0, n) */
    const long c = (n - 1) / p->block_size; /* the query's own block */
    for (long blk = 0; blk <= c; ++blk) S_row[blk] = 0.0;
    for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        const uint16_t* qh = q + (((size_t)b * T + t) * Hq + h) * d;
        /* z_h(j) = scale * q_h . kappa_j */
        double zmax = -INFINITY;
        for (long j = 0; j < nkv; ++j) {
            const uint16_t* kj = kern + (((size_t)b * Hkv + g) * nk_cap + j) * d;
            double dot = 0.0;
            for (int c2 = 0; c2 < d; ++c2) dot += bf16_bits_to_f64(qh[c2]) * bf16_bits_to_f64(kj[c2]);
            zbuf[j] = p->scale * dot;
            if (zbuf[j] > zmax) zmax = zbuf[j];
        }
        /* LSE_h = log sum_j exp z_h(j), evaluated exactly (max-shifted); with lse_stride s > 1, the estimate
         * log(s * sum_{j = 0, s, 2s, ...} exp z_h(j)) from every s-th visible kernel (a reading of the pages'
         * "LogSumExp estimation", which they do not define) */
        double lse = -INFINITY;
        if (nkv > 0) {
            const long st = p->lse_stride > 1 ? p->lse_stride : 1;
            double s = 0.0;
            for (long j = 0; j < nkv; j += st) s += exp(zbuf[j] - zmax);
            lse = zmax + log(s * (double)st);
        }
        lse_heads[hh] = lse;
        /* block score of head h: max over the block's visible kernels of exp(z - LSE) */
        for (long blk = 0; blk <= c; ++blk) {
            /* j_lo..j_hi is a superset of the block's kernels; membership is decided by kernel_in_block */
            long j_lo = (blk * p->block_size - p->kernel_size) / p->kernel_stride;
            long j_hi = ((blk + 1) * p->block_size) / p->kernel_stride + 1;
            if (j_lo < 0) j_lo = 0;
            if (j_hi > nkv) j_hi = nkv;
            double best = -1.0;
            for (long j = j_lo; j < j_hi; ++j) {
                if (!kernel_in_block(j, blk, p)) continue;
                double v = exp(zbuf[j] - lse);
                if (v > best) best = v;
            }
            if (best < 0.0) {
                S_row[blk] = -INFINITY; /* no visible kernel in this block: not a candidate */
            } else if (S_row[blk] != -INFINITY) {
                S_row[blk] += best;     /* pooled over the group's heads */
            }
        }
    }
}

/* ----------------------------------------------------------------------------------------------- */
/* step 4: selection                                                                                */
/* ----------------------------------------------------------------------------------------------- */

typedef struct { double s; long blk; } cand_t;

/* score descending, then block index ascending */
static int cand_cmp(const void* a, const void* b)
{
    const cand_t* x = (const cand_t*)a;
    const cand_t* y = (const cand_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->blk < y->blk) ? -1 : (x->blk > y->blk);
}

/*
 * Selection for one row.  Writes idx_row[0..kmax) ascending, -1 padded, returns the count.
 * gap[0], gap[1] = scores of the k-th and (k+1)-th ranked candidates (NaN when there are <= k).
 * A dense row (n <= dense_len) selects every block 0..c; its count is c+1 and the first
 * min(c+1, kmax) ids are stored.
 */
static int select_row(const double* S_row, long n, const orc_params* p, int kmax, int32_t* idx_row,
                      double* gap, cand_t* cbuf, unsigned char* chosen)
{
    const long c = (n - 1) / p->block_size;
    for (int i = 0; i < kmax; ++i) idx_row[i] = -1;
    gap[0] = NAN;
    gap[1] = NAN;
    if (n <= p->dense_len) {
        for (long blk = 0; blk <= c && blk < kmax; ++blk) idx_row[blk] = (int32_t)blk;
        return (int)(c + 1);
    }
    for (long blk = 0; blk <= c; ++blk) chosen[blk] = 0;
    /* forced: initial blocks and local blocks */
    for (long blk = 0; blk < p->init_blocks && blk <= c; ++blk) chosen[blk] = 1;
    for (long blk = c - p->local_blocks + 1; blk <= c; ++blk)
        if (blk >= 0) chosen[blk] = 1;
    /* candidates */
    long nc = 0;
    for (long blk = 0; blk <= c; ++blk) {
        if (chosen[blk]) continue;
        if (S_row[blk] == -INFINITY) continue;
        cbuf[nc].s = S_row[blk];
        cbuf[nc].blk = blk;
        ++nc;
    }
    qsort(cbuf, (size_t)nc, sizeof(cand_t), cand_cmp);
    long take = nc < p->topk ? nc : p->topk;
    if (nc > p->topk) {
        gap[0] = p->topk > 0 ? cbuf[p->topk - 1].s : INFINITY;
        gap[1] = cbuf[p->topk].s;
    }
    for (long i = 0; i < take; ++i) chosen[cbuf[i].blk] = 1;
    int cnt = 0;
    for (long blk = 0; blk <= c; ++blk) {
        if (!chosen[blk]) continue;
        if (cnt < kmax) idx_row[cnt] = (int32_t)blk;
        ++cnt;
    }
    return cnt;
}

/*
 * Block scoring and selection for every query row.
 *   q: [B, T, Hq, d] bf16; kern: [B, Hkv, nk_cap, d] bf16; q_ctx: [B*T] context length n of each query.
 *   Outputs (any may be NULL except idx/cnt):
 *     S:    [B, T, Hkv, nb_max] fp64 group scores (-inf beyond c or for blocks without visible kernels)
 *     lse:  [B, T, Hq] fp64 per-head LSE over the visible kernels
 *     idx:  [B, T, Hkv, kmax] int32, cnt: [B, T, Hkv] int32
 *     gap:  [B, T, Hkv, 2] fp64 (k-th, (k+1)-th ranked candidate scores)
 *   Returns 0, or -1 on a bad argument (n < 1, c >= nb_max, Hq % Hkv != 0).
 */
int orc_block_score_topk(const uint16_t* q, int B, int T, int Hq, int Hkv, int d, const uint16_t* kern,
                         int nk_cap, const int32_t* q_ctx, const orc_params* p, int nb_max, int kmax,
                         double* S, double* lse, int32_t* idx, int32_t* cnt, double* gap)
{
    if (Hkv <= 0 || Hq % Hkv != 0) return -1;
    for (long r = 0; r < (long)B * T; ++r) {
        if (q_ctx[r] < 1) return -1;
        if ((q_ctx[r] - 1) / p->block_size >= nb_max) return -1;
        if (nk_of(q_ctx[r], p) > nk_cap) return -1;
    }
    const int G = Hq / Hkv;
    const long rows = (long)B * T * Hkv;
    int status = 0;
#pragma omp parallel
    {
        double* zbuf = (double*)malloc(sizeof(double) * (size_t)(nk_cap > 0 ? nk_cap : 1));
        double* Srow = (double*)malloc(sizeof(double) * (size_t)nb_max);
        double* lrow = (double*)malloc(sizeof(double) * (size_t)G);
        cand_t* cbuf = (cand_t*)malloc(sizeof(cand_t) * (size_t)nb_max);
        unsigned char* chosen = (unsigned char*)malloc((size_t)nb_max);
        double gtmp[2];
        if (!zbuf || !Srow || !lrow || !cbuf || !chosen) {
#pragma omp atomic write
            status = -2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long r = 0; r < rows; ++r) {
                const int g = (int)(r % Hkv);
                const long bt = r / Hkv;
                const int t = (int)(bt % T), b = (int)(bt / T);
                const long n = q_ctx[bt];
                const long c = (n - 1) / p->block_size;
                group_scores_row(q, T, Hq, Hkv, d, kern, nk_cap, p, b, t, g, n, Srow, lrow, zbuf);
                for (long blk = c + 1; blk < nb_max; ++blk) Srow[blk] = -INFINITY;
                int nsel = select_row(Srow, n, p, kmax, idx + r * kmax, gtmp, cbuf, chosen);
                cnt[r] = nsel;
                if (S) memcpy(S + r * nb_max, Srow, sizeof(double) * (size_t)nb_max);
                if (lse)
                    for (int hh = 0; hh < G; ++hh) lse[bt * Hq + g * G + hh] = lrow[hh];
                if (gap) { gap[2 * r] = gtmp[0]; gap[2 * r + 1] = gtmp[1]; }
            }
        }
        free(zbuf); free(Srow); free(lrow); free(cbuf); free(chosen);
    }
    return status;
}

/* ----------------------------------------------------------------------------------------------- */
/* step 5: block-sparse attention (and the tree-draft variant)                                      */
/* ----------------------------------------------------------------------------------------------- */

/*
 * Attention of every query row over the keys of its selected blocks.
 *   q: [B, T, Hq, d]; K, V: [B, Lcap, Hkv, d]; q_ctx: [B*T] context length n of each query.
 *   idx/cnt: the selection ([B, T, Hkv, kmax] / [B, T, Hkv]).
 *   Key set of query (b, t), group g:
 *     n <= dense_len : every key i in [0, n)                 (dense attention)
 *     otherwise      : union over blk in idx of [blk*bs, min((blk+1)*bs, n))
 *   plus, when tree_mask != NULL, the draft keys kd/vd[b, j] ([B, T, Hkv, d]) of every draft node j
 *   whose bit j is set in tree_mask[b*T + t].
 *   out: [B, T, Hq, d] fp64; lse_out: [B, T, Hq] fp64 (natural log of the softmax denominator), may be NULL.
 *   Returns 0, or -1 on a bad argument (a block id out of range, cnt > kmax on a sparse row).
 */
int orc_sparse_attention(const uint16_t* q, int B, int T, int Hq, int Hkv, int d, const uint16_t* K,
                         const uint16_t* V, int Lcap, const int32_t* q_ctx, const int32_t* idx,
                         const int32_t* cnt, int kmax, const orc_params* p, const uint16_t* kd,
                         const uint16_t* vd, const uint32_t* tree_mask, double* out, double* lse_out)
{
    if (Hkv <= 0 || Hq % Hkv != 0) return -1;
    if (tree_mask && T > 32) return -1;
    const int G = Hq / Hkv;
    const long rows = (long)B * T * Hkv;
    for (long r = 0; r < rows; ++r) {
        const long bt = r / Hkv;
        const long n = q_ctx[bt];
        if (n < 1 || n > Lcap) return -1;
        if (n <= p->dense_len) continue;
        if (cnt[r] < 0 || cnt[r] > kmax) return -1;
        for (int i = 0; i < cnt[r]; ++i) {
            long blk = idx[r * kmax + i];
            if (blk < 0 || blk * p->block_size >= n) return -1;
        }
    }
    int status = 0;
#pragma omp parallel
    {
        /* key list of the row: prefix positions, then draft node ids encoded as -(j+1) */
        long* keys = (long*)malloc(sizeof(long) * (size_t)(Lcap + 64));
        double* logit = (double*)malloc(sizeof(double) * (size_t)(Lcap + 64));
        if (!keys || !logit) {
#pragma omp atomic write
            status = -2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long r = 0; r < rows; ++r) {
                const int g = (int)(r % Hkv);
                const long bt = r / Hkv;
                const int t = (int)(bt % T), b = (int)(bt / T);
                const long n = q_ctx[bt];
                long nkeys = 0;
                if (n <= p->dense_len) {
                    for (long i = 0; i < n; ++i) keys[nkeys++] = i;
                } else {
                    for (int s = 0; s < cnt[r]; ++s) {
                        long blk = idx[r * kmax + s];
                        long k0 = blk * p->block_size, k1 = k0 + p->block_size;
                        if (k1 > n) k1 = n;
                        for (long i = k0; i < k1; ++i) keys[nkeys++] = i;
                    }
                }
                if (tree_mask) {
                    uint32_t m = tree_mask[bt];
                    for (int j = 0; j < T; ++j)
                        if ((m >> j) & 1u) keys[nkeys++] = -(long)(j + 1);
                }
                for (int hh = 0; hh < G; ++hh) {
                    const int h = g * G + hh;
                    const uint16_t* qh = q + (((size_t)b * T + t) * Hq + h) * d;
                    double* oh = out + (((size_t)b * T + t) * Hq + h) * d;
                    double mx = -INFINITY;
                    for (long e = 0; e < nkeys; ++e) {
                        const uint16_t* kr = keys[e] >= 0
                            ? K + (((size_t)b * Lcap + keys[e]) * Hkv + g) * d
                            : kd + (((size_t)b * T + (-keys[e] - 1)) * Hkv + g) * d;
                        double dot = 0.0;
                        for (int c2 = 0; c2 < d; ++c2) dot += bf16_bits_to_f64(qh[c2]) * bf16_bits_to_f64(kr[c2]);
                        logit[e] = p->scale * dot;
                        if (logit[e] > mx) mx = logit[e];
                    }
                    for (int c2 = 0; c2 < d; ++c2) oh[c2] = 0.0;
                    double den = 0.0;
                    for (long e = 0; e < nkeys; ++e) {
                        const uint16_t* vr = keys[e] >= 0
                            ? V + (((size_t)b * Lcap + keys[e]) * Hkv + g) * d
                            : vd + (((size_t)b * T + (-keys[e] - 1)) * Hkv + g) * d;
                        double w = exp(logit[e] - mx);
                        den += w;
                        for (int c2 = 0; c2 < d; ++c2) oh[c2] += w * bf16_bits_to_f64(vr[c2]);
                    }
                    if (nkeys == 0) {
                        if (lse_out) lse_out[bt * Hq + h] = -INFINITY;
                        continue;
                    }
                    for (int c2 = 0; c2 < d; ++c2) oh[c2] /= den;
                    if (lse_out) lse_out[bt * Hq + h] = mx + log(den);
                }
            }
        }
        free(keys);
        free(logit);
    }
    return status;
}

/* ----------------------------------------------------------------------------------------------- */
/* backward of the sparse attention for a fixed selection (training)                                */
/* ----------------------------------------------------------------------------------------------- */

/*
 * Gradients of L = sum over (b, t, h, c) of dout * out with respect to q, K and V, where out is the
 * sparse attention above (no tree drafts).  The pages train InfLLM v2 with the same sparse attention
 * ("Tsinghua & ModelBest: MiniCPM4 technical details", "Model architecture: InfLLM v2", item 3: efficient
 * operators for training and inference) but give no formula; this is the derivative of the forward's own
 * definition.  The selection is a piecewise-constant function of q and K, so for a fixed selection no
 * gradient flows through the block scores or the semantic kernels.
 *
 * For a row (b, t, h) with key set K(t) (the forward's), logits s_e = scale q.k_e, probabilities
 * p_e = exp(s_e) / sum exp(s), and out = sum_e p_e v_e:
 *   dp_e  = dout . v_e                       (dL/dp_e)
 *   Dsum  = sum_e p_e dp_e                   (= dout . out)
 *   ds_e  = p_e (dp_e - Dsum)                (dL/ds_e, the softmax Jacobian)
 *   dq   += scale sum_e ds_e k_e
 *   dk_e += scale ds_e q,   dv_e += p_e dout (summed over the rows that read key e)
 * dout: [B, T, Hq, d] bf16 bits.  dq: [B, T, Hq, d] fp64; dk, dv: [B, Lcap, Hkv, d] fp64, overwritten
 * (keys no row reads get 0).  Returns 0, or -1 on a bad argument (as orc_sparse_attention).
 */
int orc_sparse_attention_backward(const uint16_t* q, int B, int T, int Hq, int Hkv, int d, const uint16_t* K,
                                  const uint16_t* V, int Lcap, const int32_t* q_ctx, const int32_t* idx,
                                  const int32_t* cnt, int kmax, const orc_params* p, const uint16_t* dout,
                                  double* dq, double* dk, double* dv)
{
    if (Hkv <= 0 || Hq % Hkv != 0) return -1;
    const int G = Hq / Hkv;
    const long rows = (long)B * T * Hkv;
    for (long r = 0; r < rows; ++r) {
        const long bt = r / Hkv;
        const long n = q_ctx[bt];
        if (n < 1 || n > Lcap) return -1;
        if (n <= p->dense_len) continue;
        if (cnt[r] < 0 || cnt[r] > kmax) return -1;
        for (int i = 0; i < cnt[r]; ++i) {
            long blk = idx[r * kmax + i];
            if (blk < 0 || blk * p->block_size >= n) return -1;
        }
    }
    memset(dk, 0, sizeof(double) * (size_t)B * Lcap * Hkv * d);
    memset(dv, 0, sizeof(double) * (size_t)B * Lcap * Hkv * d);
    int status = 0;
    /* one (sequence, KV group) per task: the rows of a task are the only writers of its dk / dv slice */
#pragma omp parallel
    {
        long* keys = (long*)malloc(sizeof(long) * (size_t)(Lcap + 1));
        double* prob = (double*)malloc(sizeof(double) * (size_t)(Lcap + 1));
        double* dprob = (double*)malloc(sizeof(double) * (size_t)(Lcap + 1));
        if (!keys || !prob || !dprob) {
#pragma omp atomic write
            status = -2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bg = 0; bg < (long)B * Hkv; ++bg) {
                const int b = (int)(bg / Hkv), g = (int)(bg % Hkv);
                for (int t = 0; t < T; ++t) {
                    const long bt = (long)b * T + t;
                    const long r = bt * Hkv + g;
                    const long n = q_ctx[bt];
                    long nkeys = 0;
                    if (n <= p->dense_len) {
                        for (long i = 0; i < n; ++i) keys[nkeys++] = i;
                    } else {
                        for (int s = 0; s < cnt[r]; ++s) {
                            long blk = idx[r * kmax + s];
                            long k0 = blk * p->block_size, k1 = k0 + p->block_size;
                            if (k1 > n) k1 = n;
                            for (long i = k0; i < k1; ++i) keys[nkeys++] = i;
                        }
                    }
                    for (int hh = 0; hh < G; ++hh) {
                        const int h = g * G + hh;
                        const uint16_t* qh = q + ((size_t)bt * Hq + h) * d;
                        const uint16_t* doh = dout + ((size_t)bt * Hq + h) * d;
                        double* dqh = dq + ((size_t)bt * Hq + h) * d;
                        for (int c2 = 0; c2 < d; ++c2) dqh[c2] = 0.0;
                        if (nkeys == 0) continue;
                        /* probabilities of the forward */
                        double mx = -INFINITY;
                        for (long e = 0; e < nkeys; ++e) {
                            const uint16_t* kr = K + (((size_t)b * Lcap + keys[e]) * Hkv + g) * d;
                            double dot = 0.0;
                            for (int c2 = 0; c2 < d; ++c2) dot += bf16_bits_to_f64(qh[c2]) * bf16_bits_to_f64(kr[c2]);
                            prob[e] = p->scale * dot;
                            if (prob[e] > mx) mx = prob[e];
                        }
                        double den = 0.0;
                        for (long e = 0; e < nkeys; ++e) {
                            prob[e] = exp(prob[e] - mx);
                            den += prob[e];
                        }
                        for (long e = 0; e < nkeys; ++e) prob[e] /= den;
                        /* dL/dp and the softmax Jacobian */
                        double dsum = 0.0;
                        for (long e = 0; e < nkeys; ++e) {
                            const uint16_t* vr = V + (((size_t)b * Lcap + keys[e]) * Hkv + g) * d;
                            double dot = 0.0;
                            for (int c2 = 0; c2 < d; ++c2) dot += bf16_bits_to_f64(doh[c2]) * bf16_bits_to_f64(vr[c2]);
                            dprob[e] = dot;
                            dsum += prob[e] * dot;
                        }
                        for (long e = 0; e < nkeys; ++e) {
                            const double ds = prob[e] * (dprob[e] - dsum);
                            const size_t kv = (((size_t)b * Lcap + keys[e]) * Hkv + g) * d;
                            for (int c2 = 0; c2 < d; ++c2) {
                                dqh[c2] += p->scale * ds * bf16_bits_to_f64(K[kv + c2]);
                                dk[kv + c2] += p->scale * ds * bf16_bits_to_f64(qh[c2]);
                                dv[kv + c2] += prob[e] * bf16_bits_to_f64(doh[c2]);
                            }
                        }
                    }
                }
            }
        }
        free(keys);
        free(prob);
        free(dprob);
    }
    return status;
}

/* ----------------------------------------------------------------------------------------------- */
/* plain causal attention, written separately (used to pin the sparse routine and as the dense path) */
/* ----------------------------------------------------------------------------------------------- */

/* out[b,t,h,:] = sum_{lo <= i < n} softmax_i(scale q.k_i) v_i with n = q_ctx[b*T+t] and lo = 0, or
 * lo = max(0, n - window) when window > 0; GQA head h -> group h/G. */
static int range_attention(const uint16_t* q, int B, int T, int Hq, int Hkv, int d, const uint16_t* K,
                           const uint16_t* V, int Lcap, const int32_t* q_ctx, long window, double scale,
                           double* out, double* lse_out)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || window < 0) return -1;
    const int G = Hq / Hkv;
    for (long r = 0; r < (long)B * T; ++r)
        if (q_ctx[r] < 1 || q_ctx[r] > Lcap) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < (long)B * T * Hq; ++r) {
        const int h = (int)(r % Hq);
        const long bt = r / Hq;
        const int b = (int)(bt / T);
        const long n = q_ctx[bt];
        const long lo = (window > 0 && n > window) ? n - window : 0;
        const uint16_t* qh = q + (size_t)r * d;
        double* oh = out + (size_t)r * d;
        double mx = -INFINITY;
        for (long i = lo; i < n; ++i) {
            const uint16_t* kr = K + (((size_t)b * Lcap + i) * Hkv + h / G) * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += bf16_bits_to_f64(qh[c]) * bf16_bits_to_f64(kr[c]);
            if (scale * dot > mx) mx = scale * dot;
        }
        double den = 0.0;
        for (int c = 0; c < d; ++c) oh[c] = 0.0;
        for (long i = lo; i < n; ++i) {
            const uint16_t* kr = K + (((size_t)b * Lcap + i) * Hkv + h / G) * d;
            const uint16_t* vr = V + (((size_t)b * Lcap + i) * Hkv + h / G) * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += bf16_bits_to_f64(qh[c]) * bf16_bits_to_f64(kr[c]);
            double w = exp(scale * dot - mx);
            den += w;
            for (int c = 0; c < d; ++c) oh[c] += w * bf16_bits_to_f64(vr[c]);
        }
        for (int c = 0; c < d; ++c) oh[c] /= den;
        if (lse_out) lse_out[r] = mx + log(den);
    }
    return 0;
}

/* plain causal attention over keys [0, n) */
int orc_dense_attention(const uint16_t* q, int B, int T, int Hq, int Hkv, int d, const uint16_t* K,
                        const uint16_t* V, int Lcap, const int32_t* q_ctx, double scale, double* out,
                        double* lse_out)
{
    return range_attention(q, B, T, Hq, Hkv, d, K, V, Lcap, q_ctx, 0, scale, out, lse_out);
}

/* sliding-window attention of the draft model: keys [max(0, n - window), n), window >= 1
 *   -- QbitAI article, section "speculative sampling, quantisation and long text", long-context bullet
 *      (the draft model attends with a sliding window; the pages give no window size) */
int orc_window_attention(const uint16_t* q, int B, int T, int Hq, int Hkv, int d, const uint16_t* K,
                         const uint16_t* V, int Lcap, const int32_t* q_ctx, int window, double scale, double* out,
                         double* lse_out)
{
    if (window < 1) return -1;
    return range_attention(q, B, T, Hq, Hkv, d, K, V, Lcap, q_ctx, window, scale, out, lse_out);
}

/* ----------------------------------------------------------------------------------------------- */
/* step 8: gradient of the semantic kernels with respect to K                                       */
/* ----------------------------------------------------------------------------------------------- */

/*
 * The transpose of step 1's window mean (its bf16 rounding taken as the identity): every kernel j in
 * [0, nk(lens[b])) hands 1/ks of its gradient to each of the ks keys of its window,
 *   dk[b, i, g, :] = sum_{j : j*kst <= i < j*kst + ks} dkern[b, g, j, :] / ks.
 * dkern: [B, Hkv, nk_cap, d] fp32; dk: [B, Lcap, Hkv, d] fp64, overwritten (rows no kernel reads are 0).
 * Returns 0, or -1 when a length exceeds Lcap or nk(lens[b]) exceeds nk_cap.
 */
int orc_kernel_pool_backward(const float* dkern, int B, int Lcap, int Hkv, int d, const int32_t* lens,
                             int kernel_size, int kernel_stride, int nk_cap, double* dk)
{
    orc_params p;
    memset(&p, 0, sizeof p);
    p.kernel_size = kernel_size;
    p.kernel_stride = kernel_stride;
    for (int b = 0; b < B; ++b)
        if (lens[b] < 0 || lens[b] > Lcap || nk_of(lens[b], &p) > nk_cap) return -1;
    memset(dk, 0, sizeof(double) * (size_t)B * Lcap * Hkv * d);
    for (int b = 0; b < B; ++b) {
        const long nk = nk_of(lens[b], &p);
        for (int g = 0; g < Hkv; ++g)
            for (long j = 0; j < nk; ++j)
                for (long i = j * kernel_stride; i < j * kernel_stride + kernel_size; ++i)
                    for (int c = 0; c < d; ++c)
                        dk[(((size_t)b * Lcap + i) * Hkv + g) * d + c] +=
                            (double)dkern[(((size_t)b * Hkv + g) * nk_cap + j) * d + c] / kernel_size;
    }
    return 0;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
