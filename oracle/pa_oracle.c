/*
 * CPU oracle for ProxyAttn-style block-sparse prefill attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  The product path
 * (the CUDA library and its Python binding) never calls it, and this file
 * shares no code, header, table or constant with the CUDA path.
 *
 * Plain, slow, obviously-correct loops in fp64.  Every function follows one
 * step of the method as the ProxyAttn pages state it:
 *
 *   o1 pa_oracle_pool         ProxyAttn blog (HIT), "4. ProxyAttn method",
 *                             Step 1 "Head Pooling": Q and K are aggregated over
 *                             the heads of a layer (or of a group) into a proxy
 *                             head; "simple pooling" (section 3) read as the mean.
 *   o2 pa_oracle_block_scores Step 1 "Score Estimation": token-level proxy
 *                             scores, then max-pooling to 128x128 block
 *                             importance (block size from "2. Background:
 *                             why block-wise").
 *   o3 pa_oracle_head_mass    Step 2 "dynamic budget": the last Q block estimates
 *                             each head's block-level sparsity; here the exact
 *                             softmax mass each KV block receives from the last
 *                             128 query rows of that head.
 *   o4 pa_oracle_rank         Step 1 "Block Ranking": KV blocks of every query
 *      pa_oracle_budget       block sorted by proxy importance; Step 2: per-head
 *                             budget over the shared ranking; final mask = ranking
 *                             prefix of the head's length.  The budget rule
 *                             "smallest set whose cumulative mass reaches the
 *                             threshold" is XAttention's find_blocks (XAttention
 *                             blog, 2.2 "threshold block selection", equation).
 *   o5 pa_oracle_sparse_attn  Step 2 end: the block-sparse mask is fed to a
 *                             FlashAttention-style kernel; attention = softmax of
 *                             the scaled Q.K products (section 2 "Background"),
 *                             restricted to the selected causal keys.
 *   o6 pa_oracle_dense_attn   Plain causal softmax attention, written separately.
 *   o8 pa_oracle_xattn_mass   XAttention's antidiagonal block estimate (XAttention
 *      pa_oracle_find_blocks  blog 2.1-2.2) and its threshold selection find_blocks.
 *   o7 pa_oracle_sparse_attn_skip  o5 with BLASST's running-max block skip
 *                             (BLASST introduction, 3.1): a visited block far
 *                             below the running max is left out.
 *
 * Readings where the pages are silent, each the plainest one that the
 * surviving text supports:
 *   mean pooling; K pooled over the expanded KV heads of the group's q heads;
 *   pre-softmax scaled logits as token scores; proxies rounded to bf16 (RNE)
 *   before scoring; budget from exactly the last 128-row Q block; budget
 *   k_h counted at the last row and scaled to row qb as ceil(k_h*(qb+1)/nb);
 *   sink block 0 and diagonal block qb lead every list and count toward the
 *   budget; ties broken by lower block index; masses compared in 2^-40 fixed
 *   point; softmax scale 1/sqrt(d) unless given.
 *
 * Layouts: q is [B][N][H][d] bf16 bits addressed with element strides
 * (sb, ss, sh) and unit stride along d; k, v likewise with Hkv heads.
 * Proxies are [B][G][N][d].  Block scores and ranked lists are [B][G][T] with
 * T = nb(nb+1)/2 and row qb starting at tri(qb) = qb(qb+1)/2.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define BLK 128

static double bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even (IEEE 754
 * roundTiesToEven), straight from the definition: bf16 keeps 8 significant
 * bits, so the spacing of representable values in the binade [2^e, 2^(e+1))
 * is 2^(e-7); below 2^-126 the spacing stays 2^-133 (subnormals).  x / 2^(e-7)
 * is exact, nearbyint() rounds it to an integer with ties to even, and the
 * product is the rounded value, which float holds exactly. */
uint16_t pa_oracle_f64_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    int e;
    (void)frexp(x, &e);       /* |x| in [2^(e-1), 2^e) */
    int e2 = e - 1;
    if (x == 0.0) e2 = -126;
    if (e2 < -126) e2 = -126;
    double q = ldexp(1.0, e2 - 7);
    double r = nearbyint(x / q) * q;
    float f = (float)r;        /* exact; overflows to inf past the bf16 range */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

static inline int64_t tri(int64_t qb) { return qb * (qb + 1) / 2; }

/* Per-(b, g) arrays of block scores and ranked lists.  Causal: row qb holds
 * the blocks 0..qb at offset tri(qb) (T = tri(nb) entries).  Non-causal
 * (every query attends to every key; the pages' DiT use, XAttention blog
 * "video generation"): row qb holds all nb blocks at offset qb*nb. */
static inline int64_t row_at(int causal, int nb, int qb) { return causal ? tri(qb) : (int64_t)qb * nb; }
static inline int64_t rows_total(int causal, int nb) { return causal ? tri(nb) : (int64_t)nb * nb; }
static inline int row_len(int causal, int nb, int qb) { return causal ? qb + 1 : nb; }

/* q head h -> its KV head (GQA) and its proxy group. */
static inline int kv_of(int h, int H, int Hkv) { return (int)((int64_t)h * Hkv / H); }
static inline int grp_of(int h, int H, int G) { return (int)((int64_t)h * G / H); }

/* ---------------------------------------------------------------- o1 pool */
/* Q_p[b,g,i,:] = mean over q heads h of group g of Q[b,i,h,:];
 * K_p[b,g,j,:] = mean over the same q heads h of K[b,j,kv(h),:].
 * Sums run over h in ascending order, then divide by the head count. */
void pa_oracle_pool(int B, int N, int H, int Hkv, int d, int G,
                    const uint16_t *q, int64_t qsb, int64_t qss, int64_t qsh,
                    const uint16_t *k, int64_t ksb, int64_t kss, int64_t ksh,
                    double *qp, double *kp, uint16_t *qp_bf16, uint16_t *kp_bf16)
{
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; b++)
        for (int i = 0; i < N; i++)
            for (int g = 0; g < G; g++) {
                for (int c = 0; c < d; c++) {
                    double sq = 0.0, sk = 0.0;
                    int n = 0;
                    for (int h = 0; h < H; h++) {
                        if (grp_of(h, H, G) != g) continue;
                        sq += bf16_to_f64(q[b * qsb + i * qss + h * qsh + c]);
                        sk += bf16_to_f64(k[b * ksb + i * kss + (int64_t)kv_of(h, H, Hkv) * ksh + c]);
                        n++;
                    }
                    double mq = sq / n, mk = sk / n;
                    int64_t o = (((int64_t)b * G + g) * N + i) * d + c;
                    if (qp) qp[o] = mq;
                    if (kp) kp[o] = mk;
                    if (qp_bf16) qp_bf16[o] = pa_oracle_f64_to_bf16(mq);
                    if (kp_bf16) kp_bf16[o] = pa_oracle_f64_to_bf16(mk);
                }
            }
}

/* ------------------------------------------------------- o2 block scores */
/* s_ij = scale * sum_c Qp[i,c] Kp[j,c] from the bf16 proxies (the values the
 * GPU multiplies), causal j <= i; score(qb,kb) = max of s_ij over the valid
 * entries of the 128x128 tile.  scores[b][g][tri(qb)+kb], kb <= qb.
 *
 * Query-row stride (ProxyAttn blog, "5. Experiments", estimation cost: the
 * pages credit a sequence-level "sliding skip" for the low estimation cost
 * and do not define it).  Reading: with stride r only the query rows i with
 * i mod r == r-1 of each tile are scored -- the last row of every window of r
 * rows, the one whose causal key range covers the others'.  r = 1 scores
 * every row. */
static double tile_score(const uint16_t *qp, const uint16_t *kp, int d, int qb, int kb, double scale,
                         int stride, int causal)
{
    double best = -INFINITY;
    for (int ii = stride - 1; ii < BLK; ii += stride) {
        int i = qb * BLK + ii;
        for (int jj = 0; jj < BLK; jj++) {
            int j = kb * BLK + jj;
            if (causal && j > i) continue;
            double s = 0.0;
            for (int c = 0; c < d; c++)
                s += bf16_to_f64(qp[(int64_t)i * d + c]) * bf16_to_f64(kp[(int64_t)j * d + c]);
            s *= scale;
            if (s > best) best = s;
        }
    }
    return best;
}

void pa_oracle_block_scores(int B, int N, int G, int d,
                            const uint16_t *qp, const uint16_t *kp, double scale,
                            int stride, int causal, double *scores)
{
    int nb = N / BLK;
    int64_t T = rows_total(causal, nb);
    #pragma omp parallel for collapse(3) schedule(dynamic, 1)
    for (int b = 0; b < B; b++)
        for (int g = 0; g < G; g++)
            for (int qb = 0; qb < nb; qb++) {
                const uint16_t *qpg = qp + ((int64_t)b * G + g) * N * d;
                const uint16_t *kpg = kp + ((int64_t)b * G + g) * N * d;
                for (int kb = 0; kb < row_len(causal, nb, qb); kb++)
                    scores[((int64_t)b * G + g) * T + row_at(causal, nb, qb) + kb] =
                        tile_score(qpg, kpg, d, qb, kb, scale, stride, causal);
            }
}

/* Score of a list of single tiles (b, g, qb, kb): used to sample large sizes. */
void pa_oracle_block_score_tiles(int N, int G, int d, const uint16_t *qp, const uint16_t *kp,
                                 double scale, int stride, int causal, int n_tiles,
                                 const int32_t *tiles /* [n][4] */, double *out)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < n_tiles; t++) {
        int b = tiles[4 * t], g = tiles[4 * t + 1], qb = tiles[4 * t + 2], kb = tiles[4 * t + 3];
        const uint16_t *qpg = qp + ((int64_t)b * G + g) * N * d;
        const uint16_t *kpg = kp + ((int64_t)b * G + g) * N * d;
        out[t] = tile_score(qpg, kpg, d, qb, kb, scale, stride, causal);
    }
}

/* --------------------------------------------------------- o3 head mass */
/* For head h and each row i of the last query block: p_ij = softmax over the
 * causal keys j <= i of scale * Q[b,i,h,:].K[b,j,kv(h),:].  The mass of KV block
 * kb is the mean over the 128 rows of sum_{j in kb} p_ij, so the masses of a
 * head sum to one.  mass[b][h][kb].  rowsum_dev (nullable) receives, per
 * (b,h), max_i |sum_j p_ij - 1|. */
void pa_oracle_head_mass(int B, int N, int H, int Hkv, int d,
                         const uint16_t *q, int64_t qsb, int64_t qss, int64_t qsh,
                         const uint16_t *k, int64_t ksb, int64_t kss, int64_t ksh,
                         double scale, int causal, double *mass, double *rowsum_dev)
{
    int nb = N / BLK;
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++) {
            int kvh = kv_of(h, H, Hkv);
            double *m = mass + ((int64_t)b * H + h) * nb;
            double *z = (double *)malloc(sizeof(double) * N);
            double dev = 0.0;
            for (int kb = 0; kb < nb; kb++) m[kb] = 0.0;
            for (int i = N - BLK; i < N; i++) {
                int jhi = causal ? i + 1 : N;  /* keys j < jhi */
                double zmax = -INFINITY;
                for (int j = 0; j < jhi; j++) {
                    double s = 0.0;
                    for (int c = 0; c < d; c++)
                        s += bf16_to_f64(q[b * qsb + (int64_t)i * qss + h * qsh + c]) *
                             bf16_to_f64(k[b * ksb + (int64_t)j * kss + kvh * ksh + c]);
                    z[j] = s * scale;
                    if (z[j] > zmax) zmax = z[j];
                }
                double den = 0.0;
                for (int j = 0; j < jhi; j++) den += exp(z[j] - zmax);
                double rs = 0.0;
                for (int j = 0; j < jhi; j++) {
                    double p = exp(z[j] - zmax) / den;
                    m[j / BLK] += p / BLK;
                    rs += p;
                }
                if (fabs(rs - 1.0) > dev) dev = fabs(rs - 1.0);
            }
            if (rowsum_dev) rowsum_dev[(int64_t)b * H + h] = dev;
            free(z);
        }
}

/* -------------------------------------------------------- o4 rank/budget */
typedef struct { double s; int32_t kb; } keyed;

/* (score descending, block index ascending): a total order on finite scores. */
static int by_score_desc_then_index(const void *pa, const void *pb)
{
    const keyed *a = (const keyed *)pa, *b = (const keyed *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->kb < b->kb) ? -1 : (a->kb > b->kb);
}

/* Ranked list of query block qb of every (b, g): [0, qb, then the other
 * blocks of the row (1..qb-1 causal, all but 0 and qb non-causal) in (score
 * desc, index asc) order]; at qb = 0 the sink is the diagonal and leads
 * alone.  rank[b][g][row_at(qb)+t]. */
void pa_oracle_rank(int B, int G, int nb, const double *scores, int causal, int32_t *rank)
{
    int64_t T = rows_total(causal, nb);
    #pragma omp parallel for collapse(3) schedule(dynamic, 4)
    for (int b = 0; b < B; b++)
        for (int g = 0; g < G; g++)
            for (int qb = 0; qb < nb; qb++) {
                const double *row = scores + ((int64_t)b * G + g) * T + row_at(causal, nb, qb);
                int32_t *out = rank + ((int64_t)b * G + g) * T + row_at(causal, nb, qb);
                int len = row_len(causal, nb, qb);
                out[0] = 0;
                if (qb > 0) out[1] = qb;
                int lead = qb > 0 ? 2 : 1;
                int n = len - lead;
                if (n == 0) continue;
                keyed *tmp = (keyed *)malloc(sizeof(keyed) * n);
                int m = 0;
                for (int kb = 1; kb < len; kb++)
                    if (kb != qb) { tmp[m].s = row[kb]; tmp[m].kb = kb; m++; }
                qsort(tmp, n, sizeof(keyed), by_score_desc_then_index);
                for (int t = 0; t < n; t++) out[lead + t] = tmp[t].kb;
                free(tmp);
            }
}

/* Budget modes. */
enum { ORACLE_DYNAMIC = 0, ORACLE_FIXED_FRACTION = 1, ORACLE_ALL = 2 };

static inline int forced(int qb) { return qb == 0 ? 1 : 2; }

static inline int clampi(int64_t x, int lo, int hi) { return (int)(x < lo ? lo : (x > hi ? hi : x)); }

/* Per-head budget k_h and per-row counts cnt[b][h][qb].
 * DYNAMIC: fixed-point masses m_fx = rint(mass * 2^40), gamma_fx = rint(gamma *
 *   2^40); k_h = the smallest k >= |F_last| whose prefix of the last row's list
 *   (group grp(h)) carries sum m_fx >= gamma_fx, or nb if none does;
 *   cnt = clamp(ceil(k_h (qb+1) / nb), |F_qb|, qb+1) causal; non-causal every
 *   row has nb blocks, so cnt = clamp(k_h, |F_qb|, nb).
 * FIXED_FRACTION: cnt = clamp(ceil(p (qb+1) / 1000), |F_qb|, qb+1), p per mille
 *   (non-causal: ceil(p nb / 1000), up to nb).
 * ALL: cnt = the row's length.  budget[b][h] = cnt at the last row. */
void pa_oracle_budget(int B, int H, int G, int nb, int mode, double gamma, int frac_permille,
                      const int32_t *rank, const double *mass, int causal, int32_t *budget, int32_t *cnt)
{
    int64_t T = rows_total(causal, nb);
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++) {
            int g = grp_of(h, H, G);
            int32_t *c = cnt + ((int64_t)b * H + h) * nb;
            if (mode == ORACLE_DYNAMIC) {
                const int32_t *last = rank + ((int64_t)b * G + g) * T + row_at(causal, nb, nb - 1);
                const double *m = mass + ((int64_t)b * H + h) * nb;
                int64_t gfx = llrint(gamma * 1099511627776.0);
                int64_t cum = 0;
                int kh = nb;
                for (int t = 0; t < nb; t++) {
                    cum += llrint(m[last[t]] * 1099511627776.0);
                    if (t + 1 >= forced(nb - 1) && cum >= gfx) { kh = t + 1; break; }
                }
                budget[(int64_t)b * H + h] = kh;
                for (int qb = 0; qb < nb; qb++)
                    c[qb] = causal ? clampi(((int64_t)kh * (qb + 1) + nb - 1) / nb, forced(qb), qb + 1)
                                   : clampi(kh, forced(qb), nb);
            } else if (mode == ORACLE_FIXED_FRACTION) {
                for (int qb = 0; qb < nb; qb++)
                    c[qb] = causal ? clampi(((int64_t)frac_permille * (qb + 1) + 999) / 1000, forced(qb), qb + 1)
                                   : clampi(((int64_t)frac_permille * nb + 999) / 1000, forced(qb), nb);
                budget[(int64_t)b * H + h] = c[nb - 1];
            } else {
                for (int qb = 0; qb < nb; qb++) c[qb] = row_len(causal, nb, qb);
                budget[(int64_t)b * H + h] = nb;
            }
        }
}

/* ------------------------------------------------------ o5 sparse attention */
/* For each requested item (b, h, qb): S = the first cnt[b][h][qb] blocks of
 * the ranked list of group grp(h); for every row i of block qb,
 * O[i] = sum_j softmax_j(scale q_i.k_j) v_j over keys j in S with j <= i;
 * lse[i] = log sum_j exp(scale q_i.k_j).  out: [n_items][128][d], lse
 * [n_items][128].  P is not rounded. */
void pa_oracle_sparse_attn(int N, int H, int Hkv, int d, int G,
                           const uint16_t *q, int64_t qsb, int64_t qss, int64_t qsh,
                           const uint16_t *k, int64_t ksb, int64_t kss, int64_t ksh,
                           const uint16_t *v, int64_t vsb, int64_t vss, int64_t vsh,
                           const int32_t *rank, const int32_t *cnt, double scale, int causal,
                           int n_items, const int32_t *items /* [n][3] = b,h,qb */,
                           double *out, double *lse)
{
    int nb = N / BLK;
    int64_t T = rows_total(causal, nb);
    /* every (item, row) pair is independent: one item keeps every thread busy */
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int it = 0; it < n_items; it++)
        for (int ii = 0; ii < BLK; ii++) {
            int b = items[3 * it], h = items[3 * it + 1], qb = items[3 * it + 2];
            int g = grp_of(h, H, G), kvh = kv_of(h, H, Hkv);
            const int32_t *list = rank + ((int64_t)b * G + g) * T + row_at(causal, nb, qb);
            int n = cnt[((int64_t)b * H + h) * nb + qb];
            double *z = (double *)malloc(sizeof(double) * (n > 0 ? n : 1) * BLK);
            int i = qb * BLK + ii;
            double zmax = -INFINITY;
            for (int t = 0; t < n; t++)
                for (int jj = 0; jj < BLK; jj++) {
                    int j = list[t] * BLK + jj;
                    double s = -INFINITY;
                    if (!causal || j <= i) {
                        s = 0.0;
                        for (int c = 0; c < d; c++)
                            s += bf16_to_f64(q[b * qsb + (int64_t)i * qss + h * qsh + c]) *
                                 bf16_to_f64(k[b * ksb + (int64_t)j * kss + kvh * ksh + c]);
                        s *= scale;
                    }
                    z[t * BLK + jj] = s;
                    if (s > zmax) zmax = s;
                }
            double den = 0.0;
            for (int t = 0; t < n * BLK; t++) den += (z[t] == -INFINITY) ? 0.0 : exp(z[t] - zmax);
            double *o = out + ((int64_t)it * BLK + ii) * d;
            for (int c = 0; c < d; c++) o[c] = 0.0;
            for (int t = 0; t < n; t++)
                for (int jj = 0; jj < BLK; jj++) {
                    double zz = z[t * BLK + jj];
                    if (zz == -INFINITY) continue;
                    double p = exp(zz - zmax) / den;
                    int j = list[t] * BLK + jj;
                    for (int c = 0; c < d; c++)
                        o[c] += p * bf16_to_f64(v[b * vsb + (int64_t)j * vss + kvh * vsh + c]);
                }
            if (lse) lse[(int64_t)it * BLK + ii] = zmax + log(den);
            free(z);
        }
}

/* ------------------------------------------------ o7 running-max block skip */
/* BLASST (BLASST introduction; "3.1 pruning attention with the running max"):
 * while the online softmax walks the blocks, a block whose largest score lies
 * far below the running maximum of the blocks before it adds almost nothing
 * after normalisation, so its exponentials and its V product are skipped.
 * The rule's own text is cut off on the pages; readings:
 *  - visit order: the selected blocks of (b, h, qb) by ascending block index;
 *  - running max M_i of row i: the max of its scaled logits over the blocks
 *    visited before (a skipped block never raises it);
 *  - a block after the first is skipped when every row i of the query block
 *    has max_{j in block, j <= i} z_ij - M_i < ln(lambda), lambda in [0, 1]
 *    ("softmax thresholding": the block's largest probability relative to
 *    the running max is below lambda); lambda = 0 never skips;
 *  - the output is the softmax over the keys of the blocks not skipped.
 * skip_in (nullable, [B][H][T], entry tri(qb)+kb): decisions to apply instead
 * of the oracle's own.  skip_out and gap (nullable, [B][H][T]) receive, for
 * every visited block, the oracle's own decision and its margin
 * (max_i (max_j z_ij - M_i) - ln(lambda)) * log2(e) (+inf for the first
 * block); entries of blocks not visited are left as they are. */
void pa_oracle_sparse_attn_skip(int N, int H, int Hkv, int d, int G,
                                const uint16_t *q, int64_t qsb, int64_t qss, int64_t qsh,
                                const uint16_t *k, int64_t ksb, int64_t kss, int64_t ksh,
                                const uint16_t *v, int64_t vsb, int64_t vss, int64_t vsh,
                                const int32_t *rank, const int32_t *cnt, double scale, double lambda,
                                int causal, int n_items, const int32_t *items /* [n][3] = b,h,qb */,
                                const uint8_t *skip_in, uint8_t *skip_out, double *gap,
                                double *out, double *lse)
{
    int nb = N / BLK;
    int64_t T = rows_total(causal, nb);
    double lnl = (lambda > 0.0) ? log(lambda) : -INFINITY;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < n_items; it++) {
        int b = items[3 * it], h = items[3 * it + 1], qb = items[3 * it + 2];
        int g = grp_of(h, H, G), kvh = kv_of(h, H, Hkv);
        const int32_t *list = rank + ((int64_t)b * G + g) * T + row_at(causal, nb, qb);
        int n = cnt[((int64_t)b * H + h) * nb + qb];
        int64_t base = ((int64_t)b * H + h) * T + row_at(causal, nb, qb);
        int *blk = (int *)malloc(sizeof(int) * (n > 0 ? n : 1));
        double *mt = (double *)malloc(sizeof(double) * BLK * (n > 0 ? n : 1));
        unsigned char *use = (unsigned char *)malloc(n > 0 ? n : 1);
        double *row_max = (double *)malloc(sizeof(double) * BLK);
        /* visit order: ascending block index (insertion sort of the list prefix) */
        for (int t = 0; t < n; t++) {
            int x = list[t], u = t;
            while (u > 0 && blk[u - 1] > x) { blk[u] = blk[u - 1]; u--; }
            blk[u] = x;
        }
        /* every row's maximum scaled logit in every visited block */
        for (int ii = 0; ii < BLK; ii++) {
            int i = qb * BLK + ii;
            for (int t = 0; t < n; t++) {
                double best = -INFINITY;
                for (int jj = 0; jj < BLK; jj++) {
                    int j = blk[t] * BLK + jj;
                    if (causal && j > i) continue;
                    double s = 0.0;
                    for (int c = 0; c < d; c++)
                        s += bf16_to_f64(q[b * qsb + (int64_t)i * qss + h * qsh + c]) *
                             bf16_to_f64(k[b * ksb + (int64_t)j * kss + kvh * ksh + c]);
                    s *= scale;
                    if (s > best) best = s;
                }
                mt[ii * n + t] = best;
            }
        }
        /* decisions in visit order against each row's running max */
        for (int ii = 0; ii < BLK; ii++) row_max[ii] = -INFINITY;
        for (int t = 0; t < n; t++) {
            int own = 0;
            double margin = INFINITY;
            if (t > 0) {
                double worst = -INFINITY;
                for (int ii = 0; ii < BLK; ii++) {
                    double e = mt[ii * n + t] - row_max[ii];
                    if (e > worst) worst = e;
                }
                own = worst < lnl;
                margin = (worst - lnl) * 1.4426950408889634;
            }
            for (int ii = 0; ii < BLK; ii++)
                if (mt[ii * n + t] > row_max[ii]) row_max[ii] = mt[ii * n + t];
            if (skip_out) skip_out[base + blk[t]] = (uint8_t)own;
            if (gap) gap[base + blk[t]] = margin;
            use[t] = skip_in ? !skip_in[base + blk[t]] : !own;
        }
        /* softmax over the keys of the blocks kept */
        for (int ii = 0; ii < BLK; ii++) {
            int i = qb * BLK + ii;
            double zmax = -INFINITY;
            for (int t = 0; t < n; t++)
                if (use[t] && mt[ii * n + t] > zmax) zmax = mt[ii * n + t];
            double den = 0.0;
            double *o = out + ((int64_t)it * BLK + ii) * d;
            for (int c = 0; c < d; c++) o[c] = 0.0;
            for (int pass = 0; pass < 2; pass++)
                for (int t = 0; t < n; t++) {
                    if (!use[t]) continue;
                    for (int jj = 0; jj < BLK; jj++) {
                        int j = blk[t] * BLK + jj;
                        if (causal && j > i) continue;
                        double s = 0.0;
                        for (int c = 0; c < d; c++)
                            s += bf16_to_f64(q[b * qsb + (int64_t)i * qss + h * qsh + c]) *
                                 bf16_to_f64(k[b * ksb + (int64_t)j * kss + kvh * ksh + c]);
                        double e = exp(s * scale - zmax);
                        if (pass == 0) {
                            den += e;
                        } else {
                            double pr = e / den;
                            for (int c = 0; c < d; c++)
                                o[c] += pr * bf16_to_f64(v[b * vsb + (int64_t)j * vss + kvh * vsh + c]);
                        }
                    }
                }
            if (lse) lse[(int64_t)it * BLK + ii] = zmax + log(den);
        }
        free(blk);
        free(mt);
        free(use);
        free(row_max);
    }
}

/* --------------------------------------- o8 XAttention antidiagonal estimate */
/* XAttention blog, 2.1 "importance prediction" and 2.2 "threshold block
 * selection" (its block-selection algorithm).  For head h, query block qb
 * and stride S (S divides 128): every S x S sub-block of the token-level score
 * map is scored by the sum along its antidiagonal, i.e. strided row
 * R = qb*128/S + r (tokens R*S .. R*S+S-1) against strided column c (tokens
 * c*S .. c*S+S-1) scores
 *     z[R][c] = sum_{t<S} q[R*S + S-1-t] . k[c*S + t] / (sqrt(d) * S),
 * the reshaped product of that algorithm (query rows taken from S-1 down to
 * 0, key rows from 0 up).  Readings where the algorithm is silent: the causal
 * mask applies at the
 * strided level (c <= R: sub-blocks on or below the diagonal; non-causal: every
 * column, the pages' video-generation use); each strided row
 * is softmax-normalised over its valid columns; the estimate of block kb is the
 * mean over the query block's 128/S strided rows of the probability falling
 * in kb's columns, so the estimates of a row sum to one.
 * mass [B][H][T], entry row_at(qb)+kb. */
void pa_oracle_xattn_mass(int B, int N, int H, int Hkv, int d, int S,
                          const uint16_t *q, int64_t qsb, int64_t qss, int64_t qsh,
                          const uint16_t *k, int64_t ksb, int64_t kss, int64_t ksh,
                          int causal, double *mass)
{
    int nb = N / BLK, rpb = BLK / S;  /* strided rows (and columns) per block */
    int64_t T = rows_total(causal, nb);
    double scale = 1.0 / (sqrt((double)d) * S);
    #pragma omp parallel for collapse(3) schedule(dynamic, 1)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++)
            for (int qb = 0; qb < nb; qb++) {
                int kvh = kv_of(h, H, Hkv);
                double *m = mass + ((int64_t)b * H + h) * T + row_at(causal, nb, qb);
                int ncol = row_len(causal, nb, qb) * rpb;
                double *z = (double *)malloc(sizeof(double) * ncol);
                for (int kb = 0; kb < row_len(causal, nb, qb); kb++) m[kb] = 0.0;
                for (int r = 0; r < rpb; r++) {
                    int R = qb * rpb + r;
                    int cend = causal ? R + 1 : ncol;  /* strided columns c < cend */
                    double zmax = -INFINITY;
                    for (int c = 0; c < cend; c++) {
                        double s = 0.0;
                        for (int t = 0; t < S; t++)
                            for (int e = 0; e < d; e++)
                                s += bf16_to_f64(q[b * qsb + (int64_t)(R * S + S - 1 - t) * qss + h * qsh + e]) *
                                     bf16_to_f64(k[b * ksb + (int64_t)(c * S + t) * kss + kvh * ksh + e]);
                        z[c] = s * scale;
                        if (z[c] > zmax) zmax = z[c];
                    }
                    double den = 0.0;
                    for (int c = 0; c < cend; c++) den += exp(z[c] - zmax);
                    for (int c = 0; c < cend; c++) m[c / rpb] += exp(z[c] - zmax) / den / rpb;
                }
                free(z);
            }
}

/* find_blocks (XAttention blog, 2.2 equation): for every (b, h, qb) the
 * smallest set of blocks whose estimates add up to at least tau, i.e. the
 * shortest prefix of the blocks ordered by (estimate descending, lower index
 * first).  Sums run in 2^-40 fixed point as in o4; if no prefix reaches tau
 * (rounding), every block is kept.  rank [B][H][T] (the ordered blocks),
 * cnt [B][H][nb] (prefix length). */
void pa_oracle_find_blocks(int B, int H, int nb, const double *mass, double tau, int causal,
                           int32_t *rank, int32_t *cnt)
{
    int64_t T = rows_total(causal, nb);
    int64_t tfx = llrint(tau * 1099511627776.0);
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++)
            for (int qb = 0; qb < nb; qb++) {
                const double *m = mass + ((int64_t)b * H + h) * T + row_at(causal, nb, qb);
                int32_t *out = rank + ((int64_t)b * H + h) * T + row_at(causal, nb, qb);
                int len = row_len(causal, nb, qb);
                /* insertion sort by (estimate desc, index asc) */
                for (int t = 0; t < len; t++) {
                    int u = t;
                    while (u > 0 && (m[out[u - 1]] < m[t] || (m[out[u - 1]] == m[t] && out[u - 1] > t))) {
                        out[u] = out[u - 1];
                        u--;
                    }
                    out[u] = t;
                }
                int64_t cum = 0;
                int n = len;
                for (int t = 0; t < len; t++) {
                    cum += llrint(m[out[t]] * 1099511627776.0);
                    if (cum >= tfx) { n = t + 1; break; }
                }
                cnt[((int64_t)b * H + h) * nb + qb] = n;
            }
}

/* ------------------------------------------------------ o6 dense attention */
/* Causal softmax attention for requested rows (b, h, i): keys 0..i.
 * out [n_rows][d], lse [n_rows]. */
void pa_oracle_dense_attn(int N, int H, int Hkv, int d,
                          const uint16_t *q, int64_t qsb, int64_t qss, int64_t qsh,
                          const uint16_t *k, int64_t ksb, int64_t kss, int64_t ksh,
                          const uint16_t *v, int64_t vsb, int64_t vss, int64_t vsh,
                          double scale, int causal, int n_rows, const int32_t *rows /* [n][3] = b,h,i */,
                          double *out, double *lse)
{
    #pragma omp parallel for schedule(dynamic, 4)
    for (int r = 0; r < n_rows; r++) {
        int b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        int kvh = kv_of(h, H, Hkv);
        int nkeys = causal ? i + 1 : N;  /* keys 0 .. nkeys-1 */
        double *z = (double *)malloc(sizeof(double) * nkeys);
        double zmax = -INFINITY;
        for (int j = 0; j < nkeys; j++) {
            double s = 0.0;
            for (int c = 0; c < d; c++)
                s += bf16_to_f64(q[b * qsb + (int64_t)i * qss + h * qsh + c]) *
                     bf16_to_f64(k[b * ksb + (int64_t)j * kss + kvh * ksh + c]);
            z[j] = scale * s;
            if (z[j] > zmax) zmax = z[j];
        }
        double den = 0.0;
        for (int j = 0; j < nkeys; j++) den += exp(z[j] - zmax);
        double *o = out + (int64_t)r * d;
        for (int c = 0; c < d; c++) o[c] = 0.0;
        for (int j = 0; j < nkeys; j++) {
            double p = exp(z[j] - zmax) / den;
            for (int c = 0; c < d; c++)
                o[c] += p * bf16_to_f64(v[b * vsb + (int64_t)j * vss + kvh * vsh + c]);
        }
        if (lse) lse[r] = zmax + log(den);
        free(z);
    }
}

int pa_oracle_num_threads(void)
{
    int n = 1;
    #pragma omp parallel
    {
        #pragma omp single
        n = omp_get_num_threads();
    }
    return n;
}
