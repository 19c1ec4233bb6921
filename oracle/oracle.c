/*
 * oracle.c -- plain fp64 CPU reference of InfLLM-V2's dense-sparse switchable
 * attention for one causal GQA layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this code.  It shares no code with
 * the CUDA library: it is written directly from the method's definitions,
 * one query row at a time, in double precision, with no blocking or fusion.
 *
 * Sources (page titles and sections of the InfLLM-V2 material):
 *  - "InfLLM-V2 ... (ICLR 2026)" paper notes, key design 3: mean pooling of K
 *    over kernels of length l_C1 and stride s_C1; S^C1 = softmax(Q K^C1^T);
 *    S^shared = sum over the heads of a GQA group; max pooling with l, s.
 *  - same notes, key design 2: I(i) = I_init u I_local(i) u I_topk(i).
 *  - MiniCPM4 "InfLLM v2" blog, semantic kernels: a block's score is the max
 *    over the kernels that intersect the block; init and local blocks get an
 *    infinite score; sequences no longer than k blocks use dense attention.
 *  - arXiv 2509.24663 summary, Appendix A: attention of each query over the
 *    visible tokens of its selected blocks, returning O and the log-sum-exp.
 *  - same notes, key design 4, and the blog's efficient top-k: the optional
 *    LSE approximation estimates each head's log-sum-exp from coarser kernels
 *    K^C2 (l_C2 = 4 l_C1, s_C2 = 4 s_C1) instead of the K^C1 kernels.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - scale 1/sqrt(d) on the score logits and the attention logits (parameter);
 *  - a kernel is visible to query i only when its last token is <= i;
 *  - K^C1 is a bf16 tensor: the exact mean rounded once, nearest-even (the
 *    fp64 sum starts at +0, so a zero mean is +0);
 *  - the local set is {b_i - n_local + 1 .. b_i} (own block included);
 *  - k counts every selected block, init and local included;
 *  - equal block scores are ordered by lower block index;
 *  - backward (training; the arXiv summary's Appendix A returns the
 *    log-sum-exp for it): the FlashAttention-style gradients of the attention
 *    with the block lists fixed (selection is not differentiated); D = dO . O
 *    uses the forward output O that the caller holds;
 *  - LSE approximation (optional): K^C2 is rounded to bf16 like K^C1, a coarse
 *    kernel is visible under the same rule, the estimate is the log-sum-exp
 *    over the visible coarse kernels plus log(s_C2 / s_C1) (each coarse kernel
 *    stands for that many stage-1 kernels), and a row that sees no coarse
 *    kernel keeps the exact log-sum-exp.
 *
 * Parity unpinned: readings that no page fixes with a worked example, namely
 * the choice of the intersection rule over the literal max-pool window (both
 * are built; pool_rule selects), the 1/sqrt(d) logit scale, and in the
 * optional LSE approximation the bf16 rounding of K^C2 and the log(s_C2/s_C1)
 * constant.  Every function is pinned under those readings by the tests' pins.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B;        /* sparse block size (tokens) */
    int l_c1;     /* stage-1 kernel length */
    int s_c1;     /* stage-1 kernel stride */
    int pool_l;   /* max-pool length (kernels), used by the literal rule */
    int pool_s;   /* max-pool stride (kernels), used by the literal rule */
    int n_init;   /* initial blocks always selected */
    int n_local;  /* local blocks always selected (own block included) */
    int k;        /* total blocks selected per query */
    int h_q, h_kv, d;
    double scale; /* logit scale */
    int pool_rule;/* 0: kernels intersecting the block; 1: literal window */
    int lse_approx;/* 1: pass-1 log-sum-exp estimated from the coarse kernels K^C2 */
} orc_params;

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double bf16_value(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round x to the nearest bf16 value, ties to the even significand. */
uint16_t orc_bf16_round(double x) {
    uint64_t bits;
    memcpy(&bits, &x, sizeof bits);
    uint16_t sign = (uint16_t)((bits >> 48) & 0x8000u);
    if (isnan(x)) return 0x7FC0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    int e;
    (void)frexp(a, &e);          /* a = m * 2^e with 0.5 <= m < 1 */
    int q = e - 8;               /* spacing of bf16 values near a (8 significant bits) */
    if (q < -133) q = -133;      /* subnormal bf16 spacing */
    double scaled = ldexp(a, -q);        /* exact: power-of-two scaling */
    double lo = floor(scaled);
    double rem = scaled - lo;
    double r = lo;
    if (rem > 0.5) r = lo + 1.0;
    else if (rem == 0.5 && fmod(lo, 2.0) != 0.0) r = lo + 1.0;
    double y = ldexp(r, q);
    float f = (float)y;          /* exact unless it overflows to infinity */
    if (y > 3.3895313892515355e38) f = INFINITY; /* beyond the largest bf16 */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7FFFu));
}

/* Number of complete stage-1 kernels in a sequence of n tokens. */
int orc_num_kernels(const orc_params* p, int n) {
    if (n < p->l_c1) return 0;
    return (n - p->l_c1) / p->s_c1 + 1;
}

/* Kernels j whose whole window [j*s, j*s + l - 1] lies at or before query i. */
int orc_visible_kernels(const orc_params* p, int i) {
    int c = 0;
    for (int j = 0; j * p->s_c1 + p->l_c1 - 1 <= i; ++j) ++c;
    return c;
}

/* Stage 1: K^C1[j, g, :] = bf16(mean of K[t, g, :] over the kernel's tokens). */
void orc_compress_k(const orc_params* p, const uint16_t* k, int n, uint16_t* kc1) {
    int nc = orc_num_kernels(p, n);
    for (int j = 0; j < nc; ++j)
        for (int g = 0; g < p->h_kv; ++g)
            for (int c = 0; c < p->d; ++c) {
                double s = 0.0;
                for (int t = j * p->s_c1; t < j * p->s_c1 + p->l_c1; ++t)
                    s += bf16_value(k[((size_t)t * p->h_kv + g) * p->d + c]);
                kc1[((size_t)j * p->h_kv + g) * p->d + c] = orc_bf16_round(s / p->l_c1);
            }
}

/* The coarse kernels of the LSE approximation: the stage-1 definitions with
 * l_C2 = 4 l_C1 and s_C2 = 4 s_C1. */
static orc_params coarse_params(const orc_params* p) {
    orc_params c = *p;
    c.l_c1 = 4 * p->l_c1;
    c.s_c1 = 4 * p->s_c1;
    return c;
}

int orc_num_coarse_kernels(const orc_params* p, int n) {
    orc_params c = coarse_params(p);
    return orc_num_kernels(&c, n);
}

int orc_visible_coarse_kernels(const orc_params* p, int i) {
    orc_params c = coarse_params(p);
    return orc_visible_kernels(&c, i);
}

/* K^C2[c, g, :] = bf16(mean of K over the coarse kernel's l_C2 tokens). */
void orc_compress_k2(const orc_params* p, const uint16_t* k, int n, uint16_t* kc2) {
    orc_params c = coarse_params(p);
    orc_compress_k(&c, k, n, kc2);
}

/* Natural log-sum-exp over j < nv of scale * q_{i,h} . K_j (K = kc, [*, h_kv, d]). */
static double lse_over(const orc_params* p, const uint16_t* q, const uint16_t* kc, int nv,
                       int i, int h, int g, double* z) {
    const uint16_t* qr = q + ((size_t)i * p->h_q + h) * p->d;
    double m = -INFINITY;
    for (int j = 0; j < nv; ++j) {
        const uint16_t* kr = kc + ((size_t)j * p->h_kv + g) * p->d;
        double dot = 0.0;
        for (int c = 0; c < p->d; ++c) dot += bf16_value(qr[c]) * bf16_value(kr[c]);
        z[j] = p->scale * dot;
        if (z[j] > m) m = z[j];
    }
    if (nv == 0) return -INFINITY;
    double s = 0.0;
    for (int j = 0; j < nv; ++j) s += exp(z[j] - m);
    return m + log(s);
}

/* LSE approximation for row i, group g: lse_h ~= log sum over the visible
 * coarse kernels of exp(scale * q_{i,h} . K^C2_c) + log(s_C2 / s_C1).
 * Returns 0 (and writes nothing) when the row sees no coarse kernel. */
int orc_coarse_lse_row(const orc_params* p, const uint16_t* q, const uint16_t* kc2, int i, int g,
                       double* lse_out) {
    int nv2 = orc_visible_coarse_kernels(p, i);
    if (nv2 == 0) return 0;
    int G = p->h_q / p->h_kv;
    double* z = (double*)malloc(sizeof(double) * nv2);
    for (int hh = 0; hh < G; ++hh)
        lse_out[hh] = lse_over(p, q, kc2, nv2, i, g * G + hh, g, z) + log(4.0);
    free(z);
    return 1;
}

/* Stage 2 for one query row i and group g: S^shared[j] = sum over the group's
 * heads h of softmax_j(scale * q_{i,h} . K^C1_j), j over the visible kernels.
 * The softmax is normalised by lse_in[hh] when given (the LSE approximation),
 * else by the exact log-sum-exp over the visible kernels.  lse_out (nullable,
 * G entries) receives the log-sum-exp used. */
void orc_shared_scores_row_lse(const orc_params* p, const uint16_t* q, const uint16_t* kc1,
                               int i, int g, const double* lse_in, double* out, double* lse_out) {
    int nv = orc_visible_kernels(p, i);
    int G = p->h_q / p->h_kv;
    for (int j = 0; j < nv; ++j) out[j] = 0.0;
    if (nv == 0) {
        if (lse_out) for (int hh = 0; hh < G; ++hh) lse_out[hh] = -INFINITY;
        return;
    }
    double* z = (double*)malloc(sizeof(double) * nv);
    for (int hh = 0; hh < G; ++hh) {
        int h = g * G + hh;
        double lse = lse_over(p, q, kc1, nv, i, h, g, z);
        if (lse_in) lse = lse_in[hh];
        for (int j = 0; j < nv; ++j) out[j] += exp(z[j] - lse);
        if (lse_out) lse_out[hh] = lse;
    }
    free(z);
}

void orc_shared_scores_row(const orc_params* p, const uint16_t* q, const uint16_t* kc1,
                           int i, int g, double* out, double* lse_out) {
    orc_shared_scores_row_lse(p, q, kc1, i, g, NULL, out, lse_out);
}

/* Does stage-1 kernel j belong to block b's pooling window? */
static int in_pool_window(const orc_params* p, int j, int b) {
    if (p->pool_rule == 1) /* literal window: kernels b*s .. b*s + l - 1 */
        return j >= b * p->pool_s && j < b * p->pool_s + p->pool_l;
    /* kernels whose token span intersects the block's token span */
    int k_first = j * p->s_c1, k_last = j * p->s_c1 + p->l_c1 - 1;
    int b_first = b * p->B, b_last = b * p->B + p->B - 1;
    return k_first <= b_last && k_last >= b_first;
}

/* Stage 3: S^cmp[b] = max of S^shared over the visible kernels of block b's
 * window, for b = 0 .. i/B; -inf when the window has no visible kernel. */
void orc_block_scores_row(const orc_params* p, const double* shared, int nv, int i,
                          double* s_cmp) {
    int bi = i / p->B;
    for (int b = 0; b <= bi; ++b) {
        double best = -INFINITY;
        for (int j = 0; j < nv; ++j)
            if (in_pool_window(p, j, b) && shared[j] > best) best = shared[j];
        s_cmp[b] = best;
    }
}

typedef struct { double s; int b; } cand_t;

static int cand_order(const void* x, const void* y) {
    const cand_t* a = (const cand_t*)x;
    const cand_t* c = (const cand_t*)y;
    if (a->s > c->s) return -1;        /* higher score first */
    if (a->s < c->s) return 1;
    return (a->b > c->b) - (a->b < c->b); /* equal scores: lower block first */
}

/* Block selection for query i: the candidates are blocks 0..i/B.  When there
 * are at most k of them every one is kept (dense); otherwise the init and
 * local blocks are kept and the rest of the k slots go to the highest S^cmp.
 * Writes the chosen blocks ascending, padded with -1 to k; returns the count. */
int orc_select_row(const orc_params* p, const double* s_cmp, int i, int* idx) {
    int bi = i / p->B;
    int nc = bi + 1;
    char* chosen = (char*)calloc((size_t)nc, 1);
    int count = 0;
    if (nc <= p->k) {
        for (int b = 0; b < nc; ++b) chosen[b] = 1;
        count = nc;
    } else {
        for (int b = 0; b < nc; ++b)
            if (b < p->n_init || b > bi - p->n_local) { chosen[b] = 1; ++count; }
        cand_t* rest = (cand_t*)malloc(sizeof(cand_t) * nc);
        int nr = 0;
        for (int b = 0; b < nc; ++b)
            if (!chosen[b]) { rest[nr].s = s_cmp[b]; rest[nr].b = b; ++nr; }
        qsort(rest, (size_t)nr, sizeof(cand_t), cand_order);
        for (int r = 0; r < nr && count < p->k; ++r) { chosen[rest[r].b] = 1; ++count; }
        free(rest);
    }
    int w = 0; /* k >= n_init + n_local is required; never write past k */
    for (int b = 0; b < nc && w < p->k; ++b) if (chosen[b]) idx[w++] = b;
    for (; w < p->k; ++w) idx[w] = -1;
    free(chosen);
    return count;
}

/* Attention of query i, heads of group g, over the tokens t <= i of the
 * listed blocks (entries < 0 are ignored).  o: [G][d], lse: [G] (natural). */
void orc_attend_row(const orc_params* p, const uint16_t* q, const uint16_t* k,
                    const uint16_t* v, int i, int g, const int* idx, int cnt,
                    double* o, double* lse) {
    int G = p->h_q / p->h_kv;
    int ntok = 0;
    int* tok = (int*)malloc(sizeof(int) * ((size_t)cnt * p->B + 1));
    for (int r = 0; r < cnt; ++r) {
        if (idx[r] < 0) continue;
        for (int t = idx[r] * p->B; t < (idx[r] + 1) * p->B && t <= i; ++t) tok[ntok++] = t;
    }
    double* z = (double*)malloc(sizeof(double) * (ntok + 1));
    for (int hh = 0; hh < G; ++hh) {
        int h = g * G + hh;
        const uint16_t* qr = q + ((size_t)i * p->h_q + h) * p->d;
        double m = -INFINITY;
        for (int a = 0; a < ntok; ++a) {
            const uint16_t* kr = k + ((size_t)tok[a] * p->h_kv + g) * p->d;
            double dot = 0.0;
            for (int c = 0; c < p->d; ++c) dot += bf16_value(qr[c]) * bf16_value(kr[c]);
            z[a] = p->scale * dot;
            if (z[a] > m) m = z[a];
        }
        double L = 0.0;
        for (int a = 0; a < ntok; ++a) { z[a] = exp(z[a] - m); L += z[a]; }
        double* orow = o + (size_t)hh * p->d;
        for (int c = 0; c < p->d; ++c) orow[c] = 0.0;
        for (int a = 0; a < ntok; ++a) {
            const uint16_t* vr = v + ((size_t)tok[a] * p->h_kv + g) * p->d;
            for (int c = 0; c < p->d; ++c) orow[c] += z[a] * bf16_value(vr[c]);
        }
        for (int c = 0; c < p->d; ++c) orow[c] = ntok ? orow[c] / L : 0.0;
        lse[hh] = ntok ? m + log(L) : -INFINITY;
    }
    free(z);
    free(tok);
}

/*
 * The whole layer for selected query rows of one sequence of n tokens.
 *   rows[nrows]             query positions to evaluate
 *   idx_out  [nrows][h_kv][k]        selected blocks (ascending, -1 padded)
 *   o_out    [nrows][h_q][d]         attention output
 *   lse_out  [nrows][h_q]            attention log-sum-exp (natural log)
 *   cmp_out  [nrows][h_kv][n_blk]    nullable: S^cmp (-inf where undefined)
 *   shared_out [nrows][h_kv][n_c1]   nullable: S^shared (0 where not visible)
 *   score_lse_out [nrows][h_q]       nullable: log-sum-exp of the S^C1 softmax
 * Sequences with n <= k*B take dense attention: every visible block is used,
 * which is also what selection returns for them.
 */
void orc_prefill_rows(const orc_params* p, const uint16_t* q, const uint16_t* k,
                      const uint16_t* v, int n, const int* rows, int nrows,
                      int* idx_out, double* o_out, double* lse_out,
                      double* cmp_out, double* shared_out, double* score_lse_out) {
    int nc = orc_num_kernels(p, n);
    int n_blk = (n + p->B - 1) / p->B;
    int G = p->h_q / p->h_kv;
    int dense = n <= p->k * p->B;
    uint16_t* kc1 = (uint16_t*)malloc(sizeof(uint16_t) * ((size_t)nc * p->h_kv * p->d + 1));
    orc_compress_k(p, k, n, kc1);
    uint16_t* kc2 = NULL;
    if (p->lse_approx) {
        int nc2 = orc_num_coarse_kernels(p, n);
        kc2 = (uint16_t*)malloc(sizeof(uint16_t) * ((size_t)nc2 * p->h_kv * p->d + 1));
        orc_compress_k2(p, k, n, kc2);
    }
    int need_scores = !dense || cmp_out || shared_out || score_lse_out;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        int i = rows[r];
        int nv = orc_visible_kernels(p, i);
        int bi = i / p->B;
        double* shared = (double*)malloc(sizeof(double) * (nv + 1));
        double* cmp = (double*)malloc(sizeof(double) * (bi + 1));
        for (int g = 0; g < p->h_kv; ++g) {
            int* idx = idx_out + ((size_t)r * p->h_kv + g) * p->k;
            double* slse = score_lse_out ? score_lse_out + (size_t)r * p->h_q + g * G : NULL;
            if (need_scores) {
                double approx[64];  /* G <= 64 */
                int use = kc2 && orc_coarse_lse_row(p, q, kc2, i, g, approx);
                orc_shared_scores_row_lse(p, q, kc1, i, g, use ? approx : NULL, shared, slse);
                orc_block_scores_row(p, shared, nv, i, cmp);
            }
            if (shared_out) {
                double* so = shared_out + ((size_t)r * p->h_kv + g) * nc;
                for (int j = 0; j < nc; ++j) so[j] = j < nv ? shared[j] : 0.0;
            }
            if (cmp_out) {
                double* co = cmp_out + ((size_t)r * p->h_kv + g) * n_blk;
                for (int b = 0; b < n_blk; ++b) co[b] = b <= bi ? cmp[b] : -INFINITY;
            }
            int cnt;
            if (dense) {
                for (int b = 0; b <= bi; ++b) idx[b] = b;
                for (int b = bi + 1; b < p->k; ++b) idx[b] = -1;
                cnt = bi + 1;
            } else {
                cnt = orc_select_row(p, cmp, i, idx);
            }
            orc_attend_row(p, q, k, v, i, g, idx, cnt,
                           o_out + ((size_t)r * p->h_q + g * G) * p->d,
                           lse_out + (size_t)r * p->h_q + g * G);
        }
        free(cmp);
        free(shared);
    }
    free(kc1);
    free(kc2);
}

/* Selection alone, from given S^shared rows (values already in the precision
 * the caller wants the decision taken in).  shared: [nrows][h_kv][ld]. */
void orc_select_rows(const orc_params* p, const double* shared, int ld, const int* rows,
                     int nrows, int* idx_out, double* cmp_out, int n_blk) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int r = 0; r < nrows; ++r) {
        int i = rows[r];
        int nv = orc_visible_kernels(p, i);
        int bi = i / p->B;
        double* cmp = (double*)malloc(sizeof(double) * (bi + 1));
        for (int g = 0; g < p->h_kv; ++g) {
            orc_block_scores_row(p, shared + ((size_t)r * p->h_kv + g) * ld, nv, i, cmp);
            orc_select_row(p, cmp, i, idx_out + ((size_t)r * p->h_kv + g) * p->k);
            if (cmp_out) {
                double* co = cmp_out + ((size_t)r * p->h_kv + g) * n_blk;
                for (int b = 0; b < n_blk; ++b) co[b] = b <= bi ? cmp[b] : -INFINITY;
            }
        }
        free(cmp);
    }
}

/* Attention alone on given block lists idx [nrows][h_kv][k]. */
/* Backward of orc_attend_row for query i and the heads of group g:
 *   P_t  = softmax over the listed visible tokens t of scale * q_h . k_t
 *   D_h  = dO_h . O_h          (O_h = o_in, the forward output)
 *   dS_t = P_t * (dO_h . v_t - D_h)
 *   dq_h = scale * sum_t dS_t k_t;  dk_t += scale * dS_t q_h;  dv_t += P_t dO_h
 * o_in, dq_out: [G][d] fp64; d_o: bf16 [n, h_q, d]; dk_acc, dv_acc: fp64
 * [n, h_kv, d], added to. */
void orc_attend_bwd_row(const orc_params* p, const uint16_t* q, const uint16_t* k,
                        const uint16_t* v, const uint16_t* d_o, int i, int g, const int* idx,
                        int cnt, const double* o_in, double* dq_out, double* dk_acc,
                        double* dv_acc) {
    int G = p->h_q / p->h_kv;
    int ntok = 0;
    int* tok = (int*)malloc(sizeof(int) * ((size_t)cnt * p->B + 1));
    for (int r = 0; r < cnt; ++r) {
        if (idx[r] < 0) continue;
        for (int t = idx[r] * p->B; t < (idx[r] + 1) * p->B && t <= i; ++t) tok[ntok++] = t;
    }
    double* P = (double*)malloc(sizeof(double) * (ntok + 1));
    for (int hh = 0; hh < G; ++hh) {
        int h = g * G + hh;
        const uint16_t* qr = q + ((size_t)i * p->h_q + h) * p->d;
        const uint16_t* dor = d_o + ((size_t)i * p->h_q + h) * p->d;
        double* dq = dq_out + (size_t)hh * p->d;
        for (int c = 0; c < p->d; ++c) dq[c] = 0.0;
        if (ntok == 0) continue;
        double m = -INFINITY;
        for (int a = 0; a < ntok; ++a) {
            const uint16_t* kr = k + ((size_t)tok[a] * p->h_kv + g) * p->d;
            double dot = 0.0;
            for (int c = 0; c < p->d; ++c) dot += bf16_value(qr[c]) * bf16_value(kr[c]);
            P[a] = p->scale * dot;
            if (P[a] > m) m = P[a];
        }
        double L = 0.0;
        for (int a = 0; a < ntok; ++a) { P[a] = exp(P[a] - m); L += P[a]; }
        for (int a = 0; a < ntok; ++a) P[a] /= L;
        double D = 0.0;
        for (int c = 0; c < p->d; ++c) D += bf16_value(dor[c]) * o_in[(size_t)hh * p->d + c];
        for (int a = 0; a < ntok; ++a) {
            size_t kv = ((size_t)tok[a] * p->h_kv + g) * p->d;
            double dp = 0.0;
            for (int c = 0; c < p->d; ++c) dp += bf16_value(dor[c]) * bf16_value(v[kv + c]);
            double ds = P[a] * (dp - D);
            for (int c = 0; c < p->d; ++c) {
                dq[c] += p->scale * ds * bf16_value(k[kv + c]);
                dk_acc[kv + c] += p->scale * ds * bf16_value(qr[c]);
                dv_acc[kv + c] += P[a] * bf16_value(dor[c]);
            }
        }
    }
    free(P);
    free(tok);
}

/* Backward over the given query rows of one n-token sequence.
 *   o_in   [nrows][h_q][d] fp64: the forward output at those rows
 *   idx    [nrows][h_kv][k]
 *   dq_out [nrows][h_q][d]; dk_out, dv_out [n][h_kv][d] (overwritten: the
 *   sums over the given rows only) */
void orc_attend_bwd_rows(const orc_params* p, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, const uint16_t* d_o, int n, const int* rows,
                         int nrows, const int* idx, const double* o_in, double* dq_out,
                         double* dk_out, double* dv_out) {
    int G = p->h_q / p->h_kv;
    size_t sz = (size_t)n * p->h_kv * p->d;
    memset(dk_out, 0, sizeof(double) * sz);
    memset(dv_out, 0, sizeof(double) * sz);
#pragma omp parallel
    {
        double* dk = (double*)calloc(sz, sizeof(double));
        double* dv = (double*)calloc(sz, sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r)
            for (int g = 0; g < p->h_kv; ++g)
                orc_attend_bwd_row(p, q, k, v, d_o, rows[r], g,
                                   idx + ((size_t)r * p->h_kv + g) * p->k, p->k,
                                   o_in + ((size_t)r * p->h_q + g * G) * p->d,
                                   dq_out + ((size_t)r * p->h_q + g * G) * p->d, dk, dv);
#pragma omp critical
        for (size_t x = 0; x < sz; ++x) {
            dk_out[x] += dk[x];
            dv_out[x] += dv[x];
        }
        free(dk);
        free(dv);
    }
}

void orc_attend_rows(const orc_params* p, const uint16_t* q, const uint16_t* k,
                     const uint16_t* v, const int* rows, int nrows, const int* idx,
                     double* o_out, double* lse_out) {
    int G = p->h_q / p->h_kv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r)
        for (int g = 0; g < p->h_kv; ++g)
            orc_attend_row(p, q, k, v, rows[r], g, idx + ((size_t)r * p->h_kv + g) * p->k, p->k,
                           o_out + ((size_t)r * p->h_q + g * G) * p->d,
                           lse_out + (size_t)r * p->h_q + g * G);
}
