/*
 * oracle.c -- plain, slow, obviously-correct CPU reference for lossless
 * speculative-sampling verification of a batch of drafted tokens.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline / reference arm of bench.py load this library.  It shares no
 * code with the CUDA path and the CUDA path never calls it.
 *
 * Arithmetic: every input value is converted exactly to double (float and
 * bfloat16 both embed exactly), and every step below runs in double precision
 * with plain sequential loops in vocabulary-index order.  No blocking, no
 * reordering, no fusion.
 *
 * Sources (web pages; the rule is stated only in prose there):
 *  [NG-SD]   "AI 开始抄自己的作业——而且抄得理直气壮" (zhichai.net), section
 *            "⚡ 投机解码：让草稿先跑，考官殿后": a drafted token x is accepted with
 *            probability min(1, pi(x|c)/q(x|c)); on rejection the token is redrawn
 *            from the residual distribution, i.e. the target distribution with the
 *            part the draft already proposed taken out; worked example q=0.9,
 *            pi=0.95 -> accept surely, q=0.9, pi=0.1 -> about 0.11.
 *  [NG-EXAM] same page, section "👨🏫 考官坐镇：为什么抄作业不算作弊": the same rule
 *            restated, and the output distribution equals plain target sampling.
 *  [NG-PIPE] same page, section "🚰 真正的瓶颈不在算法，在流水线": a verification
 *            step ends in a pair (j, b): j drafts accepted, then token b; when all
 *            drafts are accepted, the next position's token is the continuation.
 *  [KC-GLOSS] "NgramRL：用Rollout历史加速RL后训练的推测解码新方案" (kongchang.com),
 *            section "一个被忽视的草稿源", glossary entry on speculative decoding:
 *            accept the prefix that matches, reject after the first mismatch
 *            (the greedy / prefix-match form).
 *  [VAT-SEQ] "今热点：让AI草稿模型学会"照镜子"：训练时就知道自己会不会被打回"
 *            (001ce.com), section "先搞懂投机解码在干什么": verification runs in
 *            order and every draft after the first rejection is discarded.
 *  [VAT-SIM] same page, section "VAT怎么把"验收规则"塞进训练里": training simulates
 *            the verification with the same probability-ratio rule, and every
 *            position from the first rejection on is labelled rejected.
 *  [VAT-W]   same page, section "第二件事，改权重分配的锚点": per-position loss
 *            weights keep full weight before the first rejection and start the
 *            fixed decay curve (EAGLE-3: 0.8^(k-1) over positions k = 1, 2, ...)
 *            at the first rejection instead of at the first position; the
 *            ablation's hard cut-off gives zero weight after it.
 *
 * Readings where the pages are silent:
 *  - residual = normalise(max(0, p - q)), the plain reading of a redraw from
 *    the target with the draft's share taken out;
 *  - all drafts accepted -> bonus token drawn from the target row L (row k+1);
 *  - target and draft logits are both divided by the same temperature T;
 *  - uniforms[b*(k_max+1) + i] is the acceptance draw for draft i; the separate
 *    slot uniforms[b*(k_max+1) + k_max] drives the final (residual / bonus) draw;
 *  - accept iff u < a (u in [0,1)), so a = 1 always accepts, a = 0 never does;
 *  - inverse CDF: the token is the smallest t with C_t > u*W (C_t = prefix sum
 *    of the weights in index order, W = total); if rounding leaves none, the
 *    largest t with w_t > 0;
 *  - W <= 0 (only possible when p == q numerically) -> draw from p_j instead;
 *  - no draft logits -> q is a point mass at the drafted id ("one-hot");
 *  - greedy: argmax with the lowest index on ties; accept x_i iff x_i equals the
 *    argmax of target row i; the emitted token is the argmax of row j;
 *  - draft_lens[b] outside [0, k_max] or a drafted id outside [0, V) for i < L
 *    -> the request is invalid: out_len = -1 and all its out_tokens = -1.
 *
 *  - acceptance simulation: E[j] = sum over m = 1..L of P(j >= m), with
 *    P(j >= m) = prod_{l<m} a_l (independent uniforms); loss weight 1 for
 *    i <= j and decay^(i - j) for i > j, 0 past the request's length.
 *
 * Near-tie flags (results are unique except inside these bands):
 *  ORACLE_FLAG_ACCEPT_TIE  |u_i - a_i| < 1e-5 at an examined position i <= j;
 *  ORACLE_FLAG_DRAW_TIE    |u*W - C_{b-1}| < 1e-5 W or |C_b - u*W| < 1e-5 W.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1

#define ORACLE_FLAG_ACCEPT_TIE 1
#define ORACLE_FLAG_DRAW_TIE 2
#define ORACLE_FLAG_INVALID 4
#define ORACLE_FLAG_ZERO_RESIDUAL 8
#define ORACLE_FLAG_DRAW_FALLBACK 16

#define ORACLE_TIE_BAND 1e-5

/* Exact conversion of one stored logit to double. */
static double load_logit(const void *row, int dtype, int64_t v)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)row)[v];
    uint32_t bits = (uint32_t)((const uint16_t *)row)[v] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Step 1 of the rule: temperature softmax of one row.
 * ell[v] = z[v] / T; M = max ell; S = sum exp(ell - M) in index order;
 * lse = M + log S.  Returns lse; ell is left filled for later use. */
static double row_log_sum_exp(const void *row, int dtype, int64_t V, double T,
                              double *ell)
{
    double M = -INFINITY;
    for (int64_t v = 0; v < V; ++v) {
        ell[v] = load_logit(row, dtype, v) / T;
        if (ell[v] > M)
            M = ell[v];
    }
    double S = 0.0;
    for (int64_t v = 0; v < V; ++v)
        S += exp(ell[v] - M);
    return M + log(S);
}

/* Greedy form: index of the largest logit, lowest index on ties. */
static int64_t row_argmax(const void *row, int dtype, int64_t V)
{
    int64_t best = 0;
    double best_val = load_logit(row, dtype, 0);
    for (int64_t v = 1; v < V; ++v) {
        double z = load_logit(row, dtype, v);
        if (z > best_val) {
            best_val = z;
            best = v;
        }
    }
    return best;
}

/* Step 4 of the rule: inverse-CDF draw over non-negative weights w[0..V).
 * Returns the smallest t with C_t > u*W; falls back to the largest t with
 * w_t > 0 when rounding leaves none.  Sets tie / fallback flags. */
static int64_t inverse_cdf_draw(const double *w, int64_t V, double u,
                                int32_t *flags)
{
    double W = 0.0;
    for (int64_t v = 0; v < V; ++v)
        W += w[v];
    double target = u * W;
    double C = 0.0;
    for (int64_t t = 0; t < V; ++t) {
        double C_prev = C;
        C += w[t];
        if (C > target) {
            if (fabs(target - C_prev) < ORACLE_TIE_BAND * W ||
                fabs(C - target) < ORACLE_TIE_BAND * W)
                *flags |= ORACLE_FLAG_DRAW_TIE;
            return t;
        }
    }
    *flags |= ORACLE_FLAG_DRAW_FALLBACK | ORACLE_FLAG_DRAW_TIE;
    for (int64_t t = V - 1; t >= 0; --t)
        if (w[t] > 0.0)
            return t;
    return 0;
}

/* Optional per-row diagnostics (natural-log lse and p, q at the drafted ids). */
typedef struct {
    double *lse_t; /* [B, k_max+1] or NULL */
    double *lse_d; /* [B, k_max]   or NULL */
    double *p;     /* [B, k_max]   or NULL */
    double *q;     /* [B, k_max]   or NULL */
} oracle_diag;

static void verify_one_request(
    int64_t b, int32_t k_max, int64_t V, int dtype, int64_t row_stride,
    int64_t req_stride_t, int64_t req_stride_d, const void *target,
    const void *draft, const int32_t *tokens, const int32_t *lens,
    const double *uniforms, double T, int greedy, int32_t *out_len,
    int32_t *out_tokens, int32_t *out_flags, const oracle_diag *diag,
    double *ell_t, double *ell_d, double *w)
{
    const int64_t esize = dtype == ORACLE_F32 ? 4 : 2;
    const char *tbase = (const char *)target + b * req_stride_t * esize;
    const char *dbase =
        draft ? (const char *)draft + b * req_stride_d * esize : NULL;
    const int32_t *x = tokens + b * (int64_t)k_max;
    const double *u = uniforms ? uniforms + b * (int64_t)(k_max + 1) : NULL;
    int32_t *tok_out = out_tokens + b * (int64_t)(k_max + 1);
    int32_t flags = 0;

    for (int32_t i = 0; i <= k_max; ++i)
        tok_out[i] = -1;
    if (diag) {
        for (int32_t i = 0; i <= k_max; ++i)
            if (diag->lse_t) diag->lse_t[b * (k_max + 1) + i] = NAN;
        for (int32_t i = 0; i < k_max; ++i) {
            if (diag->lse_d) diag->lse_d[b * k_max + i] = NAN;
            if (diag->p) diag->p[b * k_max + i] = NAN;
            if (diag->q) diag->q[b * k_max + i] = NAN;
        }
    }

    /* Input validation: the request is invalid when its length or one of its
     * first L drafted ids is out of range. */
    int32_t L = lens ? lens[b] : k_max;
    int valid = (L >= 0 && L <= k_max);
    for (int32_t i = 0; valid && i < L; ++i)
        if (x[i] < 0 || (int64_t)x[i] >= V)
            valid = 0;
    if (!valid) {
        out_len[b] = -1;
        out_flags[b] = ORACLE_FLAG_INVALID;
        return;
    }

#define TROW(i) ((const void *)(tbase + (int64_t)(i) * row_stride * esize))
#define DROW(i) ((const void *)(dbase + (int64_t)(i) * row_stride * esize))

    if (greedy) {
        /* Prefix-match verification [KC-GLOSS]: accept x_i while it equals the
         * target's argmax at row i; stop at the first mismatch [VAT-SEQ]. */
        int32_t j = L;
        for (int32_t i = 0; i < L; ++i) {
            if ((int64_t)x[i] != row_argmax(TROW(i), dtype, V)) {
                j = i;
                break;
            }
        }
        for (int32_t i = 0; i < j; ++i)
            tok_out[i] = x[i];
        tok_out[j] = (int32_t)row_argmax(TROW(j), dtype, V);
        out_len[b] = j;
        out_flags[b] = flags;
        return;
    }

    /* Steps 1-2: softmax statistics of the rows, p and q at the drafted ids. */
    double lse_t_row[L + 1];
    double lse_d_row[L > 0 ? L : 1];
    double p[L > 0 ? L : 1], q[L > 0 ? L : 1];
    for (int32_t i = 0; i <= L; ++i) {
        lse_t_row[i] = row_log_sum_exp(TROW(i), dtype, V, T, ell_t);
        if (i == L)
            break;
        p[i] = exp(ell_t[x[i]] - lse_t_row[i]);
        if (dbase) {
            lse_d_row[i] = row_log_sum_exp(DROW(i), dtype, V, T, ell_d);
            q[i] = exp(ell_d[x[i]] - lse_d_row[i]);
        } else {
            q[i] = 1.0; /* one-hot q at the drafted id */
        }
    }
    if (diag) {
        for (int32_t i = 0; i <= L; ++i)
            if (diag->lse_t) diag->lse_t[b * (k_max + 1) + i] = lse_t_row[i];
        for (int32_t i = 0; i < L; ++i) {
            if (diag->lse_d && dbase) diag->lse_d[b * k_max + i] = lse_d_row[i];
            if (diag->p) diag->p[b * k_max + i] = p[i];
            if (diag->q) diag->q[b * k_max + i] = q[i];
        }
    }

    /* Acceptance scan [NG-SD], [VAT-SEQ]: a_i = min(1, p_i / q_i); accept while
     * u_i < a_i, stop at the first rejection. */
    int32_t j = L;
    for (int32_t i = 0; i < L; ++i) {
        double a = p[i] / q[i];
        if (a > 1.0)
            a = 1.0;
        if (fabs(u[i] - a) < ORACLE_TIE_BAND)
            flags |= ORACLE_FLAG_ACCEPT_TIE;
        if (u[i] < a) {
            tok_out[i] = x[i];
        } else {
            j = i;
            break;
        }
    }

    /* Step 3: weights of the final draw on row j. */
    (void)row_log_sum_exp(TROW(j), dtype, V, T, ell_t);
    for (int64_t v = 0; v < V; ++v)
        w[v] = exp(ell_t[v] - lse_t_row[j]); /* p_j(v) */
    if (j < L) {
        /* Rejection: residual max(0, p_j - q_j) [NG-SD]. */
        if (dbase) {
            (void)row_log_sum_exp(DROW(j), dtype, V, T, ell_d);
            for (int64_t v = 0; v < V; ++v) {
                double r = w[v] - exp(ell_d[v] - lse_d_row[j]);
                w[v] = r > 0.0 ? r : 0.0;
            }
        } else {
            double r = w[x[j]] - 1.0; /* p - one-hot q at x_j */
            w[x[j]] = r > 0.0 ? r : 0.0;
        }
        double W = 0.0;
        for (int64_t v = 0; v < V; ++v)
            W += w[v];
        if (!(W > 0.0)) {
            /* Zero residual mass: draw from p_j. */
            flags |= ORACLE_FLAG_ZERO_RESIDUAL;
            for (int64_t v = 0; v < V; ++v)
                w[v] = exp(ell_t[v] - lse_t_row[j]);
        }
    }
    /* else j == L: bonus draw from p_L [NG-PIPE]; w already holds p_L. */

    /* Step 4: inverse-CDF draw with the final uniform slot. */
    tok_out[j] = (int32_t)inverse_cdf_draw(w, V, u[k_max], &flags);
    out_len[b] = j;
    out_flags[b] = flags;
#undef TROW
#undef DROW
}

/*
 * Verify B requests.  Layout (elements of dtype):
 *   target  request b, row i (0..k_max) at target + b*req_stride_t + i*row_stride
 *   draft   request b, row i (0..k_max-1) at draft + b*req_stride_d + i*row_stride,
 *           or draft == NULL for one-hot q
 *   tokens  [B, k_max] int32;  lens [B] int32 or NULL (all k_max)
 *   uniforms [B, k_max+1] double in [0,1) (may be NULL when greedy)
 * Outputs: out_len [B], out_tokens [B, k_max+1], out_flags [B]; the four
 * diagnostic arrays may each be NULL.  A request stride of 0 repeats the same
 * logits for every request.  Returns 0, or -1 on bad arguments / no memory.
 */
int oracle_spec_verify(int64_t B, int32_t k_max, int64_t V, int32_t dtype,
                       int64_t row_stride, int64_t req_stride_t,
                       int64_t req_stride_d, const void *target,
                       const void *draft, const int32_t *tokens,
                       const int32_t *lens, const double *uniforms,
                       double temperature, int32_t greedy, int32_t *out_len,
                       int32_t *out_tokens, int32_t *out_flags,
                       double *out_lse_t, double *out_lse_d, double *out_p,
                       double *out_q)
{
    if (B < 0 || k_max < 0 || V < 1 || row_stride < V || !target ||
        (k_max > 0 && !tokens) || !out_len || !out_tokens || !out_flags ||
        (dtype != ORACLE_F32 && dtype != ORACLE_BF16))
        return -1;
    if (!greedy && (!uniforms || !(temperature > 0.0)))
        return -1;
    double *scratch = (double *)malloc(sizeof(double) * (size_t)V * 3);
    if (!scratch)
        return -1;
    oracle_diag diag = {out_lse_t, out_lse_d, out_p, out_q};
    int any_diag = out_lse_t || out_lse_d || out_p || out_q;
    for (int64_t b = 0; b < B; ++b)
        verify_one_request(b, k_max, V, dtype, row_stride, req_stride_t,
                           req_stride_d, target, draft, tokens, lens, uniforms,
                           temperature, greedy, out_len, out_tokens, out_flags,
                           any_diag ? &diag : NULL, scratch, scratch + V,
                           scratch + 2 * V);
    free(scratch);
    return 0;
}

/*
 * Acceptance simulation over a batch [VAT-SIM], [VAT-W], from the per-position
 * probabilities p[b*k_max + i] = p_i(x_i) and q[b*k_max + i] = q_i(x_i) that
 * oracle_spec_verify returns (q = 1 for one-hot drafts):
 *   out_a[b*k_max + i]  a_i = min(1, p_i / q_i) for i < L_b, NaN after;
 *   out_e[b]            E[j] = sum_{m=1..L_b} prod_{l<m} a_l;
 *   out_j[b]            (uniforms != NULL) the first i < L_b with
 *                       u_i >= a_i (accept iff u < a), else L_b;
 *   out_w[b*k_max + i]  (uniforms != NULL) 1 for i <= j, decay^(i-j) for
 *                       j < i < L_b, 0 for i >= L_b.
 * A request with L_b outside [0, k_max] or a drafted id outside [0, V) is
 * invalid: out_j = -1, NaN elsewhere.  out_j / out_w may be NULL.
 */
int oracle_accept_sim(int64_t B, int32_t k_max, int64_t V, const int32_t *tokens,
                      const int32_t *lens, const double *p, const double *q,
                      const double *uniforms, double decay, double *out_a,
                      double *out_e, int32_t *out_j, double *out_w)
{
    for (int64_t b = 0; b < B; ++b) {
        const int32_t L = lens ? lens[b] : k_max;
        int valid = L >= 0 && L <= k_max;
        for (int32_t i = 0; valid && i < L; ++i)
            if (tokens[b * k_max + i] < 0 || tokens[b * k_max + i] >= V)
                valid = 0;
        double *a = out_a + b * k_max;
        if (!valid) {
            for (int32_t i = 0; i < k_max; ++i) {
                a[i] = NAN;
                if (out_w)
                    out_w[b * k_max + i] = NAN;
            }
            out_e[b] = NAN;
            if (out_j)
                out_j[b] = -1;
            continue;
        }
        for (int32_t i = 0; i < k_max; ++i) {
            if (i < L) {
                const double r = p[b * k_max + i] / q[b * k_max + i];
                a[i] = r > 1.0 ? 1.0 : r;
            } else {
                a[i] = NAN;
            }
        }
        /* expected number of accepted drafts */
        double e = 0.0, reach = 1.0; /* reach = P(j >= m) */
        for (int32_t m = 1; m <= L; ++m) {
            reach *= a[m - 1];
            e += reach;
        }
        out_e[b] = e;
        if (!uniforms)
            continue;
        int32_t j = L;
        for (int32_t i = 0; i < L; ++i) {
            if (!(uniforms[b * (k_max + 1) + i] < a[i])) {
                j = i;
                break;
            }
        }
        if (out_j)
            out_j[b] = j;
        if (out_w)
            for (int32_t i = 0; i < k_max; ++i)
                out_w[b * k_max + i] = i >= L ? 0.0 : (i <= j ? 1.0 : pow(decay, (double)(i - j)));
    }
    return 0;
}
