/*
 * hs_oracle.c -- plain fp64 CPU oracle for the HySparse / HySparse2 hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * path.  It is deliberately slow and literal: every query row is computed on
 * its own, with explicit loops, in double precision, from inputs that the
 * caller has already rounded to the precision under test and upcast to double.
 *
 * Sources (titles of the pages the method is described on):
 *  [HS-1]  "HySparse 混合稀疏注意力（一）：用全注意力当 Oracle，打通 Token 选择与 KV 复用"
 *          sections "从精确注意力里提取块级分数", "为什么不需要重新物化注意力矩阵",
 *          "GQA 下为什么要组内共享索引", "跨层 KV Cache 复用怎样成立",
 *          "同一个 Query，查询两种记忆", "工程实现中的关键约束" (item 4).
 *  [HS-P]  "HySparse: A Hybrid Sparse Attention Architecture with Oracle Token
 *          Selection and KV Cache Sharing", sections 3.2 (Algorithm 1) and 3.3.
 *  [HS2-N] "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
 *          (reading notes), section 4.2, "改造一" and "改造二".
 *  [HS2-S] "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
 *          (summary), "KV Reuse (Inner Level)".
 *
 * Readings taken where the pages are silent (all stated in the design notes):
 *  - positions are 0-based; query t sees keys 0..t (causal);
 *  - block r covers keys rB .. min((r+1)B-1, t)                    [HS-1 eq. B_r]
 *  - the token-level score of key i is the max over the group's heads of the
 *    attention probability p_{h,t,i} (the block rule with B = 1);
 *  - ties in the group score are broken towards the lower index;
 *  - token mode: the window is {max(0,t-w+1) .. t}; the remaining k-w slots go
 *    to the best keys in {0 .. t-w};  k is the TOTAL budget (window included);
 *  - when every candidate fits in the budget, everything is selected.
 *
 * Layouts (row-major, contiguous):
 *   q, o     [batch][hq ][t_q ][d]
 *   k, v     [batch][hkv][t_kv][d]
 * Query head h belongs to group u = h / (hq/hkv).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int batch, hq, hkv, head_dim;
    int t_q;        /* query rows per (batch, head) stored in q            */
    int t_kv;       /* key rows per (batch, kv head) stored in k, v       */
    int q_offset;   /* absolute position of query row 0 (prefill)        */
    int mode;       /* 0: block selection (HySparse), 1: token (HySparse2) */
    int block_size; /* B                                                  */
    int k;          /* token budget (token mode: window included)        */
    int window;     /* w                                                  */
    double scale;   /* softmax scale tau (1/sqrt(d) on the pages)         */
} orc_params;

/* A row to evaluate: batch b, kv group u, query row j (0 .. t_q-1). */
typedef struct { int b, u, j; } orc_row;

enum { ORC_OK = 0, ORC_BAD_ARG = 1 };

static int orc_group(const orc_params* p) { return p->hq / p->hkv; }

/* Number of selected entries stored per row: k/B blocks or k tokens. */
int orc_ksel(const orc_params* p) {
    return p->mode == 0 ? p->k / p->block_size : p->k;
}

/* Query position of listed row number n; the row sees keys 0..t.
 * Prefill: t = q_offset + j.  Decode (kv_len given): the single query is the
 * newest token, t = kv_len[b]-1.  q_pos (nullable) gives each listed row its
 * position explicitly, so a caller can pass just the query vectors it wants
 * evaluated (row j of q is then only storage, not a position).            */
static int orc_position(const orc_params* p, const int* kv_len, const int* q_pos, int n,
                        const orc_row* r) {
    if (q_pos) return q_pos[n];
    if (kv_len) return kv_len[r->b] - 1;
    return p->q_offset + r->j;
}

static const double* q_row(const orc_params* p, const double* q, int b, int h, int j) {
    return q + (((size_t)b * p->hq + h) * p->t_q + j) * p->head_dim;
}
static const double* kv_row(const orc_params* p, const double* kv, int b, int u, int i) {
    return kv + (((size_t)b * p->hkv + u) * p->t_kv + i) * p->head_dim;
}

static double dot(const double* a, const double* b, int d) {
    double s = 0.0;
    for (int x = 0; x < d; ++x) s += a[x] * b[x];
    return s;
}

/*
 * Exact softmax attention of one query vector over an explicit key list.
 * [HS-1] "从精确注意力里提取块级分数": a_i = q.k_i / sqrt(d),
 * p_i = exp(a_i) / sum_j exp(a_j), o = sum_i p_i v_i.  The max shift only
 * keeps exp() in range; lse = log sum_i exp(a_i).
 * logit_out (n entries) receives a_i; prob_out (nullable) receives p_i.
 */
static void attend_list(const orc_params* p, const double* qv, const double* kbase,
                        const double* vbase, int b, int u, const int* keys, int n,
                        double* o, double* lse, double* logit_out, double* prob_out) {
    const int d = p->head_dim;
    double m = -INFINITY;
    for (int x = 0; x < n; ++x) {
        logit_out[x] = p->scale * dot(qv, kv_row(p, kbase, b, u, keys[x]), d);
        if (logit_out[x] > m) m = logit_out[x];
    }
    double l = 0.0;
    for (int x = 0; x < n; ++x) l += exp(logit_out[x] - m);
    *lse = m + log(l);
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int x = 0; x < n; ++x) {
        double pr = exp(logit_out[x] - *lse);
        if (prob_out) prob_out[x] = pr;
        const double* vr = kv_row(p, vbase, b, u, keys[x]);
        for (int c = 0; c < d; ++c) o[c] += pr * vr[c];
    }
}

typedef struct { double s; int id; } orc_cand;

/* Order used by every top-k on the pages: higher score first; equal scores go
 * to the lower index (the deterministic tie-break this build adopts).        */
static int cand_cmp(const void* a, const void* b) {
    const orc_cand* x = (const orc_cand*)a;
    const orc_cand* y = (const orc_cand*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->id > y->id) - (x->id < y->id);
}
static int int_cmp(const void* a, const void* b) {
    int x = *(const int*)a, y = *(const int*)b;
    return (x > y) - (x < y);
}

/*
 * Full-attention layer acting as the oracle indexer, for a list of rows.
 *
 * For every listed row (b, u, j) and every head h of group u:
 *   o_h, lse_h            exact causal softmax attention           [HS-1]
 * then the group's selection:
 *   block mode:  S^(h)_{t,r} = max_{i in B_r} p_{h,t,i}              [HS-1], [HS-P 3.2]
 *                S_bar_{t,r} = max_{h in G_u} S^(h)_{t,r}            [HS-1 GQA], [HS-P 3.2]
 *                I_t = top (k/B) blocks by S_bar                      [HS-1 TopKBlocks]
 *   token mode:  S_bar_{t,i} = max_{h in G_u} p_{h,t,i}
 *                I_t = {max(0,t-w+1)..t}  U  top (k-w) of {0..t-w}    [HS2-N 改造二], [HS2-S]
 * The selection is written in ascending id order, padded with -1.
 *
 * Outputs (per listed row r):
 *   o         [n_rows][g][d]         lse [n_rows][g]
 *   idx       [n_rows][ksel]         cnt [n_rows]
 *   sel_score [n_rows][ksel] (nullable)  S_bar of each selected id, 0 padded
 *   scores    [n_rows][scores_stride] (nullable)  S_bar of every candidate
 *             (blocks 0..nb-1 or tokens 0..t), -1 beyond
 */
int orc_full_attn_index(const orc_params* p, const double* q, const double* k,
                        const double* v, const int* kv_len, const int* q_pos, int n_rows,
                        const orc_row* rows, double* o, double* lse, int* idx,
                        int* cnt, double* sel_score, double* scores,
                        int scores_stride) {
    if (!p || p->hkv <= 0 || p->hq % p->hkv != 0 || p->head_dim <= 0) return ORC_BAD_ARG;
    if (p->mode == 0 && (p->block_size <= 0 || p->k % p->block_size != 0)) return ORC_BAD_ARG;
    if (p->mode == 1 && (p->window < 0 || p->window > p->k)) return ORC_BAD_ARG;
    const int g = orc_group(p), d = p->head_dim, ksel = orc_ksel(p);
    int bad = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int r = 0; r < n_rows; ++r) {
        const orc_row* row = &rows[r];
        const int t = orc_position(p, kv_len, q_pos, r, row);
        const int n = t + 1; /* visible keys 0..t */
        if (t < 0 || t >= p->t_kv) { bad = 1; continue; }
        int* keys = (int*)malloc(sizeof(int) * n);
        double* logit = (double*)malloc(sizeof(double) * n);
        double* prob = (double*)malloc(sizeof(double) * (size_t)g * n);
        for (int i = 0; i < n; ++i) keys[i] = i;

        /* 1. exact attention per head; keep the probabilities of this row. */
        for (int hh = 0; hh < g; ++hh) {
            const int h = row->u * g + hh;
            attend_list(p, q_row(p, q, row->b, h, row->j), k, v, row->b, row->u, keys, n,
                        o + ((size_t)r * g + hh) * d, lse + (size_t)r * g + hh, logit,
                        prob + (size_t)hh * n);
        }

        /* 2. group scores of every candidate. */
        const int B = p->mode == 0 ? p->block_size : 1;
        const int nb = (n + B - 1) / B; /* candidates: blocks, or tokens when B = 1 */
        orc_cand* cand = (orc_cand*)malloc(sizeof(orc_cand) * nb);
        for (int c = 0; c < nb; ++c) {
            double sbar = -INFINITY;
            for (int hh = 0; hh < g; ++hh) {
                double sh = -INFINITY; /* S^(h) = max over the block's visible keys */
                for (int i = c * B; i <= t && i < (c + 1) * B; ++i)
                    if (prob[(size_t)hh * n + i] > sh) sh = prob[(size_t)hh * n + i];
                if (sh > sbar) sbar = sh;
            }
            cand[c].s = sbar;
            cand[c].id = c;
        }
        if (scores) {
            double* srow = scores + (size_t)r * scores_stride;
            for (int c = 0; c < scores_stride; ++c) srow[c] = c < nb ? cand[c].s : -1.0;
        }

        /* 3. selection. */
        int* out = idx + (size_t)r * ksel;
        int m = 0;
        if (p->mode == 0) {
            qsort(cand, nb, sizeof(orc_cand), cand_cmp);
            m = nb < ksel ? nb : ksel;
            for (int x = 0; x < m; ++x) out[x] = cand[x].id;
        } else if (n <= p->k) {
            m = n; /* budget covers every visible token */
            for (int x = 0; x < m; ++x) out[x] = x;
        } else {
            const int w = p->window;
            const int lo = t - w + 1; /* first window position (>= 1 here since n > k >= w) */
            /* top (k-w) of the tokens outside the window, 0 .. t-w */
            qsort(cand, lo, sizeof(orc_cand), cand_cmp);
            for (int x = 0; x < p->k - w; ++x) out[m++] = cand[x].id;
            for (int i = lo; i <= t; ++i) out[m++] = i; /* forced window */
        }
        qsort(out, m, sizeof(int), int_cmp);
        for (int x = m; x < ksel; ++x) out[x] = -1;
        cnt[r] = m;

        if (sel_score) {
            /* scores are re-derived from the per-head probabilities so that the
             * window members (never ranked) also get their S_bar.            */
            double* ss = sel_score + (size_t)r * ksel;
            for (int x = 0; x < ksel; ++x) {
                if (x >= m) { ss[x] = 0.0; continue; }
                const int c = out[x];
                double sbar = -INFINITY;
                for (int hh = 0; hh < g; ++hh)
                    for (int i = c * B; i <= t && i < (c + 1) * B; ++i)
                        if (prob[(size_t)hh * n + i] > sbar) sbar = prob[(size_t)hh * n + i];
                ss[x] = sbar;
            }
        }
        free(cand);
        free(prob);
        free(logit);
        free(keys);
    }
    return bad ? ORC_BAD_ARG : ORC_OK;
}

/*
 * Sparse layer reusing the full layer's K^F / V^F and index set, for a list
 * of rows, with the row's own query q' (one per head of the group).
 *
 *   global branch  R_t = the selected tokens (token mode), or the union of the
 *                  selected blocks' keys clipped to 0..t (block mode; the
 *                  in-block causal mask of [HS-1] "工程实现中的关键约束" item 4);
 *                  o' = sum_{i in R_t} softmax_{R_t}(tau q'.k^F_i) v^F_i
 *                  [HS-1] "跨层 KV Cache 复用怎样成立" and "同一个 Query，查询两种记忆",
 *                  [HS-P 3.3]
 *   local branch   (block mode only, when k_loc != NULL): banded softmax over
 *                  the layer's own K', V' for keys max(0,t-w+1)..t   [HS-1], [HS-P 3.3]
 *
 * idx_rows [n_rows][ksel] and cnt_rows [n_rows] give each row's index set
 * (the caller chooses whose: the oracle's own, or the one under test).
 * Outputs: o_g [n_rows][g][d], lse_g [n_rows][g]; o_l, lse_l likewise
 * (only written when k_loc != NULL).
 */
int orc_sparse_attn(const orc_params* p, const double* q, const double* kf,
                    const double* vf, const int* kv_len, const int* q_pos, int n_rows,
                    const orc_row* rows,
                    const int* idx_rows, const int* cnt_rows, const double* k_loc,
                    const double* v_loc, double* o_g, double* lse_g, double* o_l,
                    double* lse_l) {
    if (!p || p->hkv <= 0 || p->hq % p->hkv != 0) return ORC_BAD_ARG;
    const int g = orc_group(p), d = p->head_dim, ksel = orc_ksel(p);
    int bad = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int r = 0; r < n_rows; ++r) {
        const orc_row* row = &rows[r];
        const int t = orc_position(p, kv_len, q_pos, r, row);
        const int c = cnt_rows[r];
        const int B = p->mode == 0 ? p->block_size : 1;
        if (t < 0 || t >= p->t_kv || c < 0 || c > ksel) { bad = 1; continue; }
        int* keys = (int*)malloc(sizeof(int) * ((size_t)c * B + p->window + 1));
        double* logit = (double*)malloc(sizeof(double) * ((size_t)c * B + p->window + 1));
        int n = 0;
        for (int x = 0; x < c; ++x) {
            const int id = idx_rows[(size_t)r * ksel + x];
            for (int i = id * B; i < (id + 1) * B; ++i)
                if (i >= 0 && i <= t) keys[n++] = i;
        }
        for (int hh = 0; hh < g; ++hh) {
            const int h = row->u * g + hh;
            const double* qv = q_row(p, q, row->b, h, row->j);
            double* og = o_g + ((size_t)r * g + hh) * d;
            if (n == 0) { /* empty set: defined as a zero output, lse = -inf */
                for (int x = 0; x < d; ++x) og[x] = 0.0;
                lse_g[(size_t)r * g + hh] = -INFINITY;
            } else {
                attend_list(p, qv, kf, vf, row->b, row->u, keys, n, og,
                            lse_g + (size_t)r * g + hh, logit, NULL);
            }
        }
        if (k_loc) {
            const int lo = t - p->window + 1 > 0 ? t - p->window + 1 : 0;
            int nl = 0;
            for (int i = lo; i <= t; ++i) keys[nl++] = i;
            for (int hh = 0; hh < g; ++hh) {
                const int h = row->u * g + hh;
                attend_list(p, q_row(p, q, row->b, h, row->j), k_loc, v_loc, row->b, row->u,
                            keys, nl, o_l + ((size_t)r * g + hh) * d,
                            lse_l + (size_t)r * g + hh, logit, NULL);
            }
        }
        free(logit);
        free(keys);
    }
    return bad ? ORC_BAD_ARG : ORC_OK;
}

/*
 * Output of a sparse layer: a sink per branch, then the sigmoid-gate fusion of
 * the two branches.
 *   [HS-1] "两个 sigmoid gate，而不是二选一": o_t = g^G (.) o^global + g^L (.) o^local,
 *          g^G, g^L = sigma(W_g x_t), two independent sigmoids (no softmax
 *          between the branches);
 *   [HS-P] 3.3, branch fusion (sigmoid gates on both outputs, then the sum), and
 *          the configuration note: sparse and SWA branches carry a learnable
 *          per-head sink bias (the gpt-oss construction).
 * Readings: a gate acts per head (one value per row and head); the caller
 * supplies its pre-activation z (the projection W_g x_t belongs to the model).
 * A sink is one more logit s_h in the branch's softmax whose value vector is
 * zero, so the branch output and log-sum-exp become
 *     o' = o e^lse / (e^lse + e^s),     lse' = log(e^lse + e^s).
 * n entries (row, head) of d channels each; o_l, lse_l, s_l, z_l may be NULL
 * (one branch); s_* NULL: no sink; z_* NULL: gate 1.  Writes o [n][d] and the
 * branches' lse' (lse_g_out always, lse_l_out when o_l is given).
 */
static double log_add_exp(double a, double b) {
    const double m = a > b ? a : b;
    if (m == -INFINITY) return -INFINITY;
    return m + log(exp(a - m) + exp(b - m));
}

int orc_gate_sink(int n, int d, const double* o_g, const double* lse_g, const double* s_g,
                  const double* z_g, const double* o_l, const double* lse_l, const double* s_l,
                  const double* z_l, double* o, double* lse_g_out, double* lse_l_out) {
    if (n < 0 || d <= 0 || !o_g || !lse_g || !o || !lse_g_out) return ORC_BAD_ARG;
    if (o_l && (!lse_l || !lse_l_out)) return ORC_BAD_ARG;
    for (int e = 0; e < n; ++e) {
        /* global branch: share of its softmax mass on real keys, and its gate */
        const double lg = s_g ? log_add_exp(lse_g[e], s_g[e]) : lse_g[e];
        const double fg = s_g ? exp(lse_g[e] - lg) : 1.0;
        const double gg = z_g ? 1.0 / (1.0 + exp(-z_g[e])) : 1.0;
        lse_g_out[e] = lg;
        double fl = 0.0, gl = 0.0;
        if (o_l) {
            const double ll = s_l ? log_add_exp(lse_l[e], s_l[e]) : lse_l[e];
            fl = s_l ? exp(lse_l[e] - ll) : 1.0;
            gl = z_l ? 1.0 / (1.0 + exp(-z_l[e])) : 1.0;
            lse_l_out[e] = ll;
        }
        for (int x = 0; x < d; ++x) {
            double v = gg * fg * o_g[(size_t)e * d + x];
            if (o_l) v += gl * fl * o_l[(size_t)e * d + x];
            o[(size_t)e * d + x] = v;
        }
    }
    return ORC_OK;
}

int orc_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
