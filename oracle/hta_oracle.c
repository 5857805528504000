/*
 * hta_oracle.c -- plain, slow, fp64 CPU oracle for Hybrid Tree Attention,
 * the verification attention of LongSpec.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library; both sides only see the same seeded input bytes.
 *
 * What it computes is the plain definition, not the method's fast route:
 *
 *   For batch b, query head h and tree node t, let G = Hq / Hkv and
 *   kvh = h / G (query heads are grouped contiguously onto KV heads).  The
 *   query q[b][h][t] attends over the concatenated key list
 *       [ k_prefix[b][kvh][0 .. L_b-1] ; k_tree[b][kvh][0 .. T-1] ]
 *   under a visibility mask that is spelled out key by key:
 *       prefix key j          : visible (the prefix is unmasked)
 *       tree key  i           : visible iff i == t or i is an ancestor of t,
 *                               following parent[] up to -1.
 *   scores x_j = scale * sum_d q[d] * k_j[d]   (fp64, bf16 inputs upcast
 *   exactly), m = max over visible x_j, l = sum_visible exp(x_j - m),
 *   out = sum_visible exp(x_j - m) v_j / l,  lse = m + ln(l).
 *
 * Sources (the pages give the decomposition, not formulas):
 *   - LongSpec README (sail-sg/LongSpec), "Introduction", third contribution
 *     "Hybrid Attention Aggregation": fast prefix computation combined with
 *     standard attention for the tree mask.
 *   - LongSpec paper summary (Elamur Research), "Summary", the Hybrid Tree
 *     Attention bullet: a Flash Attention pass over the prefix plus a kernel
 *     for the speculated tree; and the title / first sentence: lossless,
 *     outputs unchanged.  Lossless aggregation of two softmax partials has
 *     one exact form, log-sum-exp rescaling, written out in
 *     hta_oracle_lse_merge below.
 *   - LongSpec arXiv abstract (jarxiv.com, original abstract): attention
 *     aggregation combining fast prefix implementations with standard
 *     attention for tree mask handling.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   a node sees itself (ancestor-or-self); parent -1 means "child of the
 *   prefix end"; parent[i] must lie in [-1, i) (topological order), anything
 *   else is rejected; scale 0 means 1/sqrt(D); lse is the natural log.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Problem description shared by every entry point (mirrored by ctypes). */
typedef struct {
    int B, Hq, Hkv, D, T, L_cap;
    double scale;                 /* 0 => 1/sqrt(D) */
    const uint16_t *q;            /* bf16 bits [B][Hq][T][D] */
    const uint16_t *k_prefix;     /* bf16 bits [B][Hkv][L_cap][D] */
    const uint16_t *v_prefix;     /* bf16 bits [B][Hkv][L_cap][D] */
    const int32_t *prefix_len;    /* [B], 0 <= L_b <= L_cap */
    const uint16_t *k_tree;       /* bf16 bits [B][Hkv][T][D] */
    const uint16_t *v_tree;       /* bf16 bits [B][Hkv][T][D] */
    const int32_t *parent;        /* [B][T], parent[i] in [-1, i) */
} hta_oracle_problem;

enum {
    HTA_ORACLE_OK = 0,
    HTA_ORACLE_BAD_DIMS = -1,
    HTA_ORACLE_BAD_PARENT = -2,
    HTA_ORACLE_BAD_PREFIX_LEN = -3,
    HTA_ORACLE_BAD_ROW = -4,
    HTA_ORACLE_NO_MEMORY = -5,
    HTA_ORACLE_NO_VISIBLE_KEY = -6
};

/*
 * Planted mistakes, for the tests that show each pin can fail.  0 = the
 * oracle as specified.  Any other value breaks one step on purpose:
 *   1 drop the self bit from the tree mask
 *   2 ignore the tree keys altogether
 *   3 map query head h to KV head h % Hkv instead of h / G
 *   4 leave out the softmax scale
 *   5 merge partials with weights exp(lse_c) not renormalised (wrong merge)
 *   6 read the prefix one key short (drop the last prefix key)
 */
static int g_mutation = 0;
void hta_oracle_set_mutation(int code) { g_mutation = code; }
int hta_oracle_get_mutation(void) { return g_mutation; }

/* bf16 -> fp64, exact: the 16 bits are the top half of an IEEE float. */
static double bf16_to_f64(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double hta_oracle_bf16_value(uint16_t bits) { return bf16_to_f64(bits); }

static double effective_scale(const hta_oracle_problem *p)
{
    if (g_mutation == 4) return 1.0;
    return p->scale != 0.0 ? p->scale : 1.0 / sqrt((double)p->D);
}

static int kv_head_of(const hta_oracle_problem *p, int h)
{
    int G = p->Hq / p->Hkv;
    if (g_mutation == 3) return h % p->Hkv;
    return h / G;
}

/* ------------------------------------------------------------------------ */
/* Tree mask                                                                 */
/* ------------------------------------------------------------------------ */

/*
 * Ancestor-or-self bitmask of one tree: anc[i*words + w] bit k set iff node
 * 32*w + k is node i or one of its ancestors, found by following parent[]
 * from i up to -1.  The tree mask of the pages ("standard attention for tree
 * mask handling", LongSpec README, Introduction; arXiv abstract) restricted
 * to tree keys: a speculated token sees the path that led to it.
 * Returns HTA_ORACLE_BAD_PARENT if some parent[i] is outside [-1, i).
 */
int hta_oracle_tree_mask(int T, const int32_t *parent, uint32_t *anc, int words)
{
    if (T < 0 || words < (T + 31) / 32) return HTA_ORACLE_BAD_DIMS;
    for (int i = 0; i < T; ++i)
        if (parent[i] < -1 || parent[i] >= i) return HTA_ORACLE_BAD_PARENT;
    memset(anc, 0, sizeof(uint32_t) * (size_t)T * (size_t)words);
    for (int i = 0; i < T; ++i) {
        uint32_t *row = anc + (size_t)i * words;
        if (g_mutation != 1) row[i / 32] |= 1u << (i % 32);
        for (int j = parent[i]; j != -1; j = parent[j])
            row[j / 32] |= 1u << (j % 32);
    }
    return HTA_ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Masked softmax attention of one query over an explicit key list           */
/* ------------------------------------------------------------------------ */

/*
 * keys/values: n row pointers of D bf16 values each; vis[j] != 0 marks the
 * visible keys.  Writes out[D] and *lse.  With no visible key, out = 0 and
 * lse = -inf (an empty partial).
 */
static void attend(int D, double scale, const uint16_t *q, int n,
                   const uint16_t *const *keys, const uint16_t *const *vals,
                   const unsigned char *vis, double *x, double *out,
                   double *lse)
{
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        if (!vis[j]) continue;
        double s = 0.0;
        for (int d = 0; d < D; ++d)
            s += bf16_to_f64(q[d]) * bf16_to_f64(keys[j][d]);
        x[j] = scale * s;
        if (x[j] > m) m = x[j];
    }
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (m == -INFINITY) { *lse = -INFINITY; return; }
    double l = 0.0;
    for (int j = 0; j < n; ++j) {
        if (!vis[j]) continue;
        double w = exp(x[j] - m);
        l += w;
        for (int d = 0; d < D; ++d) out[d] += w * bf16_to_f64(vals[j][d]);
    }
    for (int d = 0; d < D; ++d) out[d] /= l;
    *lse = m + log(l);
}

static int check_problem(const hta_oracle_problem *p)
{
    if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->D < 1 || p->T < 0 ||
        p->L_cap < 0 || p->Hq % p->Hkv != 0)
        return HTA_ORACLE_BAD_DIMS;
    for (int b = 0; b < p->B; ++b) {
        if (p->prefix_len[b] < 0 || p->prefix_len[b] > p->L_cap)
            return HTA_ORACLE_BAD_PREFIX_LEN;
        for (int i = 0; i < p->T; ++i) {
            int32_t par = p->parent[(size_t)b * p->T + i];
            if (par < -1 || par >= i) return HTA_ORACLE_BAD_PARENT;
        }
    }
    return HTA_ORACLE_OK;
}

/* Row selection: rows == NULL means all B*Hq*T rows in (b, h, t) order;
 * otherwise rows holds n_rows triples (b, h, t). */
static int row_bht(const hta_oracle_problem *p, const int32_t *rows, int r,
                   int *b, int *h, int *t)
{
    if (rows) {
        *b = rows[3 * r]; *h = rows[3 * r + 1]; *t = rows[3 * r + 2];
    } else {
        *t = r % p->T; *h = (r / p->T) % p->Hq; *b = r / (p->T * p->Hq);
    }
    if (*b < 0 || *b >= p->B || *h < 0 || *h >= p->Hq || *t < 0 || *t >= p->T)
        return HTA_ORACLE_BAD_ROW;
    return HTA_ORACLE_OK;
}

/* Which part of the concatenated key list a pass looks at. */
enum { PASS_ONE = 0, PASS_PREFIX = 1, PASS_TREE = 2 };

/*
 * Core of every entry point: for each selected row, spell out the key list
 * [prefix(L_b); tree(T)] and its visibility mask, then attend.
 *   PASS_ONE    : prefix keys visible, tree keys visible by ancestry.
 *   PASS_PREFIX : only prefix keys j with key_begin <= j < key_end visible.
 *   PASS_TREE   : only tree keys visible by ancestry.
 */
static int run_pass(const hta_oracle_problem *p, int pass, int key_begin,
                    int key_end, int n_rows, const int32_t *rows, double *out,
                    double *lse)
{
    int rc = check_problem(p);
    if (rc) return rc;
    int words = (p->T + 31) / 32;
    if (words == 0) words = 1;
    int n_max = p->L_cap + p->T;
    const uint16_t **keys = malloc(sizeof(*keys) * (size_t)(n_max + 1));
    const uint16_t **vals = malloc(sizeof(*vals) * (size_t)(n_max + 1));
    unsigned char *vis = malloc((size_t)n_max + 1);
    double *x = malloc(sizeof(double) * (size_t)(n_max + 1));
    uint32_t *anc = malloc(sizeof(uint32_t) * (size_t)(p->T + 1) * words);
    if (!keys || !vals || !vis || !x || !anc) { rc = HTA_ORACLE_NO_MEMORY; goto done; }
    double scale = effective_scale(p);
    int D = p->D;
    for (int r = 0; r < n_rows; ++r) {
        int b, h, t;
        rc = row_bht(p, rows, r, &b, &h, &t);
        if (rc) goto done;
        int kvh = kv_head_of(p, h);
        int L = p->prefix_len[b];
        if (g_mutation == 6 && L > 0) L -= 1;
        rc = hta_oracle_tree_mask(p->T, p->parent + (size_t)b * p->T, anc, words);
        if (rc) goto done;
        size_t kv_base = ((size_t)b * p->Hkv + kvh);
        for (int j = 0; j < L; ++j) {
            keys[j] = p->k_prefix + (kv_base * p->L_cap + j) * D;
            vals[j] = p->v_prefix + (kv_base * p->L_cap + j) * D;
            vis[j] = (pass == PASS_ONE) ||
                     (pass == PASS_PREFIX && j >= key_begin && j < key_end);
        }
        const uint32_t *anc_t = anc + (size_t)t * words;
        for (int i = 0; i < p->T; ++i) {
            keys[L + i] = p->k_tree + (kv_base * p->T + i) * D;
            vals[L + i] = p->v_tree + (kv_base * p->T + i) * D;
            int ancestor = (anc_t[i / 32] >> (i % 32)) & 1u;
            vis[L + i] = (pass != PASS_PREFIX) && ancestor && g_mutation != 2;
        }
        const uint16_t *qr = p->q + (((size_t)b * p->Hq + h) * p->T + t) * D;
        attend(D, scale, qr, L + p->T, keys, vals, vis, x,
               out + (size_t)r * D, lse + r);
        if (pass == PASS_ONE && lse[r] == -INFINITY) { rc = HTA_ORACLE_NO_VISIBLE_KEY; goto done; }
    }
    rc = HTA_ORACLE_OK;
done:
    free(keys); free(vals); free(vis); free(x); free(anc);
    return rc;
}

/* One-pass masked attention over [prefix; tree]: the definition itself. */
int hta_oracle_attention(const hta_oracle_problem *p, int n_rows,
                         const int32_t *rows, double *out, double *lse)
{
    return run_pass(p, PASS_ONE, 0, 0, n_rows, rows, out, lse);
}

/* Prefix-only partial over prefix keys [key_begin, key_end) (clipped to
 * L_b): the unmasked prefix pass of the method, one split-KV chunk of it.
 * An empty chunk gives out = 0, lse = -inf. */
int hta_oracle_prefix_partial(const hta_oracle_problem *p, int key_begin,
                              int key_end, int n_rows, const int32_t *rows,
                              double *out, double *lse)
{
    return run_pass(p, PASS_PREFIX, key_begin, key_end, n_rows, rows, out, lse);
}

/* Tree-only partial: tree keys under the ancestor-or-self mask. */
int hta_oracle_tree_partial(const hta_oracle_problem *p, int n_rows,
                            const int32_t *rows, double *out, double *lse)
{
    return run_pass(p, PASS_TREE, 0, 0, n_rows, rows, out, lse);
}

/*
 * Exact aggregation of softmax partials by log-sum-exp rescaling (the
 * "attention aggregation" of the pages, in its only lossless form):
 *   m = max_c lse_c over parts with lse_c > -inf,
 *   w_c = exp(lse_c - m),
 *   out = sum_c w_c O_c / sum_c w_c,   lse = m + ln(sum_c w_c).
 * Parts with lse_c = -inf carry no mass and are skipped.  If every part is
 * empty, out = 0 and lse = -inf.
 * o_parts: [n_parts][n_rows][D], lse_parts: [n_parts][n_rows].
 */
int hta_oracle_lse_merge(int n_rows, int n_parts, int D, const double *o_parts,
                         const double *lse_parts, double *out, double *lse)
{
    if (n_rows < 0 || n_parts < 0 || D < 1) return HTA_ORACLE_BAD_DIMS;
    for (int r = 0; r < n_rows; ++r) {
        double m = -INFINITY;
        for (int c = 0; c < n_parts; ++c) {
            double v = lse_parts[(size_t)c * n_rows + r];
            if (v > m) m = v;
        }
        double *o = out + (size_t)r * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (m == -INFINITY) { lse[r] = -INFINITY; continue; }
        double wsum = 0.0;
        for (int c = 0; c < n_parts; ++c) {
            double v = lse_parts[(size_t)c * n_rows + r];
            if (v == -INFINITY) continue;
            double w = (g_mutation == 5) ? exp(v) : exp(v - m);
            wsum += w;
            const double *oc = o_parts + ((size_t)c * n_rows + r) * D;
            for (int d = 0; d < D; ++d) o[d] += w * oc[d];
        }
        if (g_mutation != 5)
            for (int d = 0; d < D; ++d) o[d] /= wsum;
        lse[r] = m + log(wsum);
    }
    return HTA_ORACLE_OK;
}
