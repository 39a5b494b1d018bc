/*
 * Float64 reference ("the oracle") for exact scaled-dot-product attention with
 * grouped-query heads.
 *
 * TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the benchmark's
 * CPU-baseline leg call this code; the CUDA library never does, and the two share
 * no source, header, table or helper.
 *
 * What it computes (plain definition, no blocking or fusion):
 *   FlashAttention-2 summary page (azimuth.plus), paragraph on standard attention:
 *     S = Q K^T, P = row-wise softmax(S), O = P V, with S and P materialised.
 *   The scale multiplies the logits inside the softmax (S = scale * Q K^T).
 *   Same page, deferred-normalisation paragraph: the per-row log-sum-exp
 *     L = m + log(l) is the statistic written out next to O.
 *   Same page, causal-masking paragraph: every entry above the diagonal is -inf,
 *     the diagonal itself is kept.
 *   Ultralytics glossary "Grouped Query Attention (GQA)", section "How GQA works":
 *     Hq query heads share Hkv key/value heads in contiguous groups of G = Hq/Hkv
 *     (the printed repeat_interleave(G, dim=1) equivalence gives query head h the
 *     key/value head h / G).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - causal alignment for Sq != Sk is bottom-right: key j is visible to query i
 *     iff j <= i + (Sk - Sq); a decode row (Sq = 1) therefore sees every key;
 *   - a row with no visible key has O = 0 and L = -inf;
 *   - L uses the natural logarithm of the scaled logits;
 *   - split-KV partials cut the keys into contiguous ranges; a partial is the
 *     attention restricted to its range (normalised), with its own L; the combine
 *     is L = M + ln sum_s exp(L_s - M), O = sum_s exp(L_s - L) O_s.
 *
 * Layouts (all contiguous, row-major):
 *   dense:  q [B, Sq, Hq, D], k and v [B, Sk, Hkv, D]; o like q; lse [B, Hq, Sq]
 *   varlen: cu_seqlens int32[B+1]; q [total, Hq, D], k and v [total, Hkv, D];
 *           sequence b owns rows cu[b]..cu[b+1]-1 of all three (self-attention,
 *           Sq = Sk = its length); o like q; lse [Hq, total]
 * Inputs are float32 (bf16 and fp32 values widen to float64 exactly); every
 * arithmetic step is float64.
 *
 * KV-cache decode (oracle_decode_kvcache): Ultralytics glossary "Grouped Query
 * Attention (GQA)" -- the KV cache holds the keys and values of every earlier
 * token and each new token reads all of it ("How GQA shrinks the KV cache");
 * PagedAttention stores that cache in fixed-size blocks and sliding-window
 * attention caps the tokens attended to ("GQA and related techniques").  Readings:
 * key j of sequence b lives in row j % page_size of page block_table[b][j /
 * page_size]; with a window W > 0 the query (the newest position) attends to the
 * last W of the L cached keys, j >= L - W.
 * FP8 cache: the GQA batch-size guide names FP8 (hardware adaptation section) without
 * a format; reading: e4m3 codes (sign, 4-bit exponent with bias 7, 3-bit mantissa,
 * subnormals 2^-6 * m/8, codes 0x7f / 0xff NaN, no infinities), one scale per tensor,
 * stored value = code value * scale.
 *
 * Block-sparse attention (oracle_attention_blocksparse): Raptor-T abstract, research
 * background -- BigBird cuts the input into blocks of a block size and computes
 * attention between blocks; several attention patterns combine into the final one.
 * Reading: a pattern of (query block, key block) pairs given as rows of key blocks
 * (CSR: row_ptr[n_qblk + 1], col[nnz]); key j is visible to query i iff block
 * j / blk is in row i / blk; otherwise exactly the definition above (non-causal).
 *
 * Backward (oracle_attention_backward): FA-2 summary page, parallelism paragraph of the
 * backward pass -- dK and dV accumulate per key/value column block, dQ is shared; GQA
 * paragraph -- dK and dV are summed over the query heads that share a K/V head.  The
 * page gives no formulas; these are the derivatives of the definition above (L's
 * derivative is not needed: only dO is given):
 *   dV = P^T dO;  dP = dO V^T;  D_i = sum_j P_ij dP_ij;  dS = P * (dP - D);
 *   dQ = scale * dS K;  dK = scale * dS^T Q.
 *
 * Return value of every entry point: 0 on success, -1 on bad arguments.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* Deliberate-mistake switch.  Only the pin-strength tests set it: each value
 * plants one plausible bug so that a test can show the pins catch it.        */
enum {
    FLAW_NONE = 0,
    FLAW_STRIDED_HEADS = 1,   /* kv head = h % Hkv instead of h / G            */
    FLAW_DROP_DIAGONAL = 2,   /* causal mask also hides the diagonal           */
    FLAW_TOP_LEFT_CAUSAL = 3, /* causal alignment j <= i instead of bottom-right */
    FLAW_NO_SCALE = 4,        /* scale left out of the logits                 */
    FLAW_LSE_NO_MAX = 5,      /* L = log(l) without adding the max back        */
    FLAW_FA1_NO_RESCALE = 6,  /* tiled FA-1 form drops exp(m_old - m_new)      */
    FLAW_SWAP_KV = 7,         /* uses K where V belongs in O = P V             */
    FLAW_PAGES_CONTIGUOUS = 8,/* paged cache read as if pages were in order     */
    FLAW_WINDOW_SHORT = 9,    /* sliding window keeps one key too few           */
    FLAW_E4M3_BIAS = 10,      /* e4m3 exponent bias 8 instead of 7              */
    FLAW_SPARSE_ROW = 11,     /* block pattern row of the next query block       */
    FLAW_BWD_NO_D = 12,       /* backward: dS = P * dP, without subtracting D    */
    FLAW_E4M3_NO_VSCALE = 13, /* e4m3 prefill: O left without the V scale        */
    FLAW_SPARSE_MAXPAD = 14,  /* varlen pattern rows numbered as if every sequence
                                 were padded to the longest one                 */
};
static int g_flaw = FLAW_NONE;
void oracle_set_flaw(int flaw) { g_flaw = flaw; }
int oracle_get_flaw(void) { return g_flaw; }

/* ------------------------------------------------------------------------- */
/* Shape of one attention problem as seen by a single (sequence, query head). */
typedef struct {
    const float* q;   /* first element of query row 0 of this head            */
    const float* k;   /* first element of key row 0 of this head's kv head     */
    const float* v;
    size_t q_stride;  /* elements between consecutive query rows               */
    size_t kv_stride; /* elements between consecutive key / value rows         */
    int Sq, Sk, D;
    double scale;
    int causal;
    int window; /* > 0 (causal only): key j visible to query i only if j > i + Sk - Sq - window */
} head_view;

/* Grouped-query mapping: query head h reads key/value head h / G. */
static int kv_head_of(int h, int Hq, int Hkv)
{
    if (g_flaw == FLAW_STRIDED_HEADS) return h % Hkv;
    return h / (Hq / Hkv);
}

/*
 * Causal visibility of key j to query i (bottom-right aligned), optionally within a
 * sliding window: query i, at key position i + Sk - Sq, sees its `window` most recent
 * keys, (i + Sk - Sq - window, i + Sk - Sq] (Ultralytics GQA glossary, "GQA and
 * related techniques": sliding-window attention caps the tokens attended to; the same
 * reading as the decode window below).
 */
static int key_visible_w(int i, int j, int Sq, int Sk, int causal, int window)
{
    if (!causal) return 1;
    int vis;
    if (g_flaw == FLAW_TOP_LEFT_CAUSAL)
        vis = j <= i;
    else if (g_flaw == FLAW_DROP_DIAGONAL)
        vis = j < i + (Sk - Sq);
    else
        vis = j <= i + (Sk - Sq);
    if (window > 0) {
        const int w = (g_flaw == FLAW_WINDOW_SHORT) ? window - 1 : window;
        vis = vis && j > i + (Sk - Sq) - w;
    }
    return vis;
}
static int key_visible(int i, int j, int Sq, int Sk, int causal)
{
    return key_visible_w(i, j, Sq, Sk, causal, 0);
}

static double dot(const float* a, const float* b, int D)
{
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += (double)a[d] * (double)b[d];
    return acc;
}

/*
 * One query row i, restricted to keys [j0, j1): materialises the score row
 * S[i, j0:j1] and the probability row P[i, j0:j1] in `row` (length >= Sk),
 * then O[i, :] = P[i, :] V and L_i = m_i + ln(l_i).
 */
static void attend_row(const head_view* hv, int i, int j0, int j1, double* row,
                       double* o_out, double* lse_out)
{
    const float* qi = hv->q + (size_t)i * hv->q_stride;
    const double scale = (g_flaw == FLAW_NO_SCALE) ? 1.0 : hv->scale;
    double m = -INFINITY;
    for (int j = j0; j < j1; ++j) {
        if (key_visible_w(i, j, hv->Sq, hv->Sk, hv->causal, hv->window)) {
            row[j] = scale * dot(qi, hv->k + (size_t)j * hv->kv_stride, hv->D);
            if (row[j] > m) m = row[j];
        } else {
            row[j] = -INFINITY;
        }
    }
    if (m == -INFINITY) { /* no visible key */
        for (int d = 0; d < hv->D; ++d) o_out[d] = 0.0;
        *lse_out = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int j = j0; j < j1; ++j) {
        row[j] = (row[j] == -INFINITY) ? 0.0 : exp(row[j] - m);
        l += row[j];
    }
    for (int j = j0; j < j1; ++j) row[j] /= l; /* row now holds P[i, j] */
    const float* vsrc = (g_flaw == FLAW_SWAP_KV) ? hv->k : hv->v;
    for (int d = 0; d < hv->D; ++d) {
        double acc = 0.0;
        for (int j = j0; j < j1; ++j)
            if (row[j] != 0.0) acc += row[j] * (double)vsrc[(size_t)j * hv->kv_stride + d];
        o_out[d] = acc;
    }
    *lse_out = (g_flaw == FLAW_LSE_NO_MAX) ? log(l) : m + log(l);
}

/* Build the view of (sequence b, query head h). */
static head_view make_view(const float* q, const float* k, const float* v, int B, int Hq,
                           int Hkv, int Sq, int Sk, int D, double scale, int causal,
                           const int32_t* cu, int b, int h, size_t* q_row0, size_t* lse_off,
                           size_t* lse_step)
{
    head_view hv;
    const int kvh = kv_head_of(h, Hq, Hkv);
    size_t qrow0, krow0;
    int sq, sk;
    if (cu) {
        qrow0 = (size_t)cu[b];
        krow0 = (size_t)cu[b];
        sq = sk = cu[b + 1] - cu[b];
        *lse_off = (size_t)h * (size_t)cu[B] + (size_t)cu[b];
    } else {
        qrow0 = (size_t)b * Sq;
        krow0 = (size_t)b * Sk;
        sq = Sq;
        sk = Sk;
        *lse_off = ((size_t)b * Hq + h) * (size_t)Sq;
    }
    *lse_step = 1;
    *q_row0 = qrow0;
    hv.q = q + (qrow0 * Hq + h) * (size_t)D;
    hv.k = k + (krow0 * Hkv + kvh) * (size_t)D;
    hv.v = v + (krow0 * Hkv + kvh) * (size_t)D;
    hv.q_stride = (size_t)Hq * D;
    hv.kv_stride = (size_t)Hkv * D;
    hv.Sq = sq;
    hv.Sk = sk;
    hv.D = D;
    hv.scale = scale;
    hv.causal = causal;
    hv.window = 0;
    return hv;
}

static int check_args(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                      int Sq, int Sk, int D, const int32_t* cu)
{
    if (!q || !k || !v) return -1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (!cu && (Sq < 0 || Sk < 0)) return -1;
    if (cu) {
        if (cu[0] != 0) return -1;
        for (int b = 0; b < B; ++b)
            if (cu[b + 1] < cu[b]) return -1;
    }
    return 0;
}

static int max_keys(int B, int Sk, const int32_t* cu)
{
    if (!cu) return Sk;
    int mx = 0;
    for (int b = 0; b < B; ++b)
        if (cu[b + 1] - cu[b] > mx) mx = cu[b + 1] - cu[b];
    return mx;
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Full attention forward: every (sequence, head, query row).
 * o has the layout of q; lse is [B, Hq, Sq] (dense) or [Hq, total] (varlen).
 */
static int attention_impl(const float* q, const float* k, const float* v, double* o,
                          double* lse, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                          double scale, int causal, int window, const int32_t* cu_seqlens,
                          int nthreads)
{
    if (check_args(q, k, v, B, Hq, Hkv, Sq, Sk, D, cu_seqlens) || !o || !lse) return -1;
    if (window < 0 || (window > 0 && !causal)) return -1;
    set_threads(nthreads);
    const int kmax = max_keys(B, Sk, cu_seqlens);
    const int nbh = B * Hq;
    int err = 0;
#pragma omp parallel
    {
        double* row = (double*)malloc(sizeof(double) * (size_t)(kmax > 0 ? kmax : 1));
        if (!row) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int bh = 0; bh < nbh; ++bh) {
            if (!row) continue;
            const int b = bh / Hq, h = bh % Hq;
            size_t qrow0, lse_off, lse_step;
            head_view hv = make_view(q, k, v, B, Hq, Hkv, Sq, Sk, D, scale, causal, cu_seqlens,
                                     b, h, &qrow0, &lse_off, &lse_step);
            hv.window = window;
            for (int i = 0; i < hv.Sq; ++i) {
                double* orow = o + ((qrow0 + (size_t)i) * Hq + h) * (size_t)D;
                attend_row(&hv, i, 0, hv.Sk, row, orow, lse + lse_off + (size_t)i * lse_step);
            }
        }
        free(row);
    }
    return err;
}

int oracle_attention(const float* q, const float* k, const float* v, double* o, double* lse,
                     int B, int Hq, int Hkv, int Sq, int Sk, int D, double scale, int causal,
                     const int32_t* cu_seqlens, int nthreads)
{
    return attention_impl(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, 0,
                          cu_seqlens, nthreads);
}

/* Causal attention within a sliding window of `window` >= 1 keys (key_visible_w). */
int oracle_attention_window(const float* q, const float* k, const float* v, double* o,
                            double* lse, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                            double scale, int window, const int32_t* cu_seqlens, int nthreads)
{
    if (window < 1) return -1;
    return attention_impl(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, D, scale, 1, window,
                          cu_seqlens, nthreads);
}

/*
 * Selected rows only: rows holds n_rows triples (b, h, i).  For each, O[i, :] of
 * query head h of sequence b goes to o_rows[r*D .. r*D+D) and L_i to lse_rows[r].
 * Used to check outputs of problems too large to evaluate in full.
 */
int oracle_attention_rows_window(const float* q, const float* k, const float* v, int B,
                                 int Hq, int Hkv, int Sq, int Sk, int D, double scale,
                                 int causal, int window, const int32_t* cu_seqlens, int n_rows,
                                 const int32_t* rows, double* o_rows, double* lse_rows,
                                 int nthreads)
{
    if (check_args(q, k, v, B, Hq, Hkv, Sq, Sk, D, cu_seqlens) || n_rows < 0) return -1;
    if (window < 0 || (window > 0 && !causal)) return -1;
    if (n_rows > 0 && (!rows || !o_rows || !lse_rows)) return -1;
    for (int r = 0; r < n_rows; ++r) {
        const int b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0) return -1;
        const int len = cu_seqlens ? cu_seqlens[b + 1] - cu_seqlens[b] : Sq;
        if (i >= len) return -1;
    }
    set_threads(nthreads);
    const int kmax = max_keys(B, Sk, cu_seqlens);
    int err = 0;
#pragma omp parallel
    {
        double* row = (double*)malloc(sizeof(double) * (size_t)(kmax > 0 ? kmax : 1));
        if (!row) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < n_rows; ++r) {
            if (!row) continue;
            size_t qrow0, lse_off, lse_step;
            head_view hv = make_view(q, k, v, B, Hq, Hkv, Sq, Sk, D, scale, causal, cu_seqlens,
                                     rows[3 * r], rows[3 * r + 1], &qrow0, &lse_off, &lse_step);
            hv.window = window;
            attend_row(&hv, rows[3 * r + 2], 0, hv.Sk, row, o_rows + (size_t)r * D,
                       lse_rows + r);
        }
        free(row);
    }
    return err;
}

int oracle_attention_rows(const float* q, const float* k, const float* v, int B, int Hq,
                          int Hkv, int Sq, int Sk, int D, double scale, int causal,
                          const int32_t* cu_seqlens, int n_rows, const int32_t* rows,
                          double* o_rows, double* lse_rows, int nthreads)
{
    return oracle_attention_rows_window(q, k, v, B, Hq, Hkv, Sq, Sk, D, scale, causal, 0,
                                        cu_seqlens, n_rows, rows, o_rows, lse_rows, nthreads);
}

/*
 * Attention restricted to keys [j0, j1) of a dense problem: the split-KV partial
 * (O_s normalised over its own keys, L_s its log-sum-exp; O_s = 0 and L_s = -inf
 * when the range holds no visible key).  Layout of o and lse as in
 * oracle_attention.
 */
int oracle_attention_keyrange(const float* q, const float* k, const float* v, double* o,
                              double* lse, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                              double scale, int causal, int j0, int j1, int nthreads)
{
    if (check_args(q, k, v, B, Hq, Hkv, Sq, Sk, D, NULL) || !o || !lse) return -1;
    if (j0 < 0 || j1 > Sk || j0 > j1) return -1;
    set_threads(nthreads);
    const int nbh = B * Hq;
    int err = 0;
#pragma omp parallel
    {
        double* row = (double*)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
        if (!row) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int bh = 0; bh < nbh; ++bh) {
            if (!row) continue;
            const int b = bh / Hq, h = bh % Hq;
            size_t qrow0, lse_off, lse_step;
            head_view hv = make_view(q, k, v, B, Hq, Hkv, Sq, Sk, D, scale, causal, NULL, b, h,
                                     &qrow0, &lse_off, &lse_step);
            for (int i = 0; i < Sq; ++i)
                attend_row(&hv, i, j0, j1, row, o + ((qrow0 + (size_t)i) * Hq + h) * (size_t)D,
                           lse + lse_off + (size_t)i);
        }
        free(row);
    }
    return err;
}

/*
 * Log-sum-exp weighted combine of n partial results of one row:
 *   M = max_s L_s,  L = M + ln sum_s exp(L_s - M),  O = sum_s exp(L_s - L) O_s.
 * Partials with L_s = -inf carry weight 0; if every L_s is -inf then O = 0 and
 * L = -inf.  Os is [n, D].
 */
void oracle_combine(int n, int D, const double* Os, const double* Ls, double* O, double* L)
{
    double M = -INFINITY;
    for (int s = 0; s < n; ++s)
        if (Ls[s] > M) M = Ls[s];
    for (int d = 0; d < D; ++d) O[d] = 0.0;
    if (M == -INFINITY) {
        *L = -INFINITY;
        return;
    }
    double sum = 0.0;
    for (int s = 0; s < n; ++s)
        if (Ls[s] != -INFINITY) sum += exp(Ls[s] - M);
    const double Lall = M + log(sum);
    for (int s = 0; s < n; ++s) {
        if (Ls[s] == -INFINITY) continue;
        const double w = exp(Ls[s] - Lall);
        for (int d = 0; d < D; ++d) O[d] += w * Os[(size_t)s * D + d];
    }
    *L = Lall;
}

/*
 * Gradients of O = attention(Q, K, V) for a given dO (dense layout, optional causal
 * mask with the forward's bottom-right alignment).  dq like q; dk, dv like k (summed
 * over the G query heads of each K/V head).  Rows without a visible key contribute
 * nothing.  P is recomputed in float64 from the definition.  Needs B*Hq*Sk*D*16 bytes
 * of host memory for the per-head partial dk, dv.
 */
int oracle_attention_backward(const float* q, const float* k, const float* v, const float* dout,
                              double* dq, double* dk, double* dv, int B, int Hq, int Hkv,
                              int Sq, int Sk, int D, double scale, int causal, int nthreads)
{
    if (check_args(q, k, v, B, Hq, Hkv, Sq, Sk, D, NULL) || !dout || !dq || !dk || !dv)
        return -1;
    const int G = Hq / Hkv;
    const size_t kv_elems = (size_t)Sk * D;  /* one head's dk (or dv) */
    memset(dq, 0, sizeof(double) * (size_t)B * Sq * Hq * D);
    memset(dk, 0, sizeof(double) * (size_t)B * Sk * Hkv * D);
    memset(dv, 0, sizeof(double) * (size_t)B * Sk * Hkv * D);
    /* each (sequence, query head) accumulates its dk, dv into a buffer of its own; the
     * G heads of a K/V head are summed afterwards, in head order */
    double* part = malloc(sizeof(double) * 2 * kv_elems * (size_t)B * Hq + 1);
    if (!part) return -1;
    memset(part, 0, sizeof(double) * 2 * kv_elems * (size_t)B * Hq);
    set_threads(nthreads);
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            double* P = malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
            double* dP = malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
            if (!P || !dP) {
                free(P);
                free(dP);
                bad = 1;
                continue;
            }
            double* pdk = part + 2 * kv_elems * ((size_t)b * Hq + h);
            double* pdv = pdk + kv_elems;
            size_t q_row0, lse_off, lse_step;
            head_view hv = make_view(q, k, v, B, Hq, Hkv, Sq, Sk, D, scale, causal, NULL, b, h,
                                     &q_row0, &lse_off, &lse_step);
            for (int i = 0; i < Sq; ++i) {
                const float* qi = hv.q + (size_t)i * hv.q_stride;
                const float* doi = dout + ((q_row0 + i) * Hq + h) * (size_t)D;
                double m = -INFINITY;
                for (int j = 0; j < Sk; ++j) {
                    P[j] = key_visible(i, j, Sq, Sk, causal)
                               ? scale * dot(qi, hv.k + (size_t)j * hv.kv_stride, D)
                               : -INFINITY;
                    if (P[j] > m) m = P[j];
                }
                if (m == -INFINITY) continue; /* no visible key: no gradient */
                double l = 0.0;
                for (int j = 0; j < Sk; ++j) {
                    P[j] = (P[j] == -INFINITY) ? 0.0 : exp(P[j] - m);
                    l += P[j];
                }
                double Di = 0.0;
                for (int j = 0; j < Sk; ++j) {
                    P[j] /= l;
                    dP[j] = 0.0;
                    if (P[j] == 0.0) continue;
                    for (int d = 0; d < D; ++d)
                        dP[j] += (double)doi[d] * (double)hv.v[(size_t)j * hv.kv_stride + d];
                    Di += P[j] * dP[j];
                }
                if (g_flaw == FLAW_BWD_NO_D) Di = 0.0;
                double* dqi = dq + ((q_row0 + i) * Hq + h) * (size_t)D;
                for (int j = 0; j < Sk; ++j) {
                    if (P[j] == 0.0) continue;
                    const double dS = P[j] * (dP[j] - Di);
                    const float* kj = hv.k + (size_t)j * hv.kv_stride;
                    for (int d = 0; d < D; ++d) {
                        dqi[d] += scale * dS * (double)kj[d];
                        pdk[(size_t)j * D + d] += scale * dS * (double)qi[d];
                        pdv[(size_t)j * D + d] += P[j] * (double)doi[d];
                    }
                }
            }
            free(P);
            free(dP);
        }
    if (!bad)
        for (int b = 0; b < B; ++b)
            for (int c = 0; c < Hkv; ++c)
                for (int h = c * G; h < (c + 1) * G; ++h) {
                    const double* pdk = part + 2 * kv_elems * ((size_t)b * Hq + h);
                    const double* pdv = pdk + kv_elems;
                    for (int j = 0; j < Sk; ++j)
                        for (int d = 0; d < D; ++d) {
                            const size_t o = (((size_t)b * Sk + j) * Hkv + c) * D + d;
                            dk[o] += pdk[(size_t)j * D + d];
                            dv[o] += pdv[(size_t)j * D + d];
                        }
                }
    free(part);
    return bad ? -1 : 0;
}

/*
 * Exact attention restricted to a block pattern (dense layout), optionally causal:
 * key j is visible to query i when its block is listed in the row of i's query block
 * and, with causal, when j <= i + Sk - Sq as well.
 * row_ptr[n_qblk + 1], col[nnz]: key blocks of each query block of `blk` positions;
 * n_qblk = ceil(Sq / blk).  o like q, lse [B, Hq, Sq].  A row whose blocks hold no
 * visible key gets O = 0, L = -inf.
 */
int oracle_attention_blocksparse(const float* q, const float* k, const float* v, double* o,
                                 double* lse, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                                 double scale, int causal, const int32_t* row_ptr,
                                 const int32_t* col, int blk, int nthreads)
{
    if (check_args(q, k, v, B, Hq, Hkv, Sq, Sk, D, NULL) || !o || !lse || !row_ptr || !col ||
        blk <= 0)
        return -1;
    const int n_qblk = (Sq + blk - 1) / blk, n_kblk = (Sk + blk - 1) / blk;
    if (row_ptr[0] != 0) return -1;
    for (int r = 0; r < n_qblk; ++r) {
        if (row_ptr[r + 1] < row_ptr[r]) return -1;
        for (int e = row_ptr[r]; e < row_ptr[r + 1]; ++e)
            if (col[e] < 0 || col[e] >= n_kblk) return -1;
    }
    set_threads(nthreads);
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            size_t q_row0, lse_off, lse_step;
            head_view hv = make_view(q, k, v, B, Hq, Hkv, Sq, Sk, D, scale, 0, NULL, b, h,
                                     &q_row0, &lse_off, &lse_step);
            double* row = malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
            unsigned char* vis = malloc((size_t)(Sk > 0 ? Sk : 1));
            if (!row || !vis) {
                free(row);
                free(vis);
                bad = 1;
                continue;
            }
            for (int i = 0; i < Sq; ++i) {
                int qb = i / blk;
                if (g_flaw == FLAW_SPARSE_ROW && qb + 1 < n_qblk) qb += 1;
                memset(vis, 0, (size_t)Sk);
                for (int e = row_ptr[qb]; e < row_ptr[qb + 1]; ++e)
                    for (int j = col[e] * blk; j < (col[e] + 1) * blk && j < Sk; ++j)
                        vis[j] = (unsigned char)key_visible(i, j, Sq, Sk, causal);
                const float* qi = hv.q + (size_t)i * hv.q_stride;
                double m = -INFINITY;
                for (int j = 0; j < Sk; ++j) {
                    row[j] = vis[j] ? scale * dot(qi, hv.k + (size_t)j * hv.kv_stride, D)
                                    : -INFINITY;
                    if (row[j] > m) m = row[j];
                }
                double* oi = o + ((q_row0 + i) * Hq + h) * (size_t)D;
                if (m == -INFINITY) {
                    for (int d = 0; d < D; ++d) oi[d] = 0.0;
                    lse[lse_off + (size_t)i * lse_step] = -INFINITY;
                    continue;
                }
                double l = 0.0;
                for (int j = 0; j < Sk; ++j) {
                    row[j] = (row[j] == -INFINITY) ? 0.0 : exp(row[j] - m);
                    l += row[j];
                }
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int j = 0; j < Sk; ++j)
                        if (row[j] != 0.0) acc += row[j] * (double)hv.v[(size_t)j * hv.kv_stride + d];
                    oi[d] = acc / l;
                }
                lse[lse_off + (size_t)i * lse_step] = m + log(l);
            }
            free(row);
            free(vis);
        }
    return bad ? -1 : 0;
}

/*
 * Block-sparse attention over packed variable-length sequences with minimum padding
 * (Raptor-T abstract: BigBird's block-sparse attention; its minimum-padding algorithm
 * pads each sequence only to whole blocks instead of to the longest sequence).
 * Sequence b holds n_b = cu[b+1] - cu[b] positions and ceil(n_b / blk) blocks; its
 * query blocks are rows blk_off[b] .. blk_off[b] + ceil(n_b / blk) - 1 of the pattern,
 * blk_off[b] = sum over earlier sequences of their block counts, and their col entries
 * are key blocks of the same sequence, 0 .. ceil(n_b / blk) - 1.  Self attention
 * within each sequence, optionally causal (key j visible to query i only if j <= i).
 * q, k, v, o packed [total, H, D], lse [Hq, total].
 */
int oracle_attention_blocksparse_varlen(const float* q, const float* k, const float* v,
                                        double* o, double* lse, const int32_t* cu, int B,
                                        int Hq, int Hkv, int D, double scale, int causal,
                                        const int32_t* row_ptr, const int32_t* col, int blk,
                                        int nthreads)
{
    if (check_args(q, k, v, B, Hq, Hkv, 0, 0, D, cu) || !o || !lse || !row_ptr || !col ||
        blk <= 0)
        return -1;
    int32_t* off = (int32_t*)malloc(sizeof(int32_t) * (size_t)(B + 1));
    if (!off) return -1;
    int maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (cu[b + 1] - cu[b] > maxlen) maxlen = cu[b + 1] - cu[b];
    off[0] = 0;
    for (int b = 0; b < B; ++b) off[b + 1] = off[b] + (cu[b + 1] - cu[b] + blk - 1) / blk;
    int bad = row_ptr[0] != 0;
    for (int b = 0; b < B && !bad; ++b) {
        const int nkb = (cu[b + 1] - cu[b] + blk - 1) / blk;
        for (int r = off[b]; r < off[b] + nkb && !bad; ++r) {
            if (row_ptr[r + 1] < row_ptr[r]) bad = 1;
            for (int e = row_ptr[r]; e < row_ptr[r + 1] && !bad; ++e)
                if (col[e] < 0 || col[e] >= nkb) bad = 1;
        }
    }
    if (bad) {
        free(off);
        return -1;
    }
    set_threads(nthreads);
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            size_t q_row0, lse_off, lse_step;
            head_view hv = make_view(q, k, v, B, Hq, Hkv, 0, 0, D, scale, 0, cu, b, h, &q_row0,
                                     &lse_off, &lse_step);
            const int n = hv.Sq, nqb = (n + blk - 1) / blk;
            double* row = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
            unsigned char* vis = malloc((size_t)(n > 0 ? n : 1));
            if (!row || !vis) {
                free(row);
                free(vis);
                bad = 1;
                continue;
            }
            for (int i = 0; i < n; ++i) {
                int qb = i / blk;
                if (g_flaw == FLAW_SPARSE_ROW && qb + 1 < nqb) qb += 1;
                int r = off[b] + qb;
                if (g_flaw == FLAW_SPARSE_MAXPAD) { /* rows of max-padded sequences */
                    r = b * ((maxlen + blk - 1) / blk) + qb;
                    if (r >= off[B]) r = off[B] - 1;
                }
                memset(vis, 0, (size_t)n);
                for (int e = row_ptr[r]; e < row_ptr[r + 1]; ++e)
                    for (int j = col[e] * blk; j < (col[e] + 1) * blk && j < n; ++j)
                        vis[j] = (unsigned char)key_visible(i, j, n, n, causal);
                const float* qi = hv.q + (size_t)i * hv.q_stride;
                double m = -INFINITY;
                for (int j = 0; j < n; ++j) {
                    row[j] = vis[j] ? scale * dot(qi, hv.k + (size_t)j * hv.kv_stride, D)
                                    : -INFINITY;
                    if (row[j] > m) m = row[j];
                }
                double* oi = o + ((q_row0 + i) * Hq + h) * (size_t)D;
                if (m == -INFINITY) {
                    for (int d = 0; d < D; ++d) oi[d] = 0.0;
                    lse[lse_off + (size_t)i * lse_step] = -INFINITY;
                    continue;
                }
                double l = 0.0;
                for (int j = 0; j < n; ++j) {
                    row[j] = (row[j] == -INFINITY) ? 0.0 : exp(row[j] - m);
                    l += row[j];
                }
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int j = 0; j < n; ++j)
                        if (row[j] != 0.0) acc += row[j] * (double)hv.v[(size_t)j * hv.kv_stride + d];
                    oi[d] = acc / l;
                }
                lse[lse_off + (size_t)i * lse_step] = m + log(l);
            }
            free(row);
            free(vis);
        }
    free(off);
    return bad ? -1 : 0;
}

/* Value of one e4m3 code. */
static double e4m3_value(uint8_t c)
{
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    const int bias = (g_flaw == FLAW_E4M3_BIAS) ? 8 : 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = (e == 0) ? ldexp((double)m / 8.0, 1 - bias)
                                : ldexp(1.0 + (double)m / 8.0, e - bias);
    return sign ? -mag : mag;
}

/* All 256 code values (out[256]). */
void oracle_e4m3_table(double* out)
{
    for (int c = 0; c < 256; ++c) out[c] = e4m3_value((uint8_t)c);
}

/* Element of a cache: float value, or e4m3 code times its scale (lut holds the 256
 * code values, filled by e4m3_value for each call). */
typedef struct {
    const float* f;
    const uint8_t* c;
    double scale;
    const double* lut;
} cache_src;

static double cache_at(const cache_src* src, size_t i)
{
    return src->f ? (double)src->f[i] : src->lut[src->c[i]] * src->scale;
}

/*
 * One decode query per sequence against a KV cache, by the plain definition.
 *   q [B, Hq, D]; o [B, Hq, D]; lse [B, Hq].
 *   dense (block_table NULL): k_cache, v_cache [B, Sk, Hkv, D];
 *   paged: k_cache, v_cache [num_pages, page_size, Hkv, D], block_table
 *     [B, max_pages];
 *   seqlens_k [B] keys per sequence, or NULL: Sk each (dense only);
 *   window > 0: keys j in [max(0, L - window), L), else [0, L).
 * For each (b, h): s_j = scale * q . k_j over those keys, m = max s_j,
 * p_j = exp(s_j - m), l = sum p_j, O = sum p_j v_j / l, L = m + ln l; no key:
 * O = 0, L = -inf.
 */
static int decode_core(const float* q, const cache_src* ks, const cache_src* vs,
                       const int32_t* block_table, const int32_t* seqlens_k, double* o,
                       double* lse, int B, int Hq, int Hkv, int D, int Sk, int page_size,
                       int max_pages, int num_pages, int window, double scale, int nthreads)
{
    if (!q || !(ks->f || ks->c) || !(vs->f || vs->c) || !o || !lse) return -1;
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0 || window < 0) return -1;
    const int paged = block_table != NULL;
    int cap = Sk;
    if (paged) {
        if (!seqlens_k || page_size <= 0 || max_pages <= 0 || num_pages <= 0) return -1;
        cap = max_pages * page_size;
    } else if (Sk < 0) {
        return -1;
    }
    for (int b = 0; b < B; ++b) {
        const int L = seqlens_k ? seqlens_k[b] : Sk;
        if (L < 0 || L > cap) return -1;
        if (paged)
            for (int pg = 0; pg < (L + page_size - 1) / page_size; ++pg) {
                const int32_t e = block_table[(size_t)b * max_pages + pg];
                if (e < 0 || e >= num_pages) return -1;
            }
    }
    set_threads(nthreads);
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            const int L = seqlens_k ? seqlens_k[b] : Sk;
            int j0 = 0;
            if (window > 0) {
                j0 = L - window;
                if (g_flaw == FLAW_WINDOW_SHORT) j0 += 1;
                if (j0 < 0) j0 = 0;
            }
            const int c = kv_head_of(h, Hq, Hkv);
            const float* qv = q + ((size_t)b * Hq + h) * D;
            double* ob = o + ((size_t)b * Hq + h) * D;
            double* row = (L > j0) ? malloc(sizeof(double) * (size_t)(L - j0)) : NULL;
            if (L > j0 && !row) {
                bad = 1;
                continue;
            }
            /* row index of key j in the cache arrays */
            size_t* kr = (L > j0) ? malloc(sizeof(size_t) * (size_t)(L - j0)) : NULL;
            if (L > j0 && !kr) {
                free(row);
                bad = 1;
                continue;
            }
            for (int j = j0; j < L; ++j) {
                size_t r;
                if (!paged)
                    r = (size_t)b * Sk + j;
                else if (g_flaw == FLAW_PAGES_CONTIGUOUS)
                    r = (size_t)b * max_pages * page_size + j;
                else
                    r = (size_t)block_table[(size_t)b * max_pages + j / page_size] * page_size +
                        (size_t)(j % page_size);
                kr[j - j0] = r;
            }
            double m = -INFINITY;
            for (int j = j0; j < L; ++j) {
                const size_t kb = (kr[j - j0] * Hkv + c) * (size_t)D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += (double)qv[d] * cache_at(ks, kb + d);
                row[j - j0] = scale * acc;
                if (row[j - j0] > m) m = row[j - j0];
            }
            if (L <= j0) {
                for (int d = 0; d < D; ++d) ob[d] = 0.0;
                lse[(size_t)b * Hq + h] = -INFINITY;
                continue;
            }
            double l = 0.0;
            for (int j = j0; j < L; ++j) {
                row[j - j0] = exp(row[j - j0] - m);
                l += row[j - j0];
            }
            for (int d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int j = j0; j < L; ++j)
                    acc += row[j - j0] * cache_at(vs, (kr[j - j0] * Hkv + c) * (size_t)D + d);
                ob[d] = acc / l;
            }
            lse[(size_t)b * Hq + h] = m + log(l);
            free(row);
            free(kr);
        }
    return bad ? -1 : 0;
}

int oracle_decode_kvcache(const float* q, const float* k_cache, const float* v_cache,
                          const int32_t* block_table, const int32_t* seqlens_k, double* o,
                          double* lse, int B, int Hq, int Hkv, int D, int Sk, int page_size,
                          int max_pages, int num_pages, int window, double scale, int nthreads)
{
    const cache_src ks = {k_cache, NULL, 1.0, NULL}, vs = {v_cache, NULL, 1.0, NULL};
    return decode_core(q, &ks, &vs, block_table, seqlens_k, o, lse, B, Hq, Hkv, D, Sk,
                       page_size, max_pages, num_pages, window, scale, nthreads);
}

/* The same with e4m3 codes: key element = value(code) * k_scale, likewise for V. */
int oracle_decode_kvcache_e4m3(const float* q, const uint8_t* k8, const uint8_t* v8,
                               double k_scale, double v_scale, const int32_t* block_table,
                               const int32_t* seqlens_k, double* o, double* lse, int B, int Hq,
                               int Hkv, int D, int Sk, int page_size, int max_pages,
                               int num_pages, int window, double scale, int nthreads)
{
    if (!k8 || !v8) return -1;
    double lut[256];
    oracle_e4m3_table(lut);
    const cache_src ks = {NULL, k8, k_scale, lut}, vs = {NULL, v8, v_scale, lut};
    return decode_core(q, &ks, &vs, block_table, seqlens_k, o, lse, B, Hq, Hkv, D, Sk,
                       page_size, max_pages, num_pages, window, scale, nthreads);
}

/*
 * Prefill with e4m3 Q, K and V (the batch-size guide names FP8 as the precision that
 * lowers memory-bandwidth pressure: hardware adaptation section, Hopper item, and the
 * precision row of its production checklist).  Each tensor holds codes with one scale:
 * element = value(code) * scale of that tensor.  The result is the plain definition
 * on those elements: S = scale * (q_scale Q)(k_scale K)^T, P = softmax(S),
 * O = P (v_scale V), L = m + ln l.  The code values are exact in float, so the codes
 * are decoded once and the per-tensor scales enter in double: q_scale * k_scale with
 * the logit scale, v_scale on O.  A NaN code (0x7f, 0xff) is rejected.
 */
int oracle_attention_e4m3(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                          double q_scale, double k_scale, double v_scale, double* o,
                          double* lse, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                          double scale, int causal, const int32_t* cu_seqlens, int nthreads)
{
    if (check_args(q8, k8, v8, B, Hq, Hkv, Sq, Sk, D, cu_seqlens) || !o || !lse) return -1;
    const size_t nq = (size_t)(cu_seqlens ? cu_seqlens[B] : B * Sq) * Hq * D;
    const size_t nk = (size_t)(cu_seqlens ? cu_seqlens[B] : B * Sk) * Hkv * D;
    float* q = (float*)malloc(sizeof(float) * (nq ? nq : 1));
    float* k = (float*)malloc(sizeof(float) * (nk ? nk : 1));
    float* v = (float*)malloc(sizeof(float) * (nk ? nk : 1));
    int rc = (q && k && v) ? 0 : -1;
    double lut[256];
    oracle_e4m3_table(lut);
    for (size_t i = 0; rc == 0 && i < nq; ++i) {
        if (isnan(lut[q8[i]])) rc = -1;
        q[i] = (float)lut[q8[i]];
    }
    for (size_t i = 0; rc == 0 && i < nk; ++i) {
        if (isnan(lut[k8[i]]) || isnan(lut[v8[i]])) rc = -1;
        k[i] = (float)lut[k8[i]];
        v[i] = (float)lut[v8[i]];
    }
    if (rc == 0)
        rc = oracle_attention(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, D, scale * q_scale * k_scale,
                              causal, cu_seqlens, nthreads);
    if (rc == 0 && g_flaw != FLAW_E4M3_NO_VSCALE)
        for (size_t i = 0; i < nq; ++i) o[i] *= v_scale;
    free(q);
    free(k);
    free(v);
    return rc;
}

/*
 * The tiled (online-softmax) forms of the same forward, in float64, on a dense
 * problem.  The outer loop walks query row blocks of Bm rows, the inner loop key
 * blocks of Bn columns, skipping blocks that lie entirely above the causal
 * diagonal.  Per row the running max m and sum l are updated per key block.
 *   form 1, per-step normalised update (FlashAttention-2 summary page, first
 *     equation of the normalisation paragraph):
 *       O_j = diag(l_{j-1} e^{m_{j-1} - m_j} / l_j) O_{j-1}
 *             + diag(l_j)^{-1} e^{S_j - m_j} V_j
 *     (the page prints the carried term as diag(l_{j-1}/l_j) O_{j-1}, with the
 *     max-shift factor left implicit; it is written out here);
 *   form 2, deferred normalisation (second equation):
 *       Ot_j = diag(e^{m_{j-1} - m_j}) Ot_{j-1} + e^{S_j - m_j} V_j,
 *     one division by l at the end;
 *   both: L = m + ln l.
 */
int oracle_attention_tiled(const float* q, const float* k, const float* v, double* o,
                           double* lse, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                           double scale, int causal, int Bm, int Bn, int form)
{
    if (check_args(q, k, v, B, Hq, Hkv, Sq, Sk, D, NULL) || !o || !lse) return -1;
    if (Bm <= 0 || Bn <= 0 || (form != 1 && form != 2)) return -1;
    double* m = (double*)malloc(sizeof(double) * (size_t)Bm);
    double* l = (double*)malloc(sizeof(double) * (size_t)Bm);
    double* acc = (double*)malloc(sizeof(double) * (size_t)Bm * D);
    double* sblk = (double*)malloc(sizeof(double) * (size_t)Bm * Bn);
    if (!m || !l || !acc || !sblk) {
        free(m); free(l); free(acc); free(sblk);
        return -1;
    }
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            size_t qrow0, lse_off, lse_step;
            head_view hv = make_view(q, k, v, B, Hq, Hkv, Sq, Sk, D, scale, causal, NULL, b, h,
                                     &qrow0, &lse_off, &lse_step);
            for (int i0 = 0; i0 < Sq; i0 += Bm) {
                const int bm = (Sq - i0 < Bm) ? Sq - i0 : Bm;
                for (int r = 0; r < bm; ++r) {
                    m[r] = -INFINITY;
                    l[r] = 0.0;
                    for (int d = 0; d < D; ++d) acc[(size_t)r * D + d] = 0.0;
                }
                for (int j0 = 0; j0 < Sk; j0 += Bn) {
                    const int bn = (Sk - j0 < Bn) ? Sk - j0 : Bn;
                    /* block entirely above the diagonal: every key invisible to every row */
                    if (causal && !key_visible(i0 + bm - 1, j0, Sq, Sk, causal)) continue;
                    for (int r = 0; r < bm; ++r) {
                        const int i = i0 + r;
                        const float* qi = hv.q + (size_t)i * hv.q_stride;
                        double mblk = -INFINITY;
                        for (int c = 0; c < bn; ++c) {
                            const int j = j0 + c;
                            double s = -INFINITY;
                            if (key_visible(i, j, Sq, Sk, causal))
                                s = scale * dot(qi, hv.k + (size_t)j * hv.kv_stride, D);
                            sblk[(size_t)r * Bn + c] = s;
                            if (s > mblk) mblk = s;
                        }
                        const double mnew = (mblk > m[r]) ? mblk : m[r];
                        if (mnew == -INFINITY) continue; /* nothing visible yet */
                        const double carry =
                            (m[r] == -INFINITY) ? 0.0
                            : (g_flaw == FLAW_FA1_NO_RESCALE && form == 1) ? 1.0
                                                                           : exp(m[r] - mnew);
                        double rowsum = 0.0;
                        for (int c = 0; c < bn; ++c) {
                            const double s = sblk[(size_t)r * Bn + c];
                            const double p = (s == -INFINITY) ? 0.0 : exp(s - mnew);
                            sblk[(size_t)r * Bn + c] = p;
                            rowsum += p;
                        }
                        const double lnew = carry * l[r] + rowsum;
                        double* ar = acc + (size_t)r * D;
                        for (int d = 0; d < D; ++d) {
                            double pv = 0.0;
                            for (int c = 0; c < bn; ++c)
                                pv += sblk[(size_t)r * Bn + c] *
                                      (double)hv.v[(size_t)(j0 + c) * hv.kv_stride + d];
                            if (form == 1) /* running O stays normalised by l_j */
                                ar[d] = (l[r] * carry / lnew) * ar[d] + pv / lnew;
                            else /* running O-tilde, unnormalised */
                                ar[d] = carry * ar[d] + pv;
                        }
                        m[r] = mnew;
                        l[r] = lnew;
                    }
                }
                for (int r = 0; r < bm; ++r) {
                    const int i = i0 + r;
                    double* orow = o + ((qrow0 + (size_t)i) * Hq + h) * (size_t)D;
                    if (m[r] == -INFINITY) {
                        for (int d = 0; d < D; ++d) orow[d] = 0.0;
                        lse[lse_off + (size_t)i] = -INFINITY;
                        continue;
                    }
                    for (int d = 0; d < D; ++d)
                        orow[d] = (form == 1) ? acc[(size_t)r * D + d]
                                              : acc[(size_t)r * D + d] / l[r];
                    lse[lse_off + (size_t)i] = m[r] + log(l[r]);
                }
            }
        }
    free(m); free(l); free(acc); free(sblk);
    return 0;
}
