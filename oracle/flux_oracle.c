/*
 * flux_oracle.c -- the reference (oracle) implementation of Flux Attention's
 * routed-attention hot path, written for checking, not for speed.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library under sparse_attention_flux_b200/) never calls it, shares no
 * code, header, table or helper with it, and fails loudly when its own CUDA
 * extension is missing instead of falling back here.
 *
 * Everything is computed in IEEE fp64 from the exact values the GPU sees:
 * bf16 tensors arrive as raw 16-bit patterns and are widened exactly to
 * double; router weights arrive as fp32 and are widened exactly.  Each
 * function is the plain definition of one step, with no blocking, fusion or
 * reordering beyond what the definition states.  OpenMP only distributes
 * independent (batch, head, query) rows over cores; each row's arithmetic is
 * the same sequential loop whatever the thread count.
 *
 * Sources (web pages about "Flux Attention: Context-Aware Hybrid Attention
 * for Efficient LLMs Inference", arXiv 2604.07394):
 *  - gist.science technical summary, section 2 "Methodology":
 *      "Layer Router" -- pool the first and last 100 prompt tokens, pass the
 *      result through an MLP context encoder, decide FA or SA per layer;
 *      "switch to hard routing" -- threshold the soft weight into a 0/1
 *      decision at inference;
 *      "efficient deployment" -- route once at prefill, reuse for every
 *      decode step; SA layers keep and read only the minimal KV.
 *  - Hugging Face model card "Flux Attention: Qwen3-4B", "Sample Usage":
 *      SA layers run on a block-sparse attention library.
 *  - arXiv abstract (fugumt / chatpaper pages): FA is exact full attention,
 *      SA a sparse attention; routing is per layer, not per head.
 * Readings where the pages are silent (listed with reasons in the design
 * notes): the two pooled means are concatenated; the MLP is
 * Linear -> ReLU -> Linear with one logit per layer; mode = FA iff
 * sigmoid(z) > thresh (a tie goes to SA); the SA block mask is sink blocks
 * plus a local window of W blocks that includes the diagonal block, with
 * token-level causal masking; GQA maps query head h to kv head h / (Hq/Hkv).
 *
 * Parity pins: every function here is pinned by tests/test_oracle.py against
 * closed forms, invariants, hand-enumerated fixtures and a library routine
 * (torch's scaled-dot-product attention in fp64 with an explicit mask).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Exact widening of a bf16 bit pattern: a bf16 value is the top half of the
 * fp32 with the same sign, exponent and leading mantissa bits. */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ---------------------------------------------------------------------------
 * Layer Router, step 1: pooling (gist.science summary, section 2, "Layer
 * Router": the first and last 100 prompt tokens are pooled).
 * hidden: [T, Hd] bf16 bits, row-major.  n = min(n_pool, T) rows per side.
 * p[0:Hd]    = mean of rows 0 .. n-1
 * p[Hd:2Hd]  = mean of rows T-n .. T-1
 * (The two windows may overlap when T < 2 n_pool.)
 * ------------------------------------------------------------------------- */
int oracle_pool(const uint16_t* hidden, int T, int Hd, int n_pool, double* p) {
    if (!hidden || !p || T <= 0 || Hd <= 0 || n_pool <= 0) return -1;
    int n = n_pool < T ? n_pool : T;
    for (int c = 0; c < Hd; ++c) {
        double head = 0.0, tail = 0.0;
        for (int t = 0; t < n; ++t) head += bf16_to_double(hidden[(size_t)t * Hd + c]);
        for (int t = T - n; t < T; ++t) tail += bf16_to_double(hidden[(size_t)t * Hd + c]);
        p[c] = head / n;
        p[Hd + c] = tail / n;
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Layer Router, step 2: the context-encoder MLP (gist.science summary,
 * section 2, "Layer Router").  u = relu(W1 p + b1); z = W2 u + b2.
 * W1: [H1, in] fp32 row-major, W2: [L, H1] fp32 row-major.
 * ------------------------------------------------------------------------- */
int oracle_mlp(const double* p, int in_dim, const float* W1, const float* b1, int H1,
               const float* W2, const float* b2, int L, double* z) {
    if (!p || !W1 || !b1 || !W2 || !b2 || !z || in_dim <= 0 || H1 <= 0 || L <= 0) return -1;
    double* u = (double*)malloc(sizeof(double) * (size_t)H1);
    if (!u) return -1;
    for (int j = 0; j < H1; ++j) {
        double acc = (double)b1[j];
        for (int i = 0; i < in_dim; ++i) acc += (double)W1[(size_t)j * in_dim + i] * p[i];
        u[j] = acc > 0.0 ? acc : 0.0;
    }
    for (int l = 0; l < L; ++l) {
        double acc = (double)b2[l];
        for (int j = 0; j < H1; ++j) acc += (double)W2[(size_t)l * H1 + j] * u[j];
        z[l] = acc;
    }
    free(u);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Layer Router, step 3: hard routing (gist.science summary, section 2,
 * "switch to hard routing": the soft weight is thresholded into 0/1).
 * r = sigmoid(z) is the soft FA weight; mode = 1 (FA) iff r > thresh.
 * The comparison is taken in fp32, the precision the GPU kernel decides in:
 * r is rounded once from fp64 to fp32 and compared with fp32 thresh.
 * ------------------------------------------------------------------------- */
int oracle_threshold(const double* z, int L, float thresh, uint8_t* mode, double* r_out) {
    if (!z || !mode || L <= 0) return -1;
    for (int l = 0; l < L; ++l) {
        double r = 1.0 / (1.0 + exp(-z[l]));
        float r32 = (float)r;
        mode[l] = (r32 > thresh) ? 1 : 0;
        if (r_out) r_out[l] = r;
    }
    return 0;
}

/* The three router steps in order (route once, at prefill). */
int oracle_route(const uint16_t* hidden, int T, int Hd, int n_pool,
                 const float* W1, const float* b1, int H1,
                 const float* W2, const float* b2, int L, float thresh,
                 uint8_t* mode, double* z_out, double* r_out) {
    double* p = (double*)malloc(sizeof(double) * 2 * (size_t)Hd);
    double* z = (double*)malloc(sizeof(double) * (size_t)L);
    int rc = -1;
    if (p && z && oracle_pool(hidden, T, Hd, n_pool, p) == 0 &&
        oracle_mlp(p, 2 * Hd, W1, b1, H1, W2, b2, L, z) == 0 &&
        oracle_threshold(z, L, thresh, mode, r_out) == 0) {
        if (z_out) memcpy(z_out, z, sizeof(double) * (size_t)L);
        rc = 0;
    }
    free(p);
    free(z);
    return rc;
}

/* ---------------------------------------------------------------------------
 * SA block mask: sink blocks plus a local window (block-sparse attention,
 * model card "Sample Usage"; sink + recent-token pattern).  For q-block i and
 * kv-block j:  mask[i][j] = (j <= i) && (j < sink || j >= i - W + 1).
 * ------------------------------------------------------------------------- */
int oracle_streaming_mask(int nqb, int nkb, int sink_blocks, int window_blocks, uint8_t* mask) {
    if (!mask || nqb <= 0 || nkb <= 0 || sink_blocks < 0 || window_blocks < 1) return -1;
    for (int i = 0; i < nqb; ++i)
        for (int j = 0; j < nkb; ++j)
            mask[(size_t)i * nkb + j] =
                (uint8_t)((j <= i) && (j < sink_blocks || j >= i - window_blocks + 1));
    return 0;
}

/* Compressed block-index list (CSR): for each q-block i, the ascending kv
 * blocks j with mask[i][j] != 0.  row_ptr has nqb+1 entries; col must hold
 * nqb*nkb entries.  Returns nnz. */
int oracle_block_index(const uint8_t* mask, int nqb, int nkb, int32_t* row_ptr, int32_t* col) {
    if (!mask || !row_ptr || !col || nqb <= 0 || nkb <= 0) return -1;
    int32_t nnz = 0;
    for (int i = 0; i < nqb; ++i) {
        row_ptr[i] = nnz;
        for (int j = 0; j < nkb; ++j)
            if (mask[(size_t)i * nkb + j]) col[nnz++] = j;
    }
    row_ptr[nqb] = nnz;
    return nnz;
}

/* Is key u visible to query t?  Causal always; with a block mask, the block
 * pair must also be kept.  mask == NULL means Full Attention. */
static int key_allowed(int t, int u, const uint8_t* mask, int nkb, int block) {
    if (u > t) return 0;
    if (!mask) return 1;
    return mask[(size_t)(t / block) * nkb + (u / block)] != 0;
}

/* Softmax attention for one query row over an explicit list of allowed keys.
 * q: d values; keys at k + key_index*kstride, values likewise.
 * o = sum_u P_u v_u with P_u = exp(s_u - m) / sum exp(s - m),
 * s_u = scale * <q, k_u>.  lse = m + log(sum exp(s - m)) (natural log).
 * With no allowed key: o = 0, lse = -inf. */
static void attend_row(const double* q, const uint16_t* k, const uint16_t* v, size_t kstride,
                       const int32_t* keys, int nkeys, int d, double scale,
                       double* s, double* o, double* lse) {
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    if (nkeys == 0) {
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int a = 0; a < nkeys; ++a) {
        const uint16_t* kr = k + (size_t)keys[a] * kstride;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += q[c] * bf16_to_double(kr[c]);
        s[a] = scale * dot;
        if (s[a] > m) m = s[a];
    }
    double sum = 0.0;
    for (int a = 0; a < nkeys; ++a) {
        s[a] = exp(s[a] - m);
        sum += s[a];
    }
    for (int a = 0; a < nkeys; ++a) {
        const uint16_t* vr = v + (size_t)keys[a] * kstride;
        double pa = s[a] / sum;
        for (int c = 0; c < d; ++c) o[c] += pa * bf16_to_double(vr[c]);
    }
    *lse = m + log(sum);
}

/* ---------------------------------------------------------------------------
 * Prefill attention, FA or SA (arXiv abstract: FA = exact causal full
 * attention; SA = block-sparse attention over the mask above).
 * q: [B, T, Hq, d] bf16 bits; k, v: [B, T, Hkv, d] bf16 bits.
 * rows: n_rows triples (b, h, t) to compute, or NULL for every row in
 * (b, t, h) order.  o: [n_rows, d] fp64; lse: [n_rows] fp64 (may be NULL).
 * block_mask: [nqb, nkb] or NULL for FA.  Query head h reads kv head
 * h / (Hq / Hkv).
 * ------------------------------------------------------------------------- */
int oracle_attn_prefill(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        int B, int T, int Hq, int Hkv, int d,
                        const uint8_t* block_mask, int nkb, int block, double scale,
                        const int32_t* rows, long long n_rows, double* o, double* lse) {
    if (!q || !k || !v || !o || B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (block_mask && (block <= 0 || nkb < (T + block - 1) / block)) return -1;
    const int G = Hq / Hkv;
    long long total = rows ? n_rows : (long long)B * T * Hq;
    int bad = 0;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)T);
        int32_t* keys = (int32_t*)malloc(sizeof(int32_t) * (size_t)T);
        double* qd = (double*)malloc(sizeof(double) * (size_t)d);
        double lse_r;
#pragma omp for schedule(dynamic, 16)
        for (long long r = 0; r < total; ++r) {
            int b, h, t;
            if (rows) {
                b = rows[3 * r];
                h = rows[3 * r + 1];
                t = rows[3 * r + 2];
            } else {
                b = (int)(r / ((long long)T * Hq));
                t = (int)((r / Hq) % T);
                h = (int)(r % Hq);
            }
            if (!s || !keys || !qd || b < 0 || b >= B || h < 0 || h >= Hq || t < 0 || t >= T) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            const int g = h / G;
            const uint16_t* qr = q + (((size_t)b * T + t) * Hq + h) * d;
            for (int c = 0; c < d; ++c) qd[c] = bf16_to_double(qr[c]);
            int nk = 0;
            for (int u = 0; u <= t; ++u)
                if (key_allowed(t, u, block_mask, nkb, block)) keys[nk++] = u;
            const uint16_t* kb = k + ((size_t)b * T * Hkv + g) * d;
            const uint16_t* vb = v + ((size_t)b * T * Hkv + g) * d;
            attend_row(qd, kb, vb, (size_t)Hkv * d, keys, nk, d, scale, s, o + (size_t)r * d, &lse_r);
            if (lse) lse[r] = lse_r;
        }
        free(s);
        free(keys);
        free(qd);
    }
    return bad ? -1 : 0;
}

/* Soft routing, forward only (gist.science summary, section 2, "training
 * process": the continuous weight r_soft forms the convex combination of the
 * FA and SA outputs).  o = r * FA + (1 - r) * SA, row by row, with the SA
 * block mask given.  rows as in oracle_attn_prefill. */
int oracle_attn_prefill_soft(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             int B, int T, int Hq, int Hkv, int d,
                             const uint8_t* block_mask, int nkb, int block, double scale, double r,
                             const int32_t* rows, long long n_rows, double* o) {
    if (!block_mask) return -1;
    long long total = rows ? n_rows : (long long)B * T * Hq;
    double* o_fa = (double*)malloc(sizeof(double) * (size_t)total * d);
    double* o_sa = (double*)malloc(sizeof(double) * (size_t)total * d);
    int rc = -1;
    if (o_fa && o_sa &&
        oracle_attn_prefill(q, k, v, B, T, Hq, Hkv, d, NULL, 0, 0, scale, rows, n_rows, o_fa, NULL) == 0 &&
        oracle_attn_prefill(q, k, v, B, T, Hq, Hkv, d, block_mask, nkb, block, scale, rows, n_rows,
                            o_sa, NULL) == 0) {
        for (long long i = 0; i < total * d; ++i) o[i] = r * o_fa[i] + (1.0 - r) * o_sa[i];
        rc = 0;
    }
    free(o_fa);
    free(o_sa);
    return rc;
}

/* The full probability matrix P[t][u] of one (b, h) pair, T x T, for the
 * invariant checks (rows sum to one, masked and causal entries are zero). */
int oracle_attn_probs(const uint16_t* q, const uint16_t* k, int B, int T, int Hq, int Hkv, int d,
                      const uint8_t* block_mask, int nkb, int block, double scale,
                      int b, int h, double* P) {
    if (!q || !k || !P || b < 0 || b >= B || h < 0 || h >= Hq || Hq % Hkv) return -1;
    const int g = h / (Hq / Hkv);
    double* s = (double*)malloc(sizeof(double) * (size_t)T);
    if (!s) return -1;
    for (int t = 0; t < T; ++t) {
        const uint16_t* qr = q + (((size_t)b * T + t) * Hq + h) * d;
        double m = -INFINITY;
        for (int u = 0; u < T; ++u) {
            s[u] = -INFINITY;
            if (!key_allowed(t, u, block_mask, nkb, block)) continue;
            const uint16_t* kr = k + (((size_t)b * T + u) * Hkv + g) * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += bf16_to_double(qr[c]) * bf16_to_double(kr[c]);
            s[u] = scale * dot;
            if (s[u] > m) m = s[u];
        }
        double sum = 0.0;
        for (int u = 0; u < T; ++u) {
            double e = (s[u] == -INFINITY) ? 0.0 : exp(s[u] - m);
            P[(size_t)t * T + u] = e;
            sum += e;
        }
        for (int u = 0; u < T; ++u) P[(size_t)t * T + u] = sum > 0.0 ? P[(size_t)t * T + u] / sum : 0.0;
    }
    free(s);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Decode attention for one new query per sequence (gist.science summary,
 * section 2, "efficient deployment": the routing bit chosen at prefill is
 * reused; SA layers read only the minimal KV -- the sink blocks and the last
 * W blocks -- and never the history in between).
 * q: [B, Hq, d] bf16 bits, the query of the token at position s-1.
 * k_cache, v_cache: [B, S_max, Hkv, d] bf16 bits; seqlens[b] = s (tokens in
 * the cache, including the new one).  mode: 1 = FA (all u < s), 0 = SA
 * (floor(u/block) < sink or floor(u/block) >= ceil(s/block) - W).
 * o: [B, Hq, d] fp64; lse: [B, Hq] fp64 (may be NULL).
 * ------------------------------------------------------------------------- */
int oracle_attn_decode(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                       int S_max, const int32_t* seqlens, int B, int Hq, int Hkv, int d,
                       int mode, int sink_blocks, int window_blocks, int block, double scale,
                       double* o, double* lse) {
    if (!q || !k_cache || !v_cache || !seqlens || !o || B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0)
        return -1;
    if (Hq % Hkv || block <= 0 || window_blocks < 1 || sink_blocks < 0) return -1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > S_max) return -1;
    const int G = Hq / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)S_max);
        int32_t* keys = (int32_t*)malloc(sizeof(int32_t) * (size_t)S_max);
        double* qd = (double*)malloc(sizeof(double) * (size_t)d);
        double lse_r;
#pragma omp for schedule(dynamic, 1)
        for (long long r = 0; r < (long long)B * Hq; ++r) {
            if (!s || !keys || !qd) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            const int b = (int)(r / Hq), h = (int)(r % Hq), g = h / G;
            const int sl = seqlens[b];
            const int nbs = (sl + block - 1) / block;
            int nk = 0;
            for (int u = 0; u < sl; ++u) {
                const int j = u / block;
                if (mode == 1 || j < sink_blocks || j >= nbs - window_blocks) keys[nk++] = u;
            }
            const uint16_t* qr = q + ((size_t)b * Hq + h) * d;
            for (int c = 0; c < d; ++c) qd[c] = bf16_to_double(qr[c]);
            const uint16_t* kb = k_cache + ((size_t)b * S_max * Hkv + g) * d;
            const uint16_t* vb = v_cache + ((size_t)b * S_max * Hkv + g) * d;
            attend_row(qd, kb, vb, (size_t)Hkv * d, keys, nk, d, scale, s, o + (size_t)r * d, &lse_r);
            if (lse) lse[r] = lse_r;
        }
        free(s);
        free(keys);
        free(qd);
    }
    return bad ? -1 : 0;
}

/*
 * Dynamic SA block selection.  The pages name a block-sparse selector as the
 * SA side's prior art (the checkpoint page's repository name
 * "full_xattn_Qwen3-4B"; XAttention among the sparse methods in the UniSparse
 * abstract on the page list) but give no algorithm.  The reading implemented
 * here follows the published idea of that family -- score each block by
 * antidiagonal sums over strided positions, then keep the fewest blocks whose
 * score mass reaches a threshold -- with every detail fixed as follows:
 *   strided positions r = 0 .. nr-1, nr = ceil(T / S): token rows r*S .. r*S+S-1,
 *     a row >= T reading as a zero vector;
 *   antidiagonal logit  z[r][c] = scale * sum_{k<S} q[r*S+k] . key[c*S+S-1-k],  c <= r;
 *   block mass  E_h[i][j] = sum of exp(z[r][c]) over the strided rows r of query
 *     block i and strided columns c of key block j (R = block / S of each), c <= r;
 *   P_h[i][j] = E_h[i][j] / sum_{j' <= i} E_h[i][j']: the share of query block
 *     i's antidiagonal attention mass that falls in key block j (head h of
 *     sequence b, kv head h / (Hq/Hkv));
 *   layer score  P[i][j] = mean over (b, h) of P_h[i][j].
 * Parity unpinned against the pages (they print no algorithm); these
 * functions are pinned to brute force, closed forms and invariants of the
 * definition above.  oracle_block_scores_rows computes the rows of the
 * listed query blocks only (P [nrows][nb], row n = query block rows[n]):
 * each row depends on its own block's queries alone, so large layers are
 * checked on sampled rows.
 */
int oracle_block_scores_rows(const uint16_t* q, const uint16_t* k, int B, int T, int Hq,
                             int Hkv, int d, int block, int stride, double scale,
                             const int* rows, int nrows, double* P) {
    if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || d < 1 || stride < 1 ||
        block < stride || block % stride || nrows < 1 || !rows) return -1;
    const int G = Hq / Hkv, S = stride, R = block / S;
    const int nr = (T + S - 1) / S, nb = (nr + R - 1) / R;
    for (int n = 0; n < nrows; ++n)
        if (rows[n] < 0 || rows[n] >= nb) return -1;
    const int nbh = B * Hq;
    double* Ph = (double*)calloc((size_t)nbh * nrows * nb, sizeof(double));
    if (!Ph) return -1;
    int bad = 0;
#pragma omp parallel
    {
        double* qs = (double*)malloc(sizeof(double) * (size_t)R * S * d);   /* block i's rows */
        double* ks = (double*)malloc(sizeof(double) * (size_t)S * d);       /* one strided col */
        double* z = (double*)malloc(sizeof(double) * (size_t)R * nr);
#pragma omp for schedule(dynamic, 1)
        for (long long w = 0; w < (long long)nbh * nrows; ++w) {
            if (!qs || !ks || !z) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            const int bh = (int)(w / nrows), n = (int)(w % nrows), i = rows[n];
            const int b = bh / Hq, h = bh % Hq, g = h / G;
            const int r0 = i * R, r1 = r0 + R < nr ? r0 + R : nr;
            /* the query rows of block i, widened (zero past T) */
            for (int r = r0; r < r1; ++r)
                for (int kk = 0; kk < S; ++kk) {
                    const int t = r * S + kk;
                    double* dst = qs + ((size_t)(r - r0) * S + kk) * d;
                    for (int c = 0; c < d; ++c)
                        dst[c] = t < T ? bf16_to_double(q[(((size_t)b * T + t) * Hq + h) * d + c]) : 0.0;
                }
            /* logits z[r][c] for c <= r, and their maximum */
            double zmax = -INFINITY;
            for (int cc = 0; cc < r1; ++cc) {
                for (int kk = 0; kk < S; ++kk) {
                    const int u = cc * S + S - 1 - kk;
                    for (int c = 0; c < d; ++c)
                        ks[(size_t)kk * d + c] =
                            u < T ? bf16_to_double(k[(((size_t)b * T + u) * Hkv + g) * d + c]) : 0.0;
                }
                for (int r = r0; r < r1; ++r) {
                    if (cc > r) continue;
                    double acc = 0.0;
                    for (int kk = 0; kk < S; ++kk) {
                        const double* qa = qs + ((size_t)(r - r0) * S + kk) * d;
                        const double* kb = ks + (size_t)kk * d;
                        for (int c = 0; c < d; ++c) acc += qa[c] * kb[c];
                    }
                    acc *= scale;
                    z[(size_t)(r - r0) * nr + cc] = acc;
                    if (acc > zmax) zmax = acc;
                }
            }
            /* block masses relative to exp(zmax), then their shares */
            double* row = Ph + ((size_t)bh * nrows + n) * nb;
            double tot = 0.0;
            for (int j = 0; j <= i; ++j) {
                double e = 0.0;
                for (int r = r0; r < r1; ++r)
                    for (int cc = j * R; cc < (j + 1) * R && cc <= r; ++cc)
                        e += exp(z[(size_t)(r - r0) * nr + cc] - zmax);
                row[j] = e;
                tot += e;
            }
            for (int j = 0; j <= i; ++j) row[j] /= tot;
        }
        free(qs);
        free(ks);
        free(z);
    }
    if (!bad) {
        /* mean over (b, h), summed in a fixed order */
        for (size_t e = 0; e < (size_t)nrows * nb; ++e) {
            double s = 0.0;
            for (int bh = 0; bh < nbh; ++bh) s += Ph[(size_t)bh * nrows * nb + e];
            P[e] = s / nbh;
        }
    }
    free(Ph);
    return bad ? -1 : 0;
}

/* All query blocks: P [nb][nb]. */
int oracle_block_scores(const uint16_t* q, const uint16_t* k, int B, int T, int Hq, int Hkv,
                        int d, int block, int stride, double scale, double* P) {
    if (T < 1 || stride < 1 || block < stride || block % stride) return -1;
    const int R = block / stride, nr = (T + stride - 1) / stride, nb = (nr + R - 1) / R;
    int* rows = (int*)malloc(sizeof(int) * (size_t)nb);
    if (!rows) return -1;
    for (int i = 0; i < nb; ++i) rows[i] = i;
    const int rc = oracle_block_scores_rows(q, k, B, T, Hq, Hkv, d, block, stride, scale, rows,
                                            nb, P);
    free(rows);
    return rc;
}

/*
 * Selection from the layer scores (same reading as above): per query block
 * i, the blocks j < sink_blocks (j <= i) and j = i are always kept; the other
 * j <= i are taken in order of decreasing score (ties: smaller j first) while
 * the running sum of the kept blocks' scores is below tau.  The scores and the
 * running sum are fp32, summed in exactly this order (the forced blocks by
 * ascending j, then the candidates as taken): the decision is an integer taken
 * in the kernel's precision.
 */
int oracle_select_blocks(const float* P, int nb, float tau, int sink_blocks, uint8_t* mask) {
    if (nb < 1 || sink_blocks < 0) return -1;
    int* order = (int*)malloc(sizeof(int) * (size_t)nb);
    if (!order) return -1;
    memset(mask, 0, (size_t)nb * nb);
    for (int i = 0; i < nb; ++i) {
        const float* p = P + (size_t)i * nb;
        uint8_t* m = mask + (size_t)i * nb;
        float cum = 0.0f;
        int n = 0;
        for (int j = 0; j <= i; ++j) {
            if (j < sink_blocks || j == i) {
                m[j] = 1;
                cum += p[j];
            } else {
                order[n++] = j;
            }
        }
        /* insertion sort: decreasing score, then increasing j */
        for (int a = 1; a < n; ++a) {
            const int x = order[a];
            int c = a - 1;
            while (c >= 0 && (p[order[c]] < p[x] || (p[order[c]] == p[x] && order[c] > x))) {
                order[c + 1] = order[c];
                --c;
            }
            order[c + 1] = x;
        }
        for (int a = 0; a < n && cum < tau; ++a) {
            m[order[a]] = 1;
            cum += p[order[a]];
        }
    }
    free(order);
    return 0;
}
