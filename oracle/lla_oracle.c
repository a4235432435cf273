/*
 * lla_oracle.c -- plain, slow, fp64 CPU oracle for Looped Latent Attention (LLA).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code, header,
 * table or constant with the CUDA path, and nothing here is tuned: every routine
 * is the definition written out with straight loops in double precision, one
 * problem instance per call, in the order and notation of the pages.
 *
 * Sources (page title, section):
 *  [R]  "Looped Latent Attention: Cross-Loop KV Compression for Looped
 *       Transformers", Pith review page -- "What carries the argument"
 *       (Eqs. 2-4: centred latent c = (x - mu) W_down of rank r, per-loop
 *       reconstruction x_hat_t = c W_up,t + mu_t, exact ratio
 *       rho = 2 T d_head / (r_k + r_v)), Figure 1 (one (K_t, V_t) pair per loop in
 *       a loop-indexed cache), Figure 10 (cache memory divided exactly by rho).
 *  [V]  Same paper, Pith verdict record -- desk-editor letter (the
 *       "absorbed-attention variant") and key_machinery.
 *  [A]  Same paper, arXiv abstract -- LLA-2D folds the heads into one latent;
 *       K/V are reconstructed "only when attention reads them".
 *  [HLA] "Hybrid Latent Attention for Looped Language Models", abstract -- exact
 *       keys and values for a sliding window of W recent tokens, latents for the
 *       older tokens, read by every loop's query.
 *  [S]  Same LLA paper, Pith verdict record -- the skeptic's concrete test: the
 *       per-token reconstruction residual ||x - (x - mu) W_down W_up^T - mu|| / ||x||
 *       on held-out tokens.
 *  [D]  Same LLA paper, Pith verdict record -- desk-editor letter: the absorbed-attention
 *       variant needs decoupled RoPE (a rotary sub-key kept exact beside the latent,
 *       as in multi-head latent attention), which the paper measures with a fidelity
 *       floor.
 *  [P]  Same LLA paper, Pith verdict record -- key_machinery (the codec leaves the
 *       attention computation and RoPE unchanged) and the domain assumptions (the
 *       codec is fitted on pre-RoPE K; a token has the same position at every loop,
 *       so RoPE can be applied after reconstruction); rotary embedding as defined by
 *       RoFormer (arXiv:2104.09864), which the paper cites: a pair of components is
 *       rotated by pos * base^(-2i/d).
 *
 * Conventions (all arrays row-major, caller-owned, doubles):
 *  - one stacked vector per token x in R^W with W = T*d (per-head) or W = T*H*d
 *    (LLA-2D); loop t of a per-head vector occupies x[t*d .. t*d+d-1].
 *  - W_down is W x r; the loop-t up-projection W_up,t is r x d (head slice
 *    already extracted by the caller for LLA-2D); mu_t is the loop-t slice of mu.
 *  - Attention is ordinary softmax attention of one query q (length d) over n
 *    cached tokens, logits l_n = scale * q . k_hat_n, with the maximum
 *    subtracted before exponentiation.  n = 0 gives o = 0 and lse = -inf.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

/* ---------------------------------------------------------------------------
 * Eq. 4 and Figure 10 of [R]: exact cache accounting.
 * Uncompressed cache: every loop t stores K_t and V_t of d_head values per
 * head, so 2*T*H*d values per (token, layer).  Latent cache: one c_K (r_k) and
 * one c_V (r_v) per (token, layer, head) -- or per (token, layer) when the
 * heads are folded (LLA-2D, [A]).  rho is returned as a reduced fraction.
 * ------------------------------------------------------------------------- */
static uint64_t gcd_u64(uint64_t a, uint64_t b)
{
    while (b != 0) {
        uint64_t t = a % b;
        a = b;
        b = t;
    }
    return a;
}

int oracle_cache_bytes(int T, int L, int H, int d, int r_k, int r_v, int fold2d,
                       int elem_bytes, int64_t n_tokens,
                       uint64_t *latent_bytes, uint64_t *uncompressed_bytes,
                       uint64_t *rho_num, uint64_t *rho_den)
{
    if (T <= 0 || L <= 0 || H <= 0 || d <= 0 || r_k <= 0 || r_v <= 0 ||
        elem_bytes <= 0 || n_tokens < 0)
        return -1;
    uint64_t heads_stored = fold2d ? 1u : (uint64_t)H;
    uint64_t per_token_uncompressed = 2ull * (uint64_t)T * (uint64_t)H * (uint64_t)d;
    uint64_t per_token_latent = heads_stored * (uint64_t)(r_k + r_v);
    *uncompressed_bytes = (uint64_t)n_tokens * (uint64_t)L * per_token_uncompressed *
                          (uint64_t)elem_bytes;
    *latent_bytes = (uint64_t)n_tokens * (uint64_t)L * per_token_latent * (uint64_t)elem_bytes;
    uint64_t g = gcd_u64(per_token_uncompressed, per_token_latent);
    *rho_num = per_token_uncompressed / g;
    *rho_den = per_token_latent / g;
    return 0;
}

/* ---------------------------------------------------------------------------
 * Eq. 2 of [R] (write path): c = (x - mu) W_down, for n tokens.
 *   x [n][W], mu [W], W_down [W][r]  ->  c [n][r]
 * ------------------------------------------------------------------------- */
void oracle_encode(int64_t n, int W, int r, const double *x, const double *mu,
                   const double *W_down, double *c)
{
    for (int64_t i = 0; i < n; ++i) {
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int k = 0; k < W; ++k)
                acc += (x[i * W + k] - mu[k]) * W_down[(int64_t)k * r + j];
            c[i * r + j] = acc;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Eq. 3 of [R] (read path): x_hat_t = c W_up,t + mu_t, for n latents.
 *   c [n][r], W_up_t [r][d], mu_t [d]  ->  x_hat [n][d]
 * ------------------------------------------------------------------------- */
void oracle_reconstruct(int64_t n, int r, int d, const double *c, const double *W_up_t,
                        const double *mu_t, double *x_hat)
{
    for (int64_t i = 0; i < n; ++i) {
        for (int k = 0; k < d; ++k) {
            double acc = mu_t[k];
            for (int j = 0; j < r; ++j)
                acc += c[i * r + j] * W_up_t[(int64_t)j * d + k];
            x_hat[i * d + k] = acc;
        }
    }
}

/* Softmax-weighted sum of rows: given logits l[n], returns p_n = exp(l_n - m)/Z
 * in p (length n) and log Z + m in *lse.  Plain max-subtracted softmax. */
static void softmax_rows(int64_t n, const double *l, double *p, double *lse)
{
    double m = -INFINITY;
    for (int64_t i = 0; i < n; ++i)
        if (l[i] > m)
            m = l[i];
    double Z = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        p[i] = exp(l[i] - m);
        Z += p[i];
    }
    for (int64_t i = 0; i < n; ++i)
        p[i] /= Z;
    *lse = m + log(Z);
}

/* ---------------------------------------------------------------------------
 * Decode attention, reconstruct-on-read form ([R] Eq. 3 + Figure 1; [A]):
 * the loop-t query attends over the n cached tokens whose loop-t keys and
 * values are rebuilt from their latents:
 *   k_hat_n = c_K[n] W_up,t^K + mu_t^K,   v_hat_n = c_V[n] W_up,t^V + mu_t^V,
 *   l_n = scale * q . k_hat_n,  p = softmax(l),  o = sum_n p_n v_hat_n,
 *   lse = log sum_n exp(l_n).
 * Returns 0, or -1 if scratch memory could not be allocated.
 * ------------------------------------------------------------------------- */
int oracle_attend_reconstruct(int64_t n, int r_k, int r_v, int d,
                              const double *c_K, const double *c_V,
                              const double *W_up_K_t, const double *mu_K_t,
                              const double *W_up_V_t, const double *mu_V_t,
                              const double *q, double scale, double *o, double *lse)
{
    for (int k = 0; k < d; ++k)
        o[k] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return 0;
    }
    double *k_hat = malloc(sizeof(double) * (size_t)d);
    double *v_hat = malloc(sizeof(double) * (size_t)d);
    double *l = malloc(sizeof(double) * (size_t)n);
    double *p = malloc(sizeof(double) * (size_t)n);
    if (!k_hat || !v_hat || !l || !p) {
        free(k_hat); free(v_hat); free(l); free(p);
        return -1;
    }
    for (int64_t i = 0; i < n; ++i) {
        oracle_reconstruct(1, r_k, d, c_K + i * r_k, W_up_K_t, mu_K_t, k_hat);
        double dot = 0.0;
        for (int k = 0; k < d; ++k)
            dot += q[k] * k_hat[k];
        l[i] = scale * dot;
    }
    softmax_rows(n, l, p, lse);
    for (int64_t i = 0; i < n; ++i) {
        oracle_reconstruct(1, r_v, d, c_V + i * r_v, W_up_V_t, mu_V_t, v_hat);
        for (int k = 0; k < d; ++k)
            o[k] += p[i] * v_hat[k];
    }
    free(k_hat); free(v_hat); free(l); free(p);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Decode attention, query-side absorption ([V] desk-editor letter: the
 * "absorbed-attention variant"; same result as the reconstruct form when no
 * rotation sits between reconstruction and the dot product).  Substituting
 * Eq. 3 into the logits and the output:
 *   q_tilde = scale * q W_up,t^K^T               (r_k values)
 *   l_n     = q_tilde . c_K[n] + scale * q . mu_t^K
 *   o       = (sum_n p_n c_V[n]) W_up,t^V + mu_t^V     (sum_n p_n = 1)
 * Written separately from the reconstruct form on purpose.
 * ------------------------------------------------------------------------- */
int oracle_attend_absorb(int64_t n, int r_k, int r_v, int d,
                         const double *c_K, const double *c_V,
                         const double *W_up_K_t, const double *mu_K_t,
                         const double *W_up_V_t, const double *mu_V_t,
                         const double *q, double scale, double *o, double *lse)
{
    for (int k = 0; k < d; ++k)
        o[k] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return 0;
    }
    double *q_tilde = malloc(sizeof(double) * (size_t)r_k);
    double *o_lat = malloc(sizeof(double) * (size_t)r_v);
    double *l = malloc(sizeof(double) * (size_t)n);
    double *p = malloc(sizeof(double) * (size_t)n);
    if (!q_tilde || !o_lat || !l || !p) {
        free(q_tilde); free(o_lat); free(l); free(p);
        return -1;
    }
    for (int j = 0; j < r_k; ++j) {
        double acc = 0.0;
        for (int k = 0; k < d; ++k)
            acc += q[k] * W_up_K_t[(int64_t)j * d + k];
        q_tilde[j] = scale * acc;
    }
    double q_mu = 0.0;
    for (int k = 0; k < d; ++k)
        q_mu += q[k] * mu_K_t[k];
    q_mu *= scale;
    for (int64_t i = 0; i < n; ++i) {
        double dot = 0.0;
        for (int j = 0; j < r_k; ++j)
            dot += q_tilde[j] * c_K[i * r_k + j];
        l[i] = dot + q_mu;
    }
    softmax_rows(n, l, p, lse);
    for (int j = 0; j < r_v; ++j)
        o_lat[j] = 0.0;
    for (int64_t i = 0; i < n; ++i)
        for (int j = 0; j < r_v; ++j)
            o_lat[j] += p[i] * c_V[i * r_v + j];
    for (int k = 0; k < d; ++k) {
        double acc = mu_V_t[k];
        for (int j = 0; j < r_v; ++j)
            acc += o_lat[j] * W_up_V_t[(int64_t)j * d + k];
        o[k] = acc;
    }
    free(q_tilde); free(o_lat); free(l); free(p);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Hybrid decode attention ([HLA] abstract): the sequence's w most recent tokens
 * keep their exact loop-t keys and values (the sliding window), its n older
 * tokens are latents.  The loop-t query attends over all n + w tokens at once:
 *   older token i:   k_i = c_K[i] W_up,t^K + mu_t^K,   v_i = c_V[i] W_up,t^V + mu_t^V
 *   window token m:  k = k_win[m],                    v = v_win[m]
 *   l = scale * q . k over the n + w tokens, p = softmax(l), o = sum p v,
 *   lse = log sum exp(l).
 *   k_win, v_win [w][d].  n + w = 0 gives o = 0 and lse = -inf.
 * Returns 0, or -1 if scratch memory could not be allocated.
 * ------------------------------------------------------------------------- */
int oracle_attend_hybrid(int64_t n, int64_t w, int r_k, int r_v, int d,
                         const double *c_K, const double *c_V,
                         const double *W_up_K_t, const double *mu_K_t,
                         const double *W_up_V_t, const double *mu_V_t,
                         const double *k_win, const double *v_win,
                         const double *q, double scale, double *o, double *lse)
{
    const int64_t total = n + w;
    for (int k = 0; k < d; ++k)
        o[k] = 0.0;
    if (total == 0) {
        *lse = -INFINITY;
        return 0;
    }
    double *k_hat = malloc(sizeof(double) * (size_t)d);
    double *v_hat = malloc(sizeof(double) * (size_t)d);
    double *l = malloc(sizeof(double) * (size_t)total);
    double *p = malloc(sizeof(double) * (size_t)total);
    if (!k_hat || !v_hat || !l || !p) {
        free(k_hat); free(v_hat); free(l); free(p);
        return -1;
    }
    for (int64_t i = 0; i < n; ++i) { /* older tokens: rebuilt loop-t keys */
        oracle_reconstruct(1, r_k, d, c_K + i * r_k, W_up_K_t, mu_K_t, k_hat);
        double dotc = 0.0;
        for (int k = 0; k < d; ++k)
            dotc += q[k] * k_hat[k];
        l[i] = scale * dotc;
    }
    for (int64_t m = 0; m < w; ++m) { /* window tokens: exact loop-t keys */
        double dotw = 0.0;
        for (int k = 0; k < d; ++k)
            dotw += q[k] * k_win[m * d + k];
        l[n + m] = scale * dotw;
    }
    softmax_rows(total, l, p, lse);
    for (int64_t i = 0; i < n; ++i) {
        oracle_reconstruct(1, r_v, d, c_V + i * r_v, W_up_V_t, mu_V_t, v_hat);
        for (int k = 0; k < d; ++k)
            o[k] += v_hat[k] * p[i];
    }
    for (int64_t m = 0; m < w; ++m)
        for (int k = 0; k < d; ++k)
            o[k] += p[n + m] * v_win[m * d + k];
    free(k_hat); free(v_hat); free(l); free(p);
    return 0;
}

/* ---------------------------------------------------------------------------
 * [P]: the faithful read with rotary position embedding.  Keys are rebuilt
 * (Eq. 3) as pre-RoPE vectors, then both the query and every rebuilt key are
 * rotated at their own positions, and attention proceeds as usual; values are
 * not rotated.  Component pairs: style 0 pairs i with i + d/2 (the half-split
 * layout), style 1 pairs 2i with 2i+1 (RoFormer's layout); pair i turns by the
 * angle pos * base^(-2i/d), counter-clockwise:
 *   (a, b) -> (a cos - b sin, a sin + b cos).
 * The cached token i of the sequence sits at position k_pos0 + i.
 * ------------------------------------------------------------------------- */
static void rope_rotate(int d, int style, double base, double pos, double *x)
{
    for (int i = 0; i < d / 2; ++i) {
        const double angle = pos * pow(base, -2.0 * i / d);
        const double cs = cos(angle), sn = sin(angle);
        const int ia = style == 0 ? i : 2 * i;
        const int ib = style == 0 ? i + d / 2 : 2 * i + 1;
        const double xa = x[ia], xb = x[ib];
        x[ia] = xa * cs - xb * sn;
        x[ib] = xa * sn + xb * cs;
    }
}

int oracle_attend_rope(int64_t n, int r_k, int r_v, int d,
                       const double *c_K, const double *c_V,
                       const double *W_up_K_t, const double *mu_K_t,
                       const double *W_up_V_t, const double *mu_V_t,
                       const double *q, double scale, int style, double base,
                       double q_pos, double k_pos0, double *o, double *lse)
{
    for (int k = 0; k < d; ++k)
        o[k] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return 0;
    }
    double *q_rot = malloc(sizeof(double) * (size_t)d);
    double *k_rot = malloc(sizeof(double) * (size_t)d);
    double *v_hat = malloc(sizeof(double) * (size_t)d);
    double *l = malloc(sizeof(double) * (size_t)n);
    double *p = malloc(sizeof(double) * (size_t)n);
    if (!q_rot || !k_rot || !v_hat || !l || !p) {
        free(q_rot); free(k_rot); free(v_hat); free(l); free(p);
        return -1;
    }
    for (int k = 0; k < d; ++k)
        q_rot[k] = q[k];
    rope_rotate(d, style, base, q_pos, q_rot);
    for (int64_t i = 0; i < n; ++i) {
        oracle_reconstruct(1, r_k, d, c_K + i * r_k, W_up_K_t, mu_K_t, k_rot);
        rope_rotate(d, style, base, k_pos0 + (double)i, k_rot);
        double dotr = 0.0;
        for (int k = 0; k < d; ++k)
            dotr += q_rot[k] * k_rot[k];
        l[i] = scale * dotr;
    }
    softmax_rows(n, l, p, lse);
    for (int64_t i = 0; i < n; ++i) {
        oracle_reconstruct(1, r_v, d, c_V + i * r_v, W_up_V_t, mu_V_t, v_hat);
        for (int k = 0; k < d; ++k)
            o[k] += p[i] * v_hat[k];
    }
    free(q_rot); free(k_rot); free(v_hat); free(l); free(p);
    return 0;
}

/* ---------------------------------------------------------------------------
 * [S]: per-token reconstruction residual of a codec.  For each of the n stacked
 * vectors x (width W = T * Dp, loop t occupying x[t*Dp .. t*Dp+Dp-1]):
 *   c = (x - mu) W_down                     (Eq. 2)
 *   x_hat_t = c W_up,t + mu_t for every t   (Eq. 3)
 *   err = ||x - x_hat||,  norm = ||x||      (Euclidean, over all W components).
 * W_up holds the T per-loop up-projections, [T][r][Dp].  The caller divides.
 * ------------------------------------------------------------------------- */
int oracle_codec_residual(int64_t n, int T, int Dp, int r, const double *x, const double *mu,
                          const double *W_down, const double *W_up, double *err, double *norm)
{
    const int W = T * Dp;
    double *c = malloc(sizeof(double) * (size_t)r);
    double *x_hat = malloc(sizeof(double) * (size_t)Dp);
    if (!c || !x_hat) {
        free(c); free(x_hat);
        return -1;
    }
    for (int64_t i = 0; i < n; ++i) {
        const double *xi = x + i * W;
        oracle_encode(1, W, r, xi, mu, W_down, c);
        double e2 = 0.0, n2 = 0.0;
        for (int t = 0; t < T; ++t) {
            oracle_reconstruct(1, r, Dp, c, W_up + (int64_t)t * r * Dp, mu + (int64_t)t * Dp, x_hat);
            for (int k = 0; k < Dp; ++k) {
                const double diff = xi[t * Dp + k] - x_hat[k];
                e2 += diff * diff;
                n2 += xi[t * Dp + k] * xi[t * Dp + k];
            }
        }
        err[i] = sqrt(e2);
        norm[i] = sqrt(n2);
    }
    free(c); free(x_hat);
    return 0;
}

/* ---------------------------------------------------------------------------
 * [D]: decoupled rotary sub-key.  Beside its latent, cached token i keeps an exact
 * sub-key k_rope[i] (d_r values), stored already rotated at the token's position;
 * the query brings a rotary part q_rope (d_r values), rotated here at q_pos.  The
 * loop-t score adds the two dot products:
 *   l_i = scale * (q . k_hat_i + rope(q_rope, q_pos) . k_rope[i]),
 * with k_hat_i rebuilt by Eq. 3; values are rebuilt as usual and not rotated.
 * ------------------------------------------------------------------------- */
int oracle_attend_decoupled(int64_t n, int r_k, int r_v, int d, int d_r,
                            const double *c_K, const double *c_V,
                            const double *W_up_K_t, const double *mu_K_t,
                            const double *W_up_V_t, const double *mu_V_t,
                            const double *k_rope, const double *q, const double *q_rope,
                            double scale, int style, double base, double q_pos,
                            double *o, double *lse)
{
    for (int k = 0; k < d; ++k)
        o[k] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return 0;
    }
    double *qr = malloc(sizeof(double) * (size_t)(d_r > 0 ? d_r : 1));
    double *k_hat = malloc(sizeof(double) * (size_t)d);
    double *v_hat = malloc(sizeof(double) * (size_t)d);
    double *l = malloc(sizeof(double) * (size_t)n);
    double *p = malloc(sizeof(double) * (size_t)n);
    if (!qr || !k_hat || !v_hat || !l || !p) {
        free(qr); free(k_hat); free(v_hat); free(l); free(p);
        return -1;
    }
    for (int k = 0; k < d_r; ++k)
        qr[k] = q_rope[k];
    rope_rotate(d_r, style, base, q_pos, qr);
    for (int64_t i = 0; i < n; ++i) {
        oracle_reconstruct(1, r_k, d, c_K + i * r_k, W_up_K_t, mu_K_t, k_hat);
        double dn = 0.0, dr = 0.0;
        for (int k = 0; k < d; ++k)
            dn += q[k] * k_hat[k];
        for (int k = 0; k < d_r; ++k)
            dr += qr[k] * k_rope[i * d_r + k];
        l[i] = scale * (dn + dr);
    }
    softmax_rows(n, l, p, lse);
    for (int64_t i = 0; i < n; ++i) {
        oracle_reconstruct(1, r_v, d, c_V + i * r_v, W_up_V_t, mu_V_t, v_hat);
        for (int k = 0; k < d; ++k)
            o[k] += p[i] * v_hat[k];
    }
    free(qr); free(k_hat); free(v_hat); free(l); free(p);
    return 0;
}
