/*
 * rope3d_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, fp64 CPU statement of the per-chunk Q/K preparation step of a
 * causal autoregressive video DiT with Causal-RoPE SP ("Accelerating Video
 * Generation Inference with Sequential-Parallel 3D Positional Encoding Using a
 * Global Time Index", Yuan & Li): position decode from the global token index,
 * QK-RMSNorm, 3D rotary embedding by complex multiplication, and the K/V cache
 * append.  Only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg may load this library.  It shares no code, header, table or constant with
 * the CUDA path; each side is written from the definitions on its own.
 *
 * Everything here is computed in double precision with libm cos/sin/pow/sqrt,
 * one token at a time, in the order the definitions give.  The only concession to
 * speed is an OpenMP loop over independent token rows in the whole-step entry
 * point; every row is computed by the same sequential code either way.
 *
 * Readings of points the paper leaves open (each is also listed in the design
 * notes of the repository):
 *   - per-axis frequency schedule: each of the t, h, w axes is an ordinary
 *     rotary embedding over its own sub-dimension d_a = 2 n_a, so pair j of axis
 *     a turns at theta^(-2j/d_a) per unit of position (schedule 0).  Schedule 1
 *     instead takes one head-wide schedule theta^(-2j/D) for pair j = 0..D/2-1 and
 *     hands the first n_t pairs to t, the next n_h to h and the last n_w to w.
 *     The paper names the three per-axis frequency sets but prints no formula, so
 *     which schedule is meant is parity unpinned: both are computed here, and each
 *     is pinned by its own closed forms.
 *   - h and w decode: the paper gives only the time index; h and w follow from
 *     the row-major (F, H, W) expansion of the frequency tables in its
 *     Algorithm 2, so h = floor(i / W) mod H and w = i mod W.
 *   - QK-RMSNorm is not on the paper's pages: it normalises one token's q (and,
 *     separately, its k) over the token's whole N*D feature vector,
 *     y = x / sqrt(mean(x^2) + eps) * weight, and runs before the rotation.
 *     V is neither normalised nor rotated.
 *   - cache placement: cache row = (slot + i) mod cache_tokens, token-major
 *     [B][cache_tokens][N][D]; rotated K is stored with its global position.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)

/*
 * Frequency schedule ("RoPE frequencies theta" of Algorithms 1-3; the three
 * per-axis frequency sets freqs[0], freqs[1], freqs[2] of Algorithm 2).
 * Writes inv[0 .. n_t+n_h+n_w-1]: the angle per unit position of every complex
 * pair of a head, t pairs first, then h, then w (the concatenation order of
 * Algorithm 2).
 */
int rope3d_oracle_inv_freq(int n_t, int n_h, int n_w, double theta, int schedule,
                           double* inv)
{
    if (n_t < 0 || n_h < 0 || n_w < 0 || !(theta > 1.0) || inv == NULL) return ORACLE_EINVAL;
    if (schedule != 0 && schedule != 1) return ORACLE_EINVAL;
    int n_axis[3] = {n_t, n_h, n_w};
    int pairs = n_t + n_h + n_w;
    int first = 0; /* index of the axis' first pair within the head */
    for (int a = 0; a < 3; ++a) {
        for (int j = 0; j < n_axis[a]; ++j) {
            double exponent;
            if (schedule == 0) {
                /* the axis' own sub-dimension: d_a = 2 n_a real elements */
                double d_a = 2.0 * n_axis[a];
                exponent = (2.0 * j) / d_a;
            } else {
                /* one head-wide schedule over D = 2 * pairs real elements */
                double d = 2.0 * pairs;
                exponent = (2.0 * (first + j)) / d;
            }
            inv[first + j] = 1.0 / pow(theta, exponent);
        }
        first += n_axis[a];
    }
    return ORACLE_OK;
}

/*
 * Position decode of Section 3.3.3: a token with global sequence index i of a
 * chunk with grid (F, H, W) = (T, H, W) and start frame s sits at local frame
 * t = floor(i / (H W)), global frame t_g = s + t (Section 3.3.2, item 1); its
 * row h and column w follow the row-major expansion of Algorithm 2.
 */
void rope3d_oracle_decode(int64_t i, int64_t s, int64_t T, int64_t H, int64_t W,
                          int64_t* t_g, int64_t* h, int64_t* w)
{
    (void)T;
    int64_t hw = H * W;
    *t_g = s + i / hw;
    *h = (i / W) % H;
    *w = i % W;
}

/* Rolling KV-cache row of global token index i (cache of cache_tokens rows). */
int64_t rope3d_oracle_cache_row(int64_t i, int64_t slot, int64_t cache_tokens)
{
    return (slot + i) % cache_tokens;
}

/* Angle of every pair of a head at position (t_g, h, w): Section 3.3.2, item 2,
 * phi = t_g theta_T + h theta_H + w theta_W, each axis on its own pairs. */
void rope3d_oracle_angles(int64_t t_g, int64_t h, int64_t w, int n_t, int n_h, int n_w,
                          const double* inv, double* phi)
{
    for (int j = 0; j < n_t; ++j) phi[j] = (double)t_g * inv[j];
    for (int j = 0; j < n_h; ++j) phi[n_t + j] = (double)h * inv[n_t + j];
    for (int j = 0; j < n_w; ++j) phi[n_t + n_h + j] = (double)w * inv[n_t + n_h + j];
}

/*
 * RoPE(x, phi) = x * e^{i phi} (Section 3.3.1) on one token row of n heads of D
 * reals each.  Elements (2j, 2j+1) of a head are the real and imaginary part of
 * complex pair j (Algorithm 2 views the last dimension as (-1, 2) pairs).
 * The same angles apply to every head.  x and y may be the same array.
 */
void rope3d_oracle_rotate(const double* x, int64_t n_heads, int64_t head_dim,
                          const double* phi, double* y)
{
    int64_t pairs = head_dim / 2;
    for (int64_t n = 0; n < n_heads; ++n) {
        for (int64_t j = 0; j < pairs; ++j) {
            double a = x[n * head_dim + 2 * j];     /* real part */
            double b = x[n * head_dim + 2 * j + 1]; /* imaginary part */
            double c = cos(phi[j]);
            double s = sin(phi[j]);
            /* (a + i b)(c + i s) = (a c - b s) + i (a s + b c) */
            y[n * head_dim + 2 * j] = a * c - b * s;
            y[n * head_dim + 2 * j + 1] = a * s + b * c;
        }
    }
}

/* RMSNorm over one token's whole feature vector of length dim:
 * y = x / sqrt(mean(x^2) + eps) * weight.  x and y may be the same array. */
void rope3d_oracle_rms_norm(const double* x, const double* weight, int64_t dim, double eps,
                            double* y)
{
    double sum_sq = 0.0;
    for (int64_t e = 0; e < dim; ++e) sum_sq += x[e] * x[e];
    double mean_sq = sum_sq / (double)dim;
    double inv_rms = 1.0 / sqrt(mean_sq + eps);
    for (int64_t e = 0; e < dim; ++e) y[e] = x[e] * inv_rms * weight[e];
}

/* Rotate one token row at the position that global index i decodes to. */
void rope3d_oracle_rotate_at(const double* x, int64_t n_heads, int64_t head_dim,
                             int64_t i, int64_t s, int64_t T, int64_t H, int64_t W,
                             int n_t, int n_h, int n_w, const double* inv, double* y)
{
    double phi[512];
    int64_t t_g, h, w;
    rope3d_oracle_decode(i, s, T, H, W, &t_g, &h, &w);
    rope3d_oracle_angles(t_g, h, w, n_t, n_h, n_w, inv, phi);
    rope3d_oracle_rotate(x, n_heads, head_dim, phi, y);
}

static int check_common(int64_t N, int64_t D, int n_t, int n_h, int n_w,
                        int64_t token_begin, int64_t token_end, int64_t frame_offset,
                        int64_t T, int64_t H, int64_t W)
{
    if (N <= 0 || D <= 0 || D % 2 != 0 || D / 2 > 512) return ORACLE_EINVAL;
    if (n_t < 0 || n_h < 0 || n_w < 0 || (int64_t)(n_t + n_h + n_w) * 2 != D) return ORACLE_EINVAL;
    if (T <= 0 || H <= 0 || W <= 0 || frame_offset < 0) return ORACLE_EINVAL;
    if (token_begin < 0 || token_end <= token_begin || token_end > T * H * W) return ORACLE_EINVAL;
    return ORACLE_OK;
}

/*
 * One token row of the fused step for one batch sample.  Inputs are that row's
 * q, k, v (N*D reals each, heads outermost); outputs are the row of q_out and
 * the rows that go to the K and V caches, plus the decoded position
 * (t_g, h, w) and the cache row in pos_out[0..3].
 *   q_out = RoPE(RMSNorm(q; q_norm_w)),  k_row = RoPE(RMSNorm(k; k_norm_w)),
 *   v_row = v  (Algorithm 1/3 step 5: KVCache[key] <- rotated k, KVCache[value] <- v)
 */
int rope3d_oracle_token(const double* q, const double* k, const double* v,
                        int64_t N, int64_t D, int64_t i, int64_t frame_offset,
                        int64_t T, int64_t H, int64_t W,
                        const double* q_norm_w, const double* k_norm_w, double eps,
                        int64_t slot, int64_t cache_tokens,
                        int n_t, int n_h, int n_w, const double* inv,
                        double* q_out, double* k_row, double* v_row, int64_t* pos_out)
{
    int rc = check_common(N, D, n_t, n_h, n_w, i, i + 1, frame_offset, T, H, W);
    if (rc != ORACLE_OK) return rc;
    if (cache_tokens <= 0 || slot < 0) return ORACLE_EINVAL;
    int64_t dim = N * D;
    int64_t t_g, h, w;
    double phi[512];
    rope3d_oracle_decode(i, frame_offset, T, H, W, &t_g, &h, &w);
    rope3d_oracle_angles(t_g, h, w, n_t, n_h, n_w, inv, phi);

    rope3d_oracle_rms_norm(q, q_norm_w, dim, eps, q_out);
    rope3d_oracle_rotate(q_out, N, D, phi, q_out);
    rope3d_oracle_rms_norm(k, k_norm_w, dim, eps, k_row);
    rope3d_oracle_rotate(k_row, N, D, phi, k_row);
    memcpy(v_row, v, (size_t)dim * sizeof(double));

    if (pos_out != NULL) {
        pos_out[0] = t_g;
        pos_out[1] = h;
        pos_out[2] = w;
        pos_out[3] = rope3d_oracle_cache_row(i, slot, cache_tokens);
    }
    return ORACLE_OK;
}

/*
 * The whole step over the token range [token_begin, token_end) of a chunk
 * (Algorithm 3 steps 2, 3 and 5 for one rank whose slice starts at
 * Delta = token_begin): q, k, v and q_out are [B][n_tok][N][D] with
 * n_tok = token_end - token_begin, row r holding global index token_begin + r;
 * k_cache and v_cache are [B][cache_tokens][N][D] and only the rows this range
 * maps to are written.  nthreads <= 0 uses the OpenMP default.
 */
int rope3d_oracle_qk_norm_rope_append(
    const double* q, const double* k, const double* v, double* q_out,
    int64_t B, int64_t N, int64_t D,
    int64_t token_begin, int64_t token_end, int64_t frame_offset,
    int64_t T, int64_t H, int64_t W,
    const double* q_norm_w, const double* k_norm_w, double eps,
    double* k_cache, double* v_cache, int64_t cache_tokens, int64_t slot,
    int n_t, int n_h, int n_w, double theta, int schedule, int nthreads)
{
    int rc = check_common(N, D, n_t, n_h, n_w, token_begin, token_end, frame_offset, T, H, W);
    if (rc != ORACLE_OK) return rc;
    if (B <= 0 || cache_tokens <= 0 || slot < 0) return ORACLE_EINVAL;
    if (token_end - token_begin > cache_tokens) return ORACLE_EINVAL;
    double inv[512];
    rc = rope3d_oracle_inv_freq(n_t, n_h, n_w, theta, schedule, inv);
    if (rc != ORACLE_OK) return rc;

    int64_t n_tok = token_end - token_begin;
    int64_t dim = N * D;
    int64_t rows = B * n_tok;
#ifdef _OPENMP
    int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#pragma omp parallel for schedule(static) num_threads(nt)
#endif
    for (int64_t u = 0; u < rows; ++u) {
        int64_t b = u / n_tok;
        int64_t r = u % n_tok;
        int64_t i = token_begin + r;
        int64_t row = rope3d_oracle_cache_row(i, slot, cache_tokens);
        int64_t in_off = (b * n_tok + r) * dim;
        int64_t cache_off = (b * cache_tokens + row) * dim;
        rope3d_oracle_token(q + in_off, k + in_off, v + in_off, N, D, i, frame_offset, T, H, W,
                            q_norm_w, k_norm_w, eps, slot, cache_tokens, n_t, n_h, n_w, inv,
                            q_out + in_off, k_cache + cache_off, v_cache + cache_off, NULL);
    }
#ifndef _OPENMP
    (void)nthreads;
#endif
    return ORACLE_OK;
}

/*
 * Rotation alone (Algorithm 2, CausalRoPE of Algorithm 3 step 3) over the token
 * range [token_begin, token_end): x and out are [B][n_tok][N][D].
 */
int rope3d_oracle_apply(const double* x, double* out, int64_t B, int64_t N, int64_t D,
                        int64_t token_begin, int64_t token_end, int64_t frame_offset,
                        int64_t T, int64_t H, int64_t W,
                        int n_t, int n_h, int n_w, double theta, int schedule)
{
    int rc = check_common(N, D, n_t, n_h, n_w, token_begin, token_end, frame_offset, T, H, W);
    if (rc != ORACLE_OK) return rc;
    if (B <= 0) return ORACLE_EINVAL;
    double inv[512];
    rc = rope3d_oracle_inv_freq(n_t, n_h, n_w, theta, schedule, inv);
    if (rc != ORACLE_OK) return rc;
    int64_t n_tok = token_end - token_begin;
    int64_t dim = N * D;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t r = 0; r < n_tok; ++r) {
            int64_t off = (b * n_tok + r) * dim;
            rope3d_oracle_rotate_at(x + off, N, D, token_begin + r, frame_offset, T, H, W,
                                    n_t, n_h, n_w, inv, out + off);
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ layout variants
 *
 * Section 3.3.1 of the paper contrasts two ways of writing the same rotation: Wan2.1's
 * complex multiply on adjacent pairs (Algorithm 2's view, used above) and Qwen2.5-VL's
 * cos/sin form with rotate_half, where element j of a head pairs with element
 * j + D/2.  The functions below add that second pairing and a head-major KV cache
 * ([B][N][cache_tokens][D], each head's rows contiguous).  Everything else -- decode,
 * angles, RMSNorm, cache row -- is the same as above.
 */
#define ORACLE_PAIRING_ADJACENT 0
#define ORACLE_PAIRING_HALF 1
#define ORACLE_CACHE_TOKEN_MAJOR 0
#define ORACLE_CACHE_HEAD_MAJOR 1

/* RoPE with the rotate_half pairing: pair j of a head is (x[j], x[j + D/2]) as
 * (re, im); x * e^{i phi_j} on it.  x and y may be the same array. */
void rope3d_oracle_rotate_half(const double* x, int64_t n_heads, int64_t head_dim,
                               const double* phi, double* y)
{
    int64_t pairs = head_dim / 2;
    for (int64_t n = 0; n < n_heads; ++n) {
        for (int64_t j = 0; j < pairs; ++j) {
            double a = x[n * head_dim + j];          /* real part: first half */
            double b = x[n * head_dim + pairs + j];  /* imaginary part: second half */
            double c = cos(phi[j]);
            double s = sin(phi[j]);
            y[n * head_dim + j] = a * c - b * s;
            y[n * head_dim + pairs + j] = a * s + b * c;
        }
    }
}

int rope3d_oracle_rotate_pairing(const double* x, int64_t n_heads, int64_t head_dim,
                                 const double* phi, int pairing, double* y)
{
    if (pairing == ORACLE_PAIRING_ADJACENT) {
        rope3d_oracle_rotate(x, n_heads, head_dim, phi, y);
        return ORACLE_OK;
    }
    if (pairing == ORACLE_PAIRING_HALF) {
        rope3d_oracle_rotate_half(x, n_heads, head_dim, phi, y);
        return ORACLE_OK;
    }
    return ORACLE_EINVAL;
}

/* rope3d_oracle_token with a choice of pairing. */
int rope3d_oracle_token_pairing(const double* q, const double* k, const double* v,
                                int64_t N, int64_t D, int64_t i, int64_t frame_offset,
                                int64_t T, int64_t H, int64_t W,
                                const double* q_norm_w, const double* k_norm_w, double eps,
                                int64_t slot, int64_t cache_tokens,
                                int n_t, int n_h, int n_w, const double* inv, int pairing,
                                double* q_out, double* k_row, double* v_row, int64_t* pos_out)
{
    int rc = check_common(N, D, n_t, n_h, n_w, i, i + 1, frame_offset, T, H, W);
    if (rc != ORACLE_OK) return rc;
    if (cache_tokens <= 0 || slot < 0) return ORACLE_EINVAL;
    if (pairing != ORACLE_PAIRING_ADJACENT && pairing != ORACLE_PAIRING_HALF)
        return ORACLE_EINVAL;
    int64_t dim = N * D;
    int64_t t_g, h, w;
    double phi[512];
    rope3d_oracle_decode(i, frame_offset, T, H, W, &t_g, &h, &w);
    rope3d_oracle_angles(t_g, h, w, n_t, n_h, n_w, inv, phi);

    rope3d_oracle_rms_norm(q, q_norm_w, dim, eps, q_out);
    rope3d_oracle_rotate_pairing(q_out, N, D, phi, pairing, q_out);
    rope3d_oracle_rms_norm(k, k_norm_w, dim, eps, k_row);
    rope3d_oracle_rotate_pairing(k_row, N, D, phi, pairing, k_row);
    memcpy(v_row, v, (size_t)dim * sizeof(double));

    if (pos_out != NULL) {
        pos_out[0] = t_g;
        pos_out[1] = h;
        pos_out[2] = w;
        pos_out[3] = rope3d_oracle_cache_row(i, slot, cache_tokens);
    }
    return ORACLE_OK;
}

/*
 * The whole step with a choice of pairing and of cache layout.  Token-major caches are
 * [B][cache_tokens][N][D]; head-major caches are [B][N][cache_tokens][D].  Head n of
 * the token's K and V rows goes to cache row `row` of head n.
 */
int rope3d_oracle_qk_norm_rope_append_layout(
    const double* q, const double* k, const double* v, double* q_out,
    int64_t B, int64_t N, int64_t D,
    int64_t token_begin, int64_t token_end, int64_t frame_offset,
    int64_t T, int64_t H, int64_t W,
    const double* q_norm_w, const double* k_norm_w, double eps,
    double* k_cache, double* v_cache, int64_t cache_tokens, int64_t slot,
    int n_t, int n_h, int n_w, double theta, int schedule, int pairing, int cache_layout,
    int nthreads)
{
    int rc = check_common(N, D, n_t, n_h, n_w, token_begin, token_end, frame_offset, T, H, W);
    if (rc != ORACLE_OK) return rc;
    if (B <= 0 || cache_tokens <= 0 || slot < 0) return ORACLE_EINVAL;
    if (token_end - token_begin > cache_tokens) return ORACLE_EINVAL;
    if (pairing != ORACLE_PAIRING_ADJACENT && pairing != ORACLE_PAIRING_HALF)
        return ORACLE_EINVAL;
    if (cache_layout != ORACLE_CACHE_TOKEN_MAJOR && cache_layout != ORACLE_CACHE_HEAD_MAJOR)
        return ORACLE_EINVAL;
    double inv[512];
    rc = rope3d_oracle_inv_freq(n_t, n_h, n_w, theta, schedule, inv);
    if (rc != ORACLE_OK) return rc;

    int64_t n_tok = token_end - token_begin;
    int64_t dim = N * D;
    int64_t rows = B * n_tok;
    int failed = 0;
#ifdef _OPENMP
    int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#pragma omp parallel num_threads(nt)
#endif
    {
        double* k_row = (double*)malloc((size_t)dim * sizeof(double));
        double* v_row = (double*)malloc((size_t)dim * sizeof(double));
        if (k_row == NULL || v_row == NULL) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            failed = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
            for (int64_t u = 0; u < rows; ++u) {
                int64_t b = u / n_tok;
                int64_t r = u % n_tok;
                int64_t i = token_begin + r;
                int64_t row = rope3d_oracle_cache_row(i, slot, cache_tokens);
                int64_t in_off = (b * n_tok + r) * dim;
                rope3d_oracle_token_pairing(q + in_off, k + in_off, v + in_off, N, D, i,
                                            frame_offset, T, H, W, q_norm_w, k_norm_w, eps,
                                            slot, cache_tokens, n_t, n_h, n_w, inv, pairing,
                                            q_out + in_off, k_row, v_row, NULL);
                for (int64_t n = 0; n < N; ++n) {
                    int64_t cache_off = cache_layout == ORACLE_CACHE_TOKEN_MAJOR
                                            ? ((b * cache_tokens + row) * N + n) * D
                                            : ((b * N + n) * cache_tokens + row) * D;
                    memcpy(k_cache + cache_off, k_row + n * D, (size_t)D * sizeof(double));
                    memcpy(v_cache + cache_off, v_row + n * D, (size_t)D * sizeof(double));
                }
            }
        }
        free(k_row);
        free(v_row);
    }
#ifndef _OPENMP
    (void)nthreads;
#endif
    return failed ? ORACLE_EINVAL : ORACLE_OK;
}

/* The rotation alone with a choice of pairing, over [B][n_tok][N][D]. */
int rope3d_oracle_apply_pairing(const double* x, double* out, int64_t B, int64_t N, int64_t D,
                                int64_t token_begin, int64_t token_end, int64_t frame_offset,
                                int64_t T, int64_t H, int64_t W,
                                int n_t, int n_h, int n_w, double theta, int schedule,
                                int pairing)
{
    int rc = check_common(N, D, n_t, n_h, n_w, token_begin, token_end, frame_offset, T, H, W);
    if (rc != ORACLE_OK) return rc;
    if (B <= 0) return ORACLE_EINVAL;
    if (pairing != ORACLE_PAIRING_ADJACENT && pairing != ORACLE_PAIRING_HALF)
        return ORACLE_EINVAL;
    double inv[512];
    rc = rope3d_oracle_inv_freq(n_t, n_h, n_w, theta, schedule, inv);
    if (rc != ORACLE_OK) return rc;
    int64_t n_tok = token_end - token_begin;
    int64_t dim = N * D;
    double phi[512];
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t r = 0; r < n_tok; ++r) {
            int64_t off = (b * n_tok + r) * dim;
            int64_t t_g, h, w;
            rope3d_oracle_decode(token_begin + r, frame_offset, T, H, W, &t_g, &h, &w);
            rope3d_oracle_angles(t_g, h, w, n_t, n_h, n_w, inv, phi);
            rope3d_oracle_rotate_pairing(x + off, N, D, phi, pairing, out + off);
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ FP8 KV cache
 *
 * Quantize-on-append: K and V rows go to the cache as FP8 E4M3 codes with one fp32
 * scale per (token, head).  The scale is a power of two, as in the OCP microscaling
 * formats: the smallest 2^e (e >= -126) with amax(|x|) / 2^e <= 448 over the head's D
 * values (2^-126 when the head is all zero), so the head's largest value lands in
 * (224, 448] and dividing by the scale is exact.  Codes are E4M3(x / scale) rounded to
 * nearest, ties to the even code, saturating at +-448.  A reader recovers
 * x ~ value(code) * scale.  The pages name
 * NVFP4 KV-cache quantization for Blackwell (the LongLive-2.0 abstract) but give no
 * format details; E4M3 with per-head scales is the reading taken here.  The decision
 * runs in fp32 (the precision the kernel computes the rows in): the oracle rounds its
 * fp64 K row to fp32 first; V is exact.
 *
 * E4M3 (the OCP 8-bit float "E4M3"): sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits; exponent field 0 is subnormal (m/8 * 2^-6); the all-ones exponent with all-ones
 * mantissa is NaN; there is no infinity; the largest finite value is 448.
 */
double rope3d_oracle_e4m3_value(int code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Nearest E4M3 code of x (finite), ties to the even code, saturating at +-448; found by
 * scanning the 127 non-negative finite codes in increasing order. */
int rope3d_oracle_e4m3_encode(float x)
{
    int sign = signbit(x) ? 0x80 : 0;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    int best = 0;
    for (int c = 0; c < 0x7E; ++c) {
        double lo = rope3d_oracle_e4m3_value(c);
        double hi = rope3d_oracle_e4m3_value(c + 1);
        if (a >= lo && a <= hi) {
            double dlo = a - lo, dhi = hi - a;
            if (dlo < dhi) best = c;
            else if (dhi < dlo) best = c + 1;
            else best = (c % 2 == 0) ? c : c + 1;  /* tie: even mantissa */
            break;
        }
    }
    return sign | best;
}

/* Exponent of the power-of-two scale of a head whose largest magnitude is amax >= 0:
 * the smallest e >= -126 with amax <= 448 * 2^e, found by stepping e (-126 for an
 * all-zero head, whose codes are zero under any scale). */
int rope3d_oracle_e4m3_scale_exponent(float amax)
{
    int e = -126;
    while ((double)amax > ldexp(448.0, e)) ++e;
    return e;
}

/* One head of n fp32 values -> codes and its scale. */
void rope3d_oracle_quantize_head_e4m3(const float* x, int64_t n, unsigned char* codes,
                                      float* scale)
{
    float amax = 0.0f;
    for (int64_t e = 0; e < n; ++e) {
        float a = fabsf(x[e]);
        if (a > amax) amax = a;
    }
    int ex = rope3d_oracle_e4m3_scale_exponent(amax);
    for (int64_t e = 0; e < n; ++e)
        codes[e] = (unsigned char)rope3d_oracle_e4m3_encode(ldexpf(x[e], -ex));  /* exact */
    *scale = ldexpf(1.0f, ex);
}

/*
 * The whole step with an FP8 E4M3 cache.  q_out is returned in fp64 as above; the
 * caches are codes [B][cache_tokens][N][D] (token-major) or [B][N][cache_tokens][D]
 * (head-major) and the scales [B][cache_tokens][N] or [B][N][cache_tokens].
 */
int rope3d_oracle_qk_norm_rope_append_fp8(
    const double* q, const double* k, const double* v, double* q_out,
    int64_t B, int64_t N, int64_t D,
    int64_t token_begin, int64_t token_end, int64_t frame_offset,
    int64_t T, int64_t H, int64_t W,
    const double* q_norm_w, const double* k_norm_w, double eps,
    unsigned char* k_codes, unsigned char* v_codes, float* k_scale, float* v_scale,
    int64_t cache_tokens, int64_t slot,
    int n_t, int n_h, int n_w, double theta, int schedule, int pairing, int cache_layout)
{
    int rc = check_common(N, D, n_t, n_h, n_w, token_begin, token_end, frame_offset, T, H, W);
    if (rc != ORACLE_OK) return rc;
    if (B <= 0 || cache_tokens <= 0 || slot < 0) return ORACLE_EINVAL;
    if (token_end - token_begin > cache_tokens) return ORACLE_EINVAL;
    if (cache_layout != ORACLE_CACHE_TOKEN_MAJOR && cache_layout != ORACLE_CACHE_HEAD_MAJOR)
        return ORACLE_EINVAL;
    double inv[512];
    rc = rope3d_oracle_inv_freq(n_t, n_h, n_w, theta, schedule, inv);
    if (rc != ORACLE_OK) return rc;
    int64_t n_tok = token_end - token_begin;
    int64_t dim = N * D;
    double* k_row = (double*)malloc((size_t)dim * sizeof(double));
    double* v_row = (double*)malloc((size_t)dim * sizeof(double));
    float* head = (float*)malloc((size_t)D * sizeof(float));
    if (k_row == NULL || v_row == NULL || head == NULL) {
        free(k_row); free(v_row); free(head);
        return ORACLE_EINVAL;
    }
    for (int64_t b = 0; b < B && rc == ORACLE_OK; ++b) {
        for (int64_t r = 0; r < n_tok; ++r) {
            int64_t i = token_begin + r;
            int64_t row = rope3d_oracle_cache_row(i, slot, cache_tokens);
            int64_t in_off = (b * n_tok + r) * dim;
            rc = rope3d_oracle_token_pairing(q + in_off, k + in_off, v + in_off, N, D, i,
                                             frame_offset, T, H, W, q_norm_w, k_norm_w, eps,
                                             slot, cache_tokens, n_t, n_h, n_w, inv, pairing,
                                             q_out + in_off, k_row, v_row, NULL);
            if (rc != ORACLE_OK) break;
            for (int64_t n = 0; n < N; ++n) {
                int64_t code_off = cache_layout == ORACLE_CACHE_TOKEN_MAJOR
                                       ? ((b * cache_tokens + row) * N + n) * D
                                       : ((b * N + n) * cache_tokens + row) * D;
                int64_t scale_off = cache_layout == ORACLE_CACHE_TOKEN_MAJOR
                                        ? (b * cache_tokens + row) * N + n
                                        : (b * N + n) * cache_tokens + row;
                for (int64_t e = 0; e < D; ++e) head[e] = (float)k_row[n * D + e];
                rope3d_oracle_quantize_head_e4m3(head, D, k_codes + code_off, k_scale + scale_off);
                for (int64_t e = 0; e < D; ++e) head[e] = (float)v_row[n * D + e];
                rope3d_oracle_quantize_head_e4m3(head, D, v_codes + code_off, v_scale + scale_off);
            }
        }
    }
    free(k_row);
    free(v_row);
    free(head);
    return rc;
}

/* ------------------------------------------------------------------ NVFP4 KV cache
 *
 * Quantize-on-append into NVFP4, the Blackwell 4-bit format the LongLive-2.0 abstract
 * names for its KV cache (the pages give no further detail; this is the format as
 * NVIDIA defines it): each block of 16 consecutive elements of a head holds 16 E2M1
 * codes and one E4M3 block scale S; a per-tensor fp32 scale g (the caller's, one for K
 * and one for V) sits above the block scales.  A reader recovers
 * x ~ value(code) * value(S) * g.  The rounding recipe used here, in fp32:
 *   k = 1 / (6 g)                      per tensor; 6 = E2M1's largest magnitude;
 *   S = E4M3(amax k)                   amax = largest |x| in the block;
 *   r = 1 / (value(S) g)  (0 if S is zero);
 *   code = E2M1(x r)                   round to nearest, ties to the even code, saturating;
 * every division, product and reciprocal a single fp32 operation rounded to nearest.
 * Codes are packed two per byte, element 2j in the low nibble.
 *
 * E2M1: sign bit, 2 exponent bits with bias 1, 1 mantissa bit; exponent field 0 is
 * subnormal (m/2); the magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6; no infinity, no NaN.
 */
double rope3d_oracle_e2m1_value(int code)
{
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double v = e == 0 ? (double)m / 2.0 : ldexp(1.0 + (double)m / 2.0, e - 1);
    return sign ? -v : v;
}

/* Nearest E2M1 code of x (finite), ties to the even code, saturating at +-6; found by
 * scanning the 8 non-negative codes in increasing order. */
int rope3d_oracle_e2m1_encode(float x)
{
    int sign = signbit(x) ? 0x8 : 0;
    double a = fabs((double)x);
    if (a >= 6.0) return sign | 0x7;
    int best = 0;
    for (int c = 0; c < 7; ++c) {
        double lo = rope3d_oracle_e2m1_value(c);
        double hi = rope3d_oracle_e2m1_value(c + 1);
        if (a >= lo && a <= hi) {
            double dlo = a - lo, dhi = hi - a;
            if (dlo < dhi) best = c;
            else if (dhi < dlo) best = c + 1;
            else best = (c % 2 == 0) ? c : c + 1;  /* tie: even mantissa */
            break;
        }
    }
    return sign | best;
}

/* One block of n (even) fp32 values -> n/2 code bytes and its E4M3 scale byte. */
void rope3d_oracle_quantize_block_nvfp4(const float* x, int64_t n, float g,
                                        unsigned char* codes, unsigned char* scale)
{
    float amax = 0.0f;
    for (int64_t e = 0; e < n; ++e) {
        float a = fabsf(x[e]);
        if (a > amax) amax = a;
    }
    float k = 1.0f / (6.0f * g);
    float sf = amax * k;
    int S = rope3d_oracle_e4m3_encode(sf);
    float sv = (float)rope3d_oracle_e4m3_value(S);
    float r = sv > 0.0f ? 1.0f / (sv * g) : 0.0f;
    for (int64_t e = 0; e < n; e += 2) {
        float lo = x[e] * r;
        float hi = x[e + 1] * r;
        codes[e / 2] = (unsigned char)(rope3d_oracle_e2m1_encode(lo) |
                                       (rope3d_oracle_e2m1_encode(hi) << 4));
    }
    *scale = (unsigned char)S;
}

/*
 * The whole step with an NVFP4 cache.  q_out is returned in fp64 as above; the caches
 * are code bytes [B][cache_tokens][N][D/2] (token-major) or [B][N][cache_tokens][D/2]
 * (head-major) and the block scales E4M3 bytes [B][cache_tokens][N][D/16] or
 * [B][N][cache_tokens][D/16].  K is quantized from its fp32 rounding, V exactly.
 */
int rope3d_oracle_qk_norm_rope_append_nvfp4(
    const double* q, const double* k, const double* v, double* q_out,
    int64_t B, int64_t N, int64_t D,
    int64_t token_begin, int64_t token_end, int64_t frame_offset,
    int64_t T, int64_t H, int64_t W,
    const double* q_norm_w, const double* k_norm_w, double eps,
    unsigned char* k_codes, unsigned char* v_codes, unsigned char* k_scales,
    unsigned char* v_scales, float k_global, float v_global,
    int64_t cache_tokens, int64_t slot,
    int n_t, int n_h, int n_w, double theta, int schedule, int pairing, int cache_layout)
{
    int rc = check_common(N, D, n_t, n_h, n_w, token_begin, token_end, frame_offset, T, H, W);
    if (rc != ORACLE_OK) return rc;
    if (B <= 0 || cache_tokens <= 0 || slot < 0 || D % 16 != 0) return ORACLE_EINVAL;
    if (token_end - token_begin > cache_tokens) return ORACLE_EINVAL;
    if (!(k_global > 0.0f) || !(v_global > 0.0f) || isinf(k_global) || isinf(v_global))
        return ORACLE_EINVAL;
    if (cache_layout != ORACLE_CACHE_TOKEN_MAJOR && cache_layout != ORACLE_CACHE_HEAD_MAJOR)
        return ORACLE_EINVAL;
    double inv[512];
    rc = rope3d_oracle_inv_freq(n_t, n_h, n_w, theta, schedule, inv);
    if (rc != ORACLE_OK) return rc;
    int64_t n_tok = token_end - token_begin;
    int64_t dim = N * D;
    double* k_row = (double*)malloc((size_t)dim * sizeof(double));
    double* v_row = (double*)malloc((size_t)dim * sizeof(double));
    float* head = (float*)malloc((size_t)D * sizeof(float));
    if (k_row == NULL || v_row == NULL || head == NULL) {
        free(k_row); free(v_row); free(head);
        return ORACLE_EINVAL;
    }
    for (int64_t b = 0; b < B && rc == ORACLE_OK; ++b) {
        for (int64_t r = 0; r < n_tok; ++r) {
            int64_t i = token_begin + r;
            int64_t row = rope3d_oracle_cache_row(i, slot, cache_tokens);
            int64_t in_off = (b * n_tok + r) * dim;
            rc = rope3d_oracle_token_pairing(q + in_off, k + in_off, v + in_off, N, D, i,
                                             frame_offset, T, H, W, q_norm_w, k_norm_w, eps,
                                             slot, cache_tokens, n_t, n_h, n_w, inv, pairing,
                                             q_out + in_off, k_row, v_row, NULL);
            if (rc != ORACLE_OK) break;
            for (int64_t n = 0; n < N; ++n) {
                int64_t head_off = cache_layout == ORACLE_CACHE_TOKEN_MAJOR
                                       ? (b * cache_tokens + row) * N + n
                                       : (b * N + n) * cache_tokens + row;
                for (int64_t blk = 0; blk < D / 16; ++blk) {
                    int64_t code_off = head_off * (D / 2) + blk * 8;
                    int64_t scale_off = head_off * (D / 16) + blk;
                    for (int64_t e = 0; e < 16; ++e)
                        head[e] = (float)k_row[n * D + blk * 16 + e];
                    rope3d_oracle_quantize_block_nvfp4(head, 16, k_global, k_codes + code_off,
                                                       k_scales + scale_off);
                    for (int64_t e = 0; e < 16; ++e)
                        head[e] = (float)v_row[n * D + blk * 16 + e];
                    rope3d_oracle_quantize_block_nvfp4(head, 16, v_global, v_codes + code_off,
                                                       v_scales + scale_off);
                }
            }
        }
    }
    free(k_row);
    free(v_row);
    free(head);
    return rc;
}

/* Threads the whole-step entry point would use with nthreads <= 0. */
int rope3d_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
