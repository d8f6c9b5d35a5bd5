/*
 * vdit_oracle.c -- plain, slow fp64 CPU oracle for spatio-temporal self-attention over the
 * latent tokens of a video diffusion transformer.
 *
 * TEST INFRASTRUCTURE. Only the test-suite, the smoke check and the CPU-baseline leg of the
 * benchmark load this library. The product library (CUDA) shares no code, header, table or
 * helper with it, and neither side includes or links the other.
 *
 * Every function below is the plain definition written out with loops, in float64, with no
 * blocking, fusion or reordering beyond what the definition states. Sources:
 *
 *   [CRoPE]  "Accelerating Video Generation Inference with Sequential-Parallel 3D Positional
 *            Encoding Using a Global Time Index", section 2.B (Causal-RoPE SP: the global time
 *            index t_global = t_local + s), section 2.A (KV cache), section 2.C (precomputed
 *            RoPE frequencies).
 *   [TR]     "Timeripple: Accelerating vDiTs by Understanding the Spatio-Temporal Correlations
 *            in Latent Space", Metodologia 1 (RoPE splits the channels into a temporal group
 *            and x / y spatial groups).
 *   [DR]     "DynamicRad: Content-Adaptive Sparse Attention for Long Video Diffusion",
 *            section 2 (logarithmic radial window of width L(t) set by the temporal distance
 *            and a decay factor gamma; long-range factor lambda; static-ratio mode).
 *   [WF]     Wave Forcing / WaveRT news item: block-causal attention over chunks of latent
 *            frames (the frame count must be divisible by 3) and a per-layer K/V cache.
 *
 * Readings where the pages leave a step open (each is also listed in the design notes):
 *   - token order is frame-major, then patch row h, then patch column w;
 *   - only time is global: h and w are local patch coordinates starting at 0;
 *   - each RoPE band is an independent 1-D rotary embedding over adjacent channel pairs
 *     (2j, 2j+1) with angular frequency theta^(-2j / band_width); bands are laid out
 *     t, h, w from channel 0;
 *   - radial: key kept iff Chebyshev patch distance <= W0 * gamma^|dt| (inclusive), with
 *     gamma = 2^-gamma_shift, or |dt| is a multiple of lambda (full width);
 *   - block-causal: chunk index floor(t / C) of the GLOBAL frame; a query sees keys whose
 *     chunk index is <= its own;
 *   - combined masks are the AND of the active predicates; a row with no kept key
 *     produces o = 0 and lse = -inf.
 *
 * Parity pins (tests/test_oracle.py): rotation norm, relative-position (global time shift)
 * invariance, group property, band membership and frequency ladder of the RoPE; single
 * chunk block-causal == bidirectional, infinite radial window == dense, closed-form kept
 * counts of the radial and block-causal masks; attention == torch fp64
 * scaled_dot_product_attention with a boolean mask and == pure-Python brute force; tile
 * list == reshape/any of the explicit mask; ring placement of the KV cache.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Token index n -> (t, h, w) with t = start_frame + local frame ([CRoPE] 2.B). */
void vo_positions(long n_tokens, int grid_h, int grid_w, int start_frame,
                  int *t, int *h, int *w)
{
    long frame_tokens = (long)grid_h * grid_w;
    for (long n = 0; n < n_tokens; ++n) {
        long f_local = n / frame_tokens;
        long rem = n % frame_tokens;
        t[n] = start_frame + (int)f_local;
        h[n] = (int)(rem / grid_w);
        w[n] = (int)(rem % grid_w);
    }
}

/* One band of a 1-D rotary embedding: rotate pairs (2j, 2j+1) of x[0..width) by the angle
 * pos * theta^(-2j/width). */
static void rope_band(const double *x, double *y, int width, int pos, double theta)
{
    for (int j = 0; j < width / 2; ++j) {
        double omega = pow(theta, -2.0 * j / width);
        double a = (double)pos * omega;
        double c = cos(a), s = sin(a);
        double x0 = x[2 * j], x1 = x[2 * j + 1];
        y[2 * j] = x0 * c - x1 * s;
        y[2 * j + 1] = x0 * s + x1 * c;
    }
}

/* 3-D RoPE of every head vector of x [n_tokens, heads, head_dim] ([TR] Metodologia 1; time
 * position from [CRoPE] 2.B). x and y may alias. */
void vo_rope3d(const double *x, double *y, long n_tokens, int heads, int head_dim,
               const int *t, const int *h, const int *w,
               int band_t, int band_h, int band_w, double theta)
{
    #pragma omp parallel for schedule(static)
    for (long n = 0; n < n_tokens; ++n) {
        for (int hh = 0; hh < heads; ++hh) {
            const double *xv = x + (n * heads + hh) * (long)head_dim;
            double *yv = y + (n * heads + hh) * (long)head_dim;
            double tmp[1024];
            rope_band(xv, tmp, band_t, t[n], theta);
            rope_band(xv + band_t, tmp + band_t, band_h, h[n], theta);
            rope_band(xv + band_t + band_h, tmp + band_t + band_h, band_w, w[n], theta);
            memcpy(yv, tmp, sizeof(double) * (size_t)head_dim);
        }
    }
}

/* Mask predicate for one (query, key) pair. */
static int keep_pair(int tq, int hq, int wq, int tk, int hk, int wk,
                     int block_causal, int radial, int chunk_frames,
                     long long w0, int gamma_shift, int lambda)
{
    if (block_causal) {
        /* [WF]: chunk-by-chunk causality over global frames; bidirectional inside a chunk */
        if (tk / chunk_frames > tq / chunk_frames)
            return 0;
    }
    if (radial) {
        /* [DR] section 2: window width L(dt) = W0 * gamma^|dt|, gamma = 2^-gamma_shift;
         * frames at |dt| multiple of lambda keep full width. */
        int dt = abs(tq - tk);
        if (lambda > 0 && dt % lambda == 0)
            return 1;
        int dh = abs(hq - hk), dw = abs(wq - wk);
        int cheb = dh > dw ? dh : dw;
        double width = (double)w0 * ldexp(1.0, -gamma_shift * dt);
        if (!((double)cheb <= width))
            return 0;
    }
    return 1;
}

/* Explicit boolean mask m[i * nk + j] for nq query tokens against nk key tokens. A key with
 * kvalid[j] == 0 (an empty cache slot) is never kept. */
void vo_mask_rows(unsigned char *m, long nq, const int *tq, const int *hq, const int *wq,
                  long nk, const int *tk, const int *hk, const int *wk,
                  const unsigned char *kvalid,
                  int block_causal, int radial, int chunk_frames, long long w0,
                  int gamma_shift, int lambda)
{
    #pragma omp parallel for schedule(static)
    for (long i = 0; i < nq; ++i)
        for (long j = 0; j < nk; ++j)
            m[i * nk + j] = (unsigned char)(kvalid[j] &&
                keep_pair(tq[i], hq[i], wq[i], tk[j], hk[j], wk[j], block_causal, radial,
                          chunk_frames, w0, gamma_shift, lambda));
}

/* Masked softmax attention, two passes per (head, query) in float64:
 *   o_i = sum_j softmax_j(scale * q_i . k_j  restricted to mask_ij) v_j,
 *   lse_i = log sum_j exp(scale * q_i . k_j) over kept j.
 * q [nq, heads, D], k and v [nk, heads, D], mask [nq, nk], o [nq, heads, D], lse [heads, nq].
 * q and k are the rotated vectors. */
void vo_attention(const double *q, const double *k, const double *v, const unsigned char *mask,
                  long nq, long nk, int heads, int head_dim, double scale,
                  double *o, double *lse)
{
    #pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
        #pragma omp for schedule(dynamic, 4) collapse(2)
        for (int hh = 0; hh < heads; ++hh) {
            for (long i = 0; i < nq; ++i) {
                const double *qi = q + (i * heads + hh) * (long)head_dim;
                double *oi = o + (i * heads + hh) * (long)head_dim;
                const unsigned char *mi = mask + i * nk;
                double mx = -INFINITY;
                for (long j = 0; j < nk; ++j) {
                    if (!mi[j])
                        continue;
                    const double *kj = k + (j * heads + hh) * (long)head_dim;
                    double dot = 0.0;
                    for (int d = 0; d < head_dim; ++d)
                        dot += qi[d] * kj[d];
                    s[j] = scale * dot;
                    if (s[j] > mx)
                        mx = s[j];
                }
                for (int d = 0; d < head_dim; ++d)
                    oi[d] = 0.0;
                if (mx == -INFINITY) {
                    lse[(long)hh * nq + i] = -INFINITY;
                    continue;
                }
                double sum = 0.0;
                for (long j = 0; j < nk; ++j) {
                    if (!mi[j])
                        continue;
                    double p = exp(s[j] - mx);
                    sum += p;
                    const double *vj = v + (j * heads + hh) * (long)head_dim;
                    for (int d = 0; d < head_dim; ++d)
                        oi[d] += p * vj[d];
                }
                for (int d = 0; d < head_dim; ++d)
                    oi[d] /= sum;
                lse[(long)hh * nq + i] = mx + log(sum);
            }
        }
        free(s);
    }
}

/* Tile list of the explicit mask: tiles of tile x tile (query rows x key columns), CSR by
 * query tile ascending, then key tile ascending. A tile is listed iff some in-range entry is
 * kept; its flag is 1 ("full") iff it lies wholly in range and every entry is kept.
 * row_ptr has n_qt + 1 entries; col_idx and full have room for n_qt * n_kt. Returns the number
 * of kept (query, key) pairs. The mask is evaluated one query tile at a time (the explicit
 * per-pair predicate, streamed so the full matrix never has to be held). */
long long vo_tiles(long nq, const int *tq, const int *hq, const int *wq,
                   long nk, const int *tk, const int *hk, const int *wk,
                   const unsigned char *kvalid,
                   int block_causal, int radial, int chunk_frames, long long w0,
                   int gamma_shift, int lambda, int tile,
                   int *row_ptr, int *col_idx, unsigned char *full)
{
    long n_qt = (nq + tile - 1) / tile, n_kt = (nk + tile - 1) / tile;
    unsigned char *m = (unsigned char *)malloc((size_t)tile * (size_t)(nk > 0 ? nk : 1));
    long long kept_total = 0;
    int count = 0;
    row_ptr[0] = 0;
    for (long qt = 0; qt < n_qt; ++qt) {
        long i0 = qt * tile, rows = nq - i0 < tile ? nq - i0 : tile;
        vo_mask_rows(m, rows, tq + i0, hq + i0, wq + i0, nk, tk, hk, wk, kvalid,
                     block_causal, radial, chunk_frames, w0, gamma_shift, lambda);
        for (long kt = 0; kt < n_kt; ++kt) {
            long j0 = kt * tile, cols = nk - j0 < tile ? nk - j0 : tile;
            long kept = 0;
            for (long r = 0; r < rows; ++r)
                for (long c = 0; c < cols; ++c)
                    kept += m[r * nk + j0 + c];
            kept_total += kept;
            if (kept > 0) {
                col_idx[count] = (int)kt;
                full[count] = (unsigned char)(rows == tile && cols == tile &&
                                              kept == (long)tile * tile);
                ++count;
            }
        }
        row_ptr[qt + 1] = count;
    }
    free(m);
    return kept_total;
}

/* Positions held by a KV cache of capacity_frames frame slots after frames
 * [first_frame, last_frame] have been written, frame f living in slot f mod capacity_frames
 * ([CRoPE] 2.A KV cache; [WF] per-layer K/V cache of past chunks). For each cache token j:
 * (t, h, w) of the token it holds and valid[j]; an empty slot gets t = -1, valid = 0. */
void vo_cache_positions(int capacity_frames, int first_frame, int last_frame,
                        int grid_h, int grid_w, int *t, int *h, int *w, unsigned char *valid)
{
    long frame_tokens = (long)grid_h * grid_w;
    for (long j = 0; j < (long)capacity_frames * frame_tokens; ++j) {
        int slot = (int)(j / frame_tokens);
        long rem = j % frame_tokens;
        int held = -1;
        for (int f = first_frame; f <= last_frame; ++f)
            if (f >= 0 && f % capacity_frames == slot)
                held = f;
        t[j] = held;
        h[j] = (int)(rem / grid_w);
        w[j] = (int)(rem % grid_w);
        valid[j] = (unsigned char)(held >= 0);
    }
}

/* KV-cache append: rotate the chunk's K with its global time positions, then place K' and V
 * of global frame f into slot f mod capacity_frames of the head-major cache
 * [heads, capacity_frames * grid_h * grid_w, head_dim]. k and v are [n_frames * frame tokens,
 * heads, head_dim]. */
void vo_kv_append(double *k_cache, double *v_cache, int capacity_frames,
                  int grid_h, int grid_w, int heads, int head_dim,
                  int band_t, int band_h, int band_w, double theta,
                  const double *k, const double *v, int start_frame, int n_frames)
{
    long frame_tokens = (long)grid_h * grid_w;
    long n_tok = frame_tokens * n_frames;
    long cap_tok = frame_tokens * capacity_frames;
    int *t = (int *)malloc(sizeof(int) * (size_t)n_tok);
    int *h = (int *)malloc(sizeof(int) * (size_t)n_tok);
    int *w = (int *)malloc(sizeof(int) * (size_t)n_tok);
    double *kr = (double *)malloc(sizeof(double) * (size_t)(n_tok * heads * head_dim));
    vo_positions(n_tok, grid_h, grid_w, start_frame, t, h, w);
    vo_rope3d(k, kr, n_tok, heads, head_dim, t, h, w, band_t, band_h, band_w, theta);
    for (long n = 0; n < n_tok; ++n) {
        int f = t[n];
        long slot_tok = (long)(f % capacity_frames) * frame_tokens + n % frame_tokens;
        for (int hh = 0; hh < heads; ++hh) {
            const double *ks = kr + (n * heads + hh) * (long)head_dim;
            const double *vs = v + (n * heads + hh) * (long)head_dim;
            double *kd = k_cache + ((long)hh * cap_tok + slot_tok) * head_dim;
            double *vd = v_cache + ((long)hh * cap_tok + slot_tok) * head_dim;
            memcpy(kd, ks, sizeof(double) * (size_t)head_dim);
            memcpy(vd, vs, sizeof(double) * (size_t)head_dim);
        }
    }
    free(t); free(h); free(w); free(kr);
}

/* Number of OpenMP threads the parallel loops above run on (for reporting). */
int vo_threads(void) { return omp_get_max_threads(); }

/* Rounds each x[i] to the nearest bfloat16 value, ties to even, in place. bfloat16 keeps 8
 * significant bits and float32's exponent range: for |x| >= 2^-126 the spacing of bfloat16
 * values around x is 2^(e-7) with e = floor(log2 |x|); below that (subnormal) it is 2^-133.
 * x / spacing is exact (a power-of-two scaling), and nearbyint rounds it to the nearest integer
 * with ties to even under the default rounding mode. Results of magnitude 2^128 or more are
 * infinite (the largest finite bfloat16 is (2 - 2^-7) 2^127). This is the precision in which
 * the dynamic-threshold mode's keep decision is taken (the tensor core multiplies bfloat16
 * operands); it is not a step of the attention itself. */
void vo_round_bf16(double *x, long n)
{
    for (long i = 0; i < n; ++i) {
        double a = x[i];
        if (a == 0.0 || isnan(a) || isinf(a)) continue;
        int e = ilogb(a);
        int step_exp = e < -126 ? -133 : e - 7;
        double r = ldexp(nearbyint(ldexp(a, -step_exp)), step_exp);
        if (fabs(r) >= ldexp(1.0, 128)) r = a > 0 ? INFINITY : -INFINITY;
        x[i] = r;
    }
}
