/*
 * hstu_oracle.c -- plain fp64 CPU oracle for the HSTU layer forward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing here is part of the product path: only
 * the tests, the package smoke check and the benchmark's CPU-baseline leg may
 * load this library. It shares no code, header, table or constant with the
 * CUDA implementation.
 *
 * What it computes (HSTU, "Actions Speak Louder than Words: Trillion-Parameter
 * Sequential Transducers for Generative Recommendations", arXiv 2402.17152;
 * the abstract names HSTU, the generative-recommenders README section
 * "HSTU Ultra attention benchmark" names the layer order: UVQK projection,
 * attention, output normalization and projection, residual connection):
 *
 *   for every sequence b (tokens o_b .. o_{b+1}-1), head h, position i:
 *     A[o_b+i,h,:] = (1/N) * sum_{j<=i} silu(s_ij) * v[o_b+j,h,:]
 *     s_ij = <q[o_b+i,h,:], k[o_b+j,h,:]>
 *          + pos[h][min(i-j, P-1)]
 *          + time[h][clamp(floor_log2(max(1, ts[o_b+i]-ts[o_b+j])), 0, NB-1)]
 *
 * N is the caller's max_seqlen. Layer: UVQK = silu(x W1^T + b1) split as
 * U|V|Q|K, attention as above, Y = LayerNorm(A) * U over the H*d features of a
 * token, out = x + Y W2^T + b2.
 *
 * Everything is evaluated in double precision, one output row at a time, in
 * the order of the definition. No blocking, no fusion, no reordering.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* floor(log2(x)) for x >= 1 by counting halvings: integer arithmetic only,
 * so int64 differences above 2^53 are still exact. */
int32_t hstu_oracle_floor_log2(int64_t x) {
    int32_t r = 0;
    while (x > 1) {
        x >>= 1;
        r += 1;
    }
    return r;
}

/* Log-time bucket of a timestamp difference: clamp(floor(log2(max(1, dt))), 0, NB-1). */
int32_t hstu_oracle_time_bucket(int64_t dt, int32_t num_buckets) {
    int64_t x = dt < 1 ? 1 : dt;
    int32_t bkt = hstu_oracle_floor_log2(x);
    if (bkt < 0) bkt = 0;
    if (bkt > num_buckets - 1) bkt = num_buckets - 1;
    return bkt;
}

/* Relative-position index: min(i - j, P - 1) for j <= i. */
int32_t hstu_oracle_pos_index(int64_t i, int64_t j, int32_t num_pos) {
    int64_t r = i - j;
    if (r > num_pos - 1) r = num_pos - 1;
    return (int32_t)r;
}

double hstu_oracle_silu(double x) { return x / (1.0 + exp(-x)); }

/* For every sequence, every i, every j <= i (row-major in i, then j), write the
 * relative-position index and the time bucket. Arrays hold sum_b n_b(n_b+1)/2
 * entries. pos_idx or bucket may be NULL. */
void hstu_oracle_bias_indices(const int64_t* seq_offsets, int32_t B, const int64_t* ts,
                              int32_t num_pos, int32_t num_buckets,
                              int32_t* pos_idx, int32_t* bucket) {
    int64_t e = 0;
    for (int32_t b = 0; b < B; ++b) {
        int64_t o = seq_offsets[b], n = seq_offsets[b + 1] - seq_offsets[b];
        for (int64_t i = 0; i < n; ++i) {
            for (int64_t j = 0; j <= i; ++j) {
                if (pos_idx) pos_idx[e] = hstu_oracle_pos_index(i, j, num_pos);
                if (bucket) bucket[e] = hstu_oracle_time_bucket(ts[o + i] - ts[o + j], num_buckets);
                ++e;
            }
        }
    }
}

/* Sequence that holds token t (seq_offsets is non-decreasing). */
static int32_t seq_of_token(const int64_t* seq_offsets, int32_t B, int64_t t) {
    for (int32_t b = 0; b < B; ++b)
        if (t >= seq_offsets[b] && t < seq_offsets[b + 1]) return b;
    return -1;
}

/* One output row (token t, all heads) of the attention. q,k,v are addressed with
 * explicit token strides so the layer can pass its U|V|Q|K buffer. */
static void attn_row(int64_t t, int32_t b, const int64_t* seq_offsets, int32_t H,
                     int32_t dqk, int32_t dv,
                     const double* q, int64_t q_tok, const double* k, int64_t k_tok,
                     const double* v, int64_t v_tok, const int64_t* ts,
                     const double* pos, int32_t num_pos, const double* tbias,
                     int32_t num_buckets, int32_t max_seqlen, double* out_row) {
    int64_t o = seq_offsets[b];
    int64_t i = t - o;
    for (int32_t h = 0; h < H; ++h) {
        double* a = out_row + (int64_t)h * dv;
        for (int32_t c = 0; c < dv; ++c) a[c] = 0.0;
        const double* qi = q + t * q_tok + (int64_t)h * dqk;
        for (int64_t j = 0; j <= i; ++j) {
            const double* kj = k + (o + j) * k_tok + (int64_t)h * dqk;
            const double* vj = v + (o + j) * v_tok + (int64_t)h * dv;
            double s = 0.0;
            for (int32_t c = 0; c < dqk; ++c) s += qi[c] * kj[c];
            if (pos) s += pos[(int64_t)h * num_pos + hstu_oracle_pos_index(i, j, num_pos)];
            if (ts && tbias)
                s += tbias[(int64_t)h * num_buckets +
                           hstu_oracle_time_bucket(ts[o + i] - ts[o + j], num_buckets)];
            double p = hstu_oracle_silu(s);
            for (int32_t c = 0; c < dv; ++c) a[c] += p * vj[c];
        }
        for (int32_t c = 0; c < dv; ++c) a[c] /= (double)max_seqlen;
    }
}

/* Attention forward. q,k: [T,H,dqk]; v: [T,H,dv] (token strides given in
 * elements). rows == NULL: out is [T,H,dv]. Otherwise out is [n_rows,H,dv] and
 * holds the requested tokens only. pos / ts / tbias may be NULL (term absent).
 * Returns 0, or -1 if a requested row is outside every sequence. */
int hstu_oracle_attn(const int64_t* seq_offsets, int32_t B, int32_t H, int32_t dqk, int32_t dv,
                     const double* q, int64_t q_tok, const double* k, int64_t k_tok,
                     const double* v, int64_t v_tok, const int64_t* ts,
                     const double* pos, int32_t num_pos, const double* tbias,
                     int32_t num_buckets, int32_t max_seqlen,
                     const int64_t* rows, int64_t n_rows, double* out) {
    int64_t T = seq_offsets[B];
    int64_t n = rows ? n_rows : T;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(|:bad)
    for (int64_t r = 0; r < n; ++r) {
        int64_t t = rows ? rows[r] : r;
        int32_t b = seq_of_token(seq_offsets, B, t);
        if (b < 0) { bad = 1; continue; }
        attn_row(t, b, seq_offsets, H, dqk, dv, q, q_tok, k, k_tok, v, v_tok, ts, pos,
                 num_pos, tbias, num_buckets, max_seqlen, out + r * (int64_t)H * dv);
    }
    return bad ? -1 : 0;
}

/* ---------------------------------------------------------------- backward
 * Gradients of the attention forward above for an upstream gradient dout
 * [T,H,dv] (the chain rule through s = q.k + pos + time, p = silu(s) / N,
 * out = sum p v; the pages' reference implementation has forward and
 * backward attention kernels, generative-recommenders README, section "HSTU
 * Ultra attention benchmark"):
 *   dv[j]  = sum_{i>=j} p_ij dout[i]
 *   ds_ij  = (dout[i] . v[j]) silu'(s_ij) / N,
 *            silu'(s) = sig(s) (1 + s (1 - sig(s))), sig(s) = 1 / (1 + e^-s)
 *   dq[i]  = sum_{j<=i} ds_ij k[j],   dk[j] = sum_{i>=j} ds_ij q[i]
 *   dpos[h][r] = sum of ds_ij over pairs with min(i-j, P-1) = r
 *   dtime[h][b] = sum of ds_ij over pairs with bucket(t_i - t_j) = b
 * All arrays contiguous: q,k,dq,dk [T,H,dqk], v,dout,dv [T,H,dv], dpos [H,P],
 * dtime [H,NB] (each may be NULL when its term is absent). Outputs are
 * overwritten. Serial over pairs (the accumulation targets are shared). */
double hstu_oracle_silu_grad(double s) {
    const double sg = 1.0 / (1.0 + exp(-s));
    return sg * (1.0 + s * (1.0 - sg));
}

void hstu_oracle_attn_bwd(const int64_t* seq_offsets, int32_t B, int32_t H, int32_t dqk,
                          int32_t dv, const double* q, const double* k, const double* v,
                          const int64_t* ts, const double* pos, int32_t num_pos,
                          const double* tbias, int32_t num_buckets, int32_t max_seqlen,
                          const double* dout, double* dq, double* dk, double* dvv,
                          double* dpos, double* dtime) {
    const int64_t T = seq_offsets[B];
    for (int64_t e = 0; e < T * H * dqk; ++e) dq[e] = dk[e] = 0.0;
    for (int64_t e = 0; e < T * H * dv; ++e) dvv[e] = 0.0;
    if (dpos) for (int64_t e = 0; e < (int64_t)H * num_pos; ++e) dpos[e] = 0.0;
    if (dtime) for (int64_t e = 0; e < (int64_t)H * num_buckets; ++e) dtime[e] = 0.0;
    const double inv_n = 1.0 / (double)max_seqlen;
    for (int32_t b = 0; b < B; ++b) {
        const int64_t o = seq_offsets[b], n = seq_offsets[b + 1] - o;
        for (int32_t h = 0; h < H; ++h) {
            for (int64_t i = 0; i < n; ++i) {
                const double* qi = q + ((o + i) * H + h) * dqk;
                const double* gi = dout + ((o + i) * H + h) * dv;
                for (int64_t j = 0; j <= i; ++j) {
                    const double* kj = k + ((o + j) * H + h) * dqk;
                    const double* vj = v + ((o + j) * H + h) * dv;
                    double s = 0.0;
                    for (int32_t c = 0; c < dqk; ++c) s += qi[c] * kj[c];
                    int32_t pidx = -1, bkt = -1;
                    if (pos) {
                        pidx = hstu_oracle_pos_index(i, j, num_pos);
                        s += pos[(int64_t)h * num_pos + pidx];
                    }
                    if (ts && tbias) {
                        bkt = hstu_oracle_time_bucket(ts[o + i] - ts[o + j], num_buckets);
                        s += tbias[(int64_t)h * num_buckets + bkt];
                    }
                    const double p = hstu_oracle_silu(s) * inv_n;
                    double dp = 0.0;
                    for (int32_t c = 0; c < dv; ++c) {
                        dvv[((o + j) * H + h) * dv + c] += p * gi[c];
                        dp += gi[c] * vj[c];
                    }
                    const double ds = dp * hstu_oracle_silu_grad(s) * inv_n;
                    for (int32_t c = 0; c < dqk; ++c) {
                        dq[((o + i) * H + h) * dqk + c] += ds * kj[c];
                        dk[((o + j) * H + h) * dqk + c] += ds * qi[c];
                    }
                    if (dpos && pidx >= 0) dpos[(int64_t)h * num_pos + pidx] += ds;
                    if (dtime && bkt >= 0) dtime[(int64_t)h * num_buckets + bkt] += ds;
                }
            }
        }
    }
}

/* y[m, :] = act(x[m, :] W^T + bias) + residual[m, :]; x [M,K], W [N,K].
 * act = 1 applies SiLU. bias / residual may be NULL. */
void hstu_oracle_linear(int64_t M, int32_t K, int32_t N, const double* x, const double* W,
                        const double* bias, int32_t act_silu, const double* residual,
                        double* y) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int32_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int32_t c = 0; c < K; ++c) acc += x[m * K + c] * W[(int64_t)n * K + c];
            if (bias) acc += bias[n];
            if (act_silu) acc = hstu_oracle_silu(acc);
            if (residual) acc += residual[m * N + n];
            y[m * N + n] = acc;
        }
    }
}

/* ---------------------------------------------------------------- FP8 (E4M3)
 * Row-wise E4M3 quantization and FP8 addmm for the layer's two projections
 * (generative-recommenders README, section "FP8 linear reference and
 * benchmark": row-wise E4M3 quantization of both operands, fp32
 * accumulation, the row scales applied to the product).
 *
 * E4M3 (the OCP 8-bit float "E4M3FN" format): 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits. Exponent field 0 holds the subnormals
 * m/8 * 2^-6; fields 1..15 hold (1 + m/8) * 2^(e - 7), except that field 15
 * with mantissa 7 is NaN (no infinities), so the largest finite magnitude is
 * 1.75 * 2^8 = 448. Conversion rounds to the nearest value, ties to an even
 * mantissa, and saturates finite overflow (and infinity) to +-448. */

float hstu_oracle_e4m3_to_float(uint8_t c) {
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return (float)(sign ? -v : v);
}

/* nearest integer to q >= 0, ties to even */
static double round_half_even(double q) {
    const double f = floor(q), r = q - f;
    if (r > 0.5) return f + 1.0;
    if (r < 0.5) return f;
    return fmod(f, 2.0) == 0.0 ? f : f + 1.0;
}

uint8_t hstu_oracle_e4m3_from_float(float x) {
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    const double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;                 /* saturate (448 itself included) */
    if (a < ldexp(1.0, -6)) {                           /* subnormal range: steps of 2^-9 */
        const double m = round_half_even(a / ldexp(1.0, -9));
        return sign | (uint8_t)m;                       /* m == 8 is the smallest normal */
    }
    int ex;
    const double f = frexp(a, &ex);                     /* a = f 2^ex, f in [0.5, 1) */
    int e = ex - 1;                                     /* a = (2f) 2^e, 2f in [1, 2) */
    double m = round_half_even((2.0 * f - 1.0) * 8.0);
    if (m == 8.0) {
        m = 0.0;
        e += 1;
    }
    const int field = e + 7;
    if (field > 15 || (field == 15 && m == 7.0)) return sign | 0x7E;
    return sign | (uint8_t)((field << 3) | (int)m);
}

/* Row-wise quantization of x [M, K] (fp32 values): amax_r = max |x[r, :]|;
 * inv_r = 448 / amax_r and scale_r = amax_r / 448 in fp32; code[r, c] =
 * e4m3(x[r, c] * inv_r) with the product rounded to fp32 first. Then
 * x[r, c] ~ e4m3_to_float(code) * scale_r. A row whose inv_r is not a finite
 * fp32 number -- all zeros, or amax_r below 448 / FLT_MAX (about 1.3e-36) --
 * takes inv 0 and scale 1, so its codes are (signed) zeros. */
void hstu_oracle_quant_rows_e4m3(int64_t M, int32_t K, const float* x, uint8_t* codes,
                                 float* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        float amax = 0.0f;
        for (int32_t c = 0; c < K; ++c) {
            const float v = fabsf(x[r * K + c]);
            if (v > amax) amax = v;
        }
        volatile float q = amax > 0.0f ? 448.0f / amax : 0.0f;
        const int finite = amax > 0.0f && q <= FLT_MAX;
        volatile float inv = finite ? q : 0.0f;
        volatile float scale = finite ? amax / 448.0f : 1.0f;
        for (int32_t c = 0; c < K; ++c) {
            volatile float y = x[r * K + c] * inv;
            codes[r * K + c] = hstu_oracle_e4m3_from_float(y);
        }
        scales[r] = scale;
    }
}

/* y[m, n] = act(sum_c e4m3(xq[m, c]) e4m3(wq[n, c]) sx[m] sw[n] + bias[n])
 *           + residual[m, n], in fp64 from the codes; xq [M, K], wq [N, K]. */
void hstu_oracle_linear_fp8(int64_t M, int32_t K, int32_t N, const uint8_t* xq,
                            const float* sx, const uint8_t* wq, const float* sw,
                            const double* bias, int32_t act_silu, const double* residual,
                            double* y) {
    double lut[256];
    for (int c = 0; c < 256; ++c) lut[c] = (double)hstu_oracle_e4m3_to_float((uint8_t)c);
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int32_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int32_t c = 0; c < K; ++c)
                acc += lut[xq[m * K + c]] * lut[wq[(int64_t)n * K + c]];
            acc *= (double)sx[m] * (double)sw[n];
            if (bias) acc += bias[n];
            if (act_silu) acc = hstu_oracle_silu(acc);
            if (residual) acc += residual[m * N + n];
            y[m * N + n] = acc;
        }
    }
}

/* One row of LayerNorm over F features: biased variance, eps inside the
 * square root, then gamma / beta (NULL = 1 / 0). */
static void ln_row(const double* ar, int32_t F, const double* gamma, const double* beta,
                   double eps, double* yr) {
    double mean = 0.0;
    for (int32_t c = 0; c < F; ++c) mean += ar[c];
    mean /= (double)F;
    double var = 0.0;
    for (int32_t c = 0; c < F; ++c) var += (ar[c] - mean) * (ar[c] - mean);
    var /= (double)F;
    double rstd = 1.0 / sqrt(var + eps);
    for (int32_t c = 0; c < F; ++c)
        yr[c] = (ar[c] - mean) * rstd * (gamma ? gamma[c] : 1.0) + (beta ? beta[c] : 0.0);
}

/* y[m, :] = LayerNorm(a[m, :]) * u[m, :] over F features (ln_row), a, u, y
 * with row strides a_ld, u_ld, F. */
void hstu_oracle_layernorm_gate(int64_t M, int32_t F, const double* a, int64_t a_ld,
                                const double* u, int64_t u_ld, const double* gamma,
                                const double* beta, double eps, double* y) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        ln_row(a + m * a_ld, F, gamma, beta, eps, y + m * F);
        for (int32_t c = 0; c < F; ++c) y[m * F + c] *= u[m * u_ld + c];
    }
}

/* y[m, :] = LayerNorm(a[m, :]) over F features (ln_row); a has row stride
 * a_ld, y row stride F. The layer's input normalization (generative-
 * recommenders README, "HSTU Ultra attention benchmark": input norm before
 * the UVQK projection). */
void hstu_oracle_layernorm(int64_t M, int32_t F, const double* a, int64_t a_ld,
                           const double* gamma, const double* beta, double eps, double* y) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) ln_row(a + m * a_ld, F, gamma, beta, eps, y + m * F);
}

/* Full layer forward for the requested rows (rows == NULL: every token).
 * x [T,D], W1 [4Hd,D] (output columns U|V|Q|K), W2 [D,Hd]; out [n,D].
 * With input_norm, the projection reads LayerNorm(x) (over D features, the
 * output norm's eps, affine in_gamma / in_beta, NULL = identity); the
 * residual adds x itself.
 * Only the prefix of each touched sequence up to its last requested row is
 * projected, since later tokens cannot reach a requested row.
 * Returns 0, -1 for a bad row, -2 on allocation failure. */
int hstu_oracle_layer(int64_t T, int32_t D, const double* x, const double* W1,
                      const double* b1, const double* W2, const double* b2,
                      const double* gamma, const double* beta, double eps,
                      const double* in_gamma, const double* in_beta, int32_t input_norm,
                      const int64_t* seq_offsets, int32_t B, int32_t H, int32_t d,
                      const int64_t* ts, const double* pos, int32_t num_pos,
                      const double* tbias, int32_t num_buckets, int32_t max_seqlen,
                      const int64_t* rows, int64_t n_rows, double* out) {
    int64_t n = rows ? n_rows : T;
    int64_t F = (int64_t)H * d, W = 4 * F;
    int64_t* upto = (int64_t*)malloc(sizeof(int64_t) * (B > 0 ? B : 1));
    double* uvqk = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * (size_t)W);
    double* attn = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * (size_t)F);
    double* ygate = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * (size_t)F);
    double* urow = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * (size_t)F);
    double* xrow = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * (size_t)D);
    double* xn = input_norm ? (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * (size_t)D)
                            : NULL;
    const double* xin = x;
    int rc = 0;
    if (!upto || !uvqk || !attn || !ygate || !urow || !xrow || (input_norm && !xn)) {
        rc = -2;
        goto done;
    }
    if (input_norm) {
        hstu_oracle_layernorm(T, D, x, D, in_gamma, in_beta, eps, xn);
        xin = xn;
    }
    for (int32_t b = 0; b < B; ++b) upto[b] = seq_offsets[b];  /* exclusive end */
    for (int64_t r = 0; r < n; ++r) {
        int64_t t = rows ? rows[r] : r;
        int32_t b = seq_of_token(seq_offsets, B, t);
        if (b < 0) { rc = -1; goto done; }
        if (t + 1 > upto[b]) upto[b] = t + 1;
    }
    /* 1. UVQK = silu(x W1^T + b1), x normalized or not, for each needed prefix */
    for (int32_t b = 0; b < B; ++b) {
        int64_t o = seq_offsets[b], m = upto[b] - o;
        if (m > 0)
            hstu_oracle_linear(m, D, (int32_t)W, xin + o * D, W1, b1, 1, NULL, uvqk + o * W);
    }
    /* 2. attention with U|V|Q|K views of the projection (token stride 4Hd) */
    rc = hstu_oracle_attn(seq_offsets, B, H, d, d, uvqk + 2 * F, W, uvqk + 3 * F, W,
                          uvqk + F, W, ts, pos, num_pos, tbias, num_buckets, max_seqlen,
                          rows ? rows : NULL, n, attn);
    if (rc) goto done;
    /* 3. Y = LayerNorm(A) * U */
    for (int64_t r = 0; r < n; ++r) {
        int64_t t = rows ? rows[r] : r;
        memcpy(urow + r * F, uvqk + t * W, sizeof(double) * (size_t)F);
    }
    hstu_oracle_layernorm_gate(n, (int32_t)F, attn, F, urow, F, gamma, beta, eps, ygate);
    /* 4. out = x + Y W2^T + b2 */
    for (int64_t r = 0; r < n; ++r) {
        int64_t t = rows ? rows[r] : r;
        memcpy(xrow + r * D, x + t * D, sizeof(double) * (size_t)D);
    }
    hstu_oracle_linear(n, (int32_t)F, D, ygate, W2, b2, 0, xrow, out);
done:
    free(upto); free(uvqk); free(attn); free(ygate); free(urow); free(xrow); free(xn);
    return rc;
}

/* Threads an OpenMP parallel region actually uses (1 without OpenMP). */
int hstu_oracle_num_threads(void) {
    int nt = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            nt = omp_get_num_threads();
#endif
        }
    }
    return nt;
}
