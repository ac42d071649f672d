/*
 * dit_oracle.c -- plain, slow, fp64 CPU oracle for the per-block memory-bound
 * operators of a dense single-stream video+audio DiT (MiniMax-H3 shaped).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library.
 *
 * Sources.  The operators are named, not defined, by:
 *   [REPORT]  the LMSYS report summary at news.cocoloop.cn (page
 *             "minimax-h3-sglang-h200", untitled in the text), section
 *             "Só com três camadas de aceleração somadas chega-se a 6
 *             vezes": fused AdaLN update, gated residual, SwiGLU,
 *             QK RMSNorm with 3D RoPE; the fused layer changes no result;
 *             Cache-DiT reuses results between neighbouring denoising steps
 *             when a residual-difference threshold (0.04 conservative, 0.08
 *             stride mode) allows it.
 *   [CEVIU]   "SGLang acelera MiniMax-H3 em GPUs H200 e redefine geração de
 *             vídeo por IA" (ceviu.com.br), first paragraph: the three
 *             pillars (fused kernels for AdaLN, SwiGLU, QK RMSNorm, 3D RoPE;
 *             Cache-DiT; SubBlock attention).
 *   [H3BASE]  "MiniMax H3 mở trọng số: H3-Base có gì và còn thiếu gì?"
 *             (studioglobal.ai), section "Kiến trúc: tạo hình và tiếng trong
 *             cùng một luồng": dense single-stream transformer whose AdaLN
 *             branch outputs can be precomputed and cached.
 * The pages print no formula; every function below is the textbook definition
 * of the named operator, with the readings listed beside it.
 *
 * Arithmetic.  Every stored input (bf16 bit patterns, fp64 modulation or
 * weights) is read exactly into fp64; the definition is evaluated in fp64 in
 * the plainest order; callers round a final output to bf16 once with
 * dito_f64_to_bf16 (round to nearest, ties to even, straight from fp64).
 *
 * Parity pins: closed forms, invariants, hand-worked golden values and exact
 * rational brute force live in the test-suite (tests/test_oracle_*.py).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------ bf16 */

/* bf16 is the upper half of an IEEE binary32 word: widen and reinterpret. */
double dito_bf16_to_f64(uint16_t h)
{
    uint32_t w = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/*
 * Round an fp64 value to the nearest bf16 (ties to even) in ONE step.
 * bf16 keeps 8 significant bits, the binary32 exponent range, subnormals down
 * to 2^-133 and overflows to infinity at (2 - 2^-8) * 2^127 and above.
 * Method: find the value's binade [2^(e-1), 2^e), take the bf16 spacing q of
 * that binade (2^(e-8); 2^-133 below the normal range), round a/q to an
 * integer with rint() in the default ties-to-even mode (a/q is an exact
 * power-of-two scaling), scale back and re-encode.  No intermediate rounding
 * to binary32 happens, so there is no double rounding.
 */
uint16_t dito_f64_to_bf16(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v)) return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(v);
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0) return sign;
    int e;
    (void)frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
    int qexp = (e - 1 >= -126) ? (e - 8) : -133;
    double k = ldexp(a, -qexp);         /* exact */
    double r = rint(k);                 /* ties to even */
    double res = ldexp(r, qexp);        /* exact */
    if (res >= 0x1p128) return (uint16_t)(sign | 0x7F80u);
    if (res == 0.0) return sign;
    float f = (float)res;               /* exact: <= 8 significant bits */
    uint32_t w;
    memcpy(&w, &f, sizeof w);
    return (uint16_t)(sign | (uint16_t)(w >> 16));
}

void dito_round_bf16(const double* v, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = dito_f64_to_bf16(v[i]);
}

void dito_widen_bf16(const uint16_t* h, double* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = dito_bf16_to_f64(h[i]);
}

/* --------------------------------------------------- AdaLN modulation (a1) */

/*
 * Non-affine LayerNorm of one row of D values, then the AdaLN modulation
 *     y_d = (x_d - mu) / sqrt(var + eps) * (1 + scale_d) + shift_d
 * with mu the row mean and var the biased (divide by D) variance, computed in
 * two passes.  Readings: the "(1 + scale)" form (zero modulation must give a
 * plain LayerNorm), eps inside the square root.  [REPORT] "atualização do
 * AdaLN"; [H3BASE] modulation vectors come precomputed from the AdaLN branch.
 */
static void adaln_row(const double* x, const double* shift, const double* scale,
                      int D, double eps, double* y)
{
    double mu = 0.0;
    for (int d = 0; d < D; ++d) mu += x[d];
    mu /= (double)D;
    double var = 0.0;
    for (int d = 0; d < D; ++d) var += (x[d] - mu) * (x[d] - mu);
    var /= (double)D;
    double inv = 1.0 / sqrt(var + eps);
    for (int d = 0; d < D; ++d)
        y[d] = (x[d] - mu) * inv * (1.0 + scale[d]) + shift[d];
}

/*
 * x: [B,N,D] bf16 bits.  shift, scale: fp64, sample b's vector starts at
 * b*mod_batch_stride.  y: [B,N,D] fp64 (unrounded).  work: D doubles.
 */
int dito_adaln_modulate(const uint16_t* x, const double* shift, const double* scale,
                        int64_t mod_batch_stride, int B, int64_t N, int D, double eps,
                        double* y, double* work)
{
    if (D <= 0 || B < 0 || N < 0) return -2;
    for (int b = 0; b < B; ++b)
        for (int64_t n = 0; n < N; ++n) {
            int64_t row = ((int64_t)b * N + n) * D;
            for (int d = 0; d < D; ++d) work[d] = dito_bf16_to_f64(x[row + d]);
            adaln_row(work, shift + b * mod_batch_stride, scale + b * mod_batch_stride,
                      D, eps, y + row);
        }
    return 0;
}

/* ------------------------------------- gated residual fused with AdaLN (a2) */

/*
 * x' = bf16(x + gate * r)  (one rounding, stored: it is the new residual
 * stream), then y = AdaLN(x') as in a1 on the ROUNDED x'.  Reading: the fused
 * operator must give what the unfused chain gives ([REPORT]: the fused layer
 * "does not change any calculation result"), and the unfused chain stores x'
 * in bf16 before the next LayerNorm reads it.  Plain (not tanh) gate.
 */
int dito_gated_residual_adaln(const uint16_t* x, const uint16_t* r,
                              const double* gate, const double* shift, const double* scale,
                              int64_t mod_batch_stride, int B, int64_t N, int D, double eps,
                              uint16_t* x_out, double* y, double* work)
{
    if (D <= 0 || B < 0 || N < 0) return -2;
    for (int b = 0; b < B; ++b) {
        const double* g = gate + b * mod_batch_stride;
        for (int64_t n = 0; n < N; ++n) {
            int64_t row = ((int64_t)b * N + n) * D;
            for (int d = 0; d < D; ++d) {
                double v = dito_bf16_to_f64(x[row + d]) + g[d] * dito_bf16_to_f64(r[row + d]);
                uint16_t h = dito_f64_to_bf16(v);
                x_out[row + d] = h;
                work[d] = dito_bf16_to_f64(h);
            }
            adaln_row(work, shift + b * mod_batch_stride, scale + b * mod_batch_stride,
                      D, eps, y + row);
        }
    }
    return 0;
}

/* ---------------------------------------- per-token modulation sets (a1, a2) */

/*
 * The two AdaLN operators with the modulation chosen per token instead of
 * per sample: token (b, n) takes set s = set_index[b*N + n] (0 <= s <
 * n_sets) of its sample, whose vectors start at b*mod_batch_stride +
 * s*mod_set_stride of shift, scale (and gate).  Everything else is the
 * operator above, row by row.  Reading: [H3BASE], section "Phần nào đã được
 * phát hành?", names first/last-frame conditioned generation (FL2VA); the
 * tokens of conditioning frames then carry modulation of their own.  The
 * pages say no more, so any assignment of tokens to a few sets is allowed.
 * An index >= n_sets returns -3 (nothing else checked).
 */
int dito_adaln_modulate_tok(const uint16_t* x, const double* shift, const double* scale,
                            int64_t mod_batch_stride, int64_t mod_set_stride,
                            const uint8_t* set_index, int n_sets, int B, int64_t N, int D,
                            double eps, double* y, double* work)
{
    if (D <= 0 || B < 0 || N < 0 || n_sets < 1) return -2;
    for (int b = 0; b < B; ++b)
        for (int64_t n = 0; n < N; ++n) {
            int64_t tok = (int64_t)b * N + n;
            int set = set_index[tok];
            if (set >= n_sets) return -3;
            int64_t m = b * mod_batch_stride + set * mod_set_stride;
            for (int d = 0; d < D; ++d) work[d] = dito_bf16_to_f64(x[tok * D + d]);
            adaln_row(work, shift + m, scale + m, D, eps, y + tok * D);
        }
    return 0;
}

int dito_gated_residual_adaln_tok(const uint16_t* x, const uint16_t* r, const double* gate,
                                  const double* shift, const double* scale,
                                  int64_t mod_batch_stride, int64_t mod_set_stride,
                                  const uint8_t* set_index, int n_sets, int B, int64_t N, int D,
                                  double eps, uint16_t* x_out, double* y, double* work)
{
    if (D <= 0 || B < 0 || N < 0 || n_sets < 1) return -2;
    for (int b = 0; b < B; ++b)
        for (int64_t n = 0; n < N; ++n) {
            int64_t tok = (int64_t)b * N + n;
            int sg = set_index[tok];
            if (sg >= n_sets) return -3;
            int64_t mg = b * mod_batch_stride + sg * mod_set_stride;
            for (int d = 0; d < D; ++d) {
                double v = dito_bf16_to_f64(x[tok * D + d]) +
                           gate[mg + d] * dito_bf16_to_f64(r[tok * D + d]);
                uint16_t h = dito_f64_to_bf16(v);
                x_out[tok * D + d] = h;
                work[d] = dito_bf16_to_f64(h);
            }
            adaln_row(work, shift + mg, scale + mg, D, eps, y + tok * D);
        }
    return 0;
}

/* ------------------------------------------------------------ SwiGLU (a3) */

/*
 * in: [M, 2F]; out[m, j] = silu(a) * b with a = in[m, j] (first half, the
 * gate) and b = in[m, F + j] (second half), silu(a) = a / (1 + exp(-a)).
 * [REPORT] "a ativação SwiGLU".  Reading: first half is the gate.
 */
int dito_swiglu(const uint16_t* in, int64_t M, int F, double* out)
{
    if (F <= 0 || M < 0) return -2;
    for (int64_t m = 0; m < M; ++m)
        for (int j = 0; j < F; ++j) {
            double a = dito_bf16_to_f64(in[m * 2 * (int64_t)F + j]);
            double b = dito_bf16_to_f64(in[m * 2 * (int64_t)F + F + j]);
            double silu = a / (1.0 + exp(-a));
            out[m * (int64_t)F + j] = silu * b;
        }
    return 0;
}

/* ------------------------------------------ QK RMSNorm + 3D RoPE (a4) */

/*
 * Row-major flattening of a (T, Hg, Wg) latent grid: token g sits at
 * t = g / (Hg*Wg), h = (g / Wg) % Hg, w = g % Wg.  Tokens n = 0..N-1 of each
 * sample get the positions of global tokens offset + n.
 */
int dito_grid_positions(int T, int Hg, int Wg, int64_t offset, int64_t N, int32_t* pos)
{
    if (T <= 0 || Hg <= 0 || Wg <= 0 || offset < 0) return -2;
    if (offset + N > (int64_t)T * Hg * Wg) return -2;
    for (int64_t n = 0; n < N; ++n) {
        int64_t g = offset + n;
        pos[3 * n + 0] = (int32_t)(g / ((int64_t)Hg * Wg));
        pos[3 * n + 1] = (int32_t)((g / Wg) % Hg);
        pos[3 * n + 2] = (int32_t)(g % Wg);
    }
    return 0;
}

/*
 * One head of hd values: RMSNorm with weight w, then 3D rotary embedding.
 *   u_j = x_j / sqrt(mean_j(x_j^2) + eps) * w_j
 * The hd/2 rotation pairs are (u_{2p}, u_{2p+1}) (interleaved reading).  Pairs
 * [0, pt) follow the temporal position, [pt, pt+ph) the height position and
 * [pt+ph, hd/2) the width position.  Inside an axis with P pairs, local pair i
 * turns by phi = pos_axis * theta^(-2i / (2P)):
 *   (u0, u1) -> (u0 cos phi - u1 sin phi,  u0 sin phi + u1 cos phi).
 * [REPORT] "QK RMSNorm com 3D RoPE"; [CEVIU] "QK RMSNorm e 3D RoPE".
 */
static void qk_head(const double* x, const double* w, int hd, const int32_t* p3,
                    int pt, int ph, int pw, double theta, double eps, double* out)
{
    double ms = 0.0;
    for (int j = 0; j < hd; ++j) ms += x[j] * x[j];
    ms /= (double)hd;
    double inv = 1.0 / sqrt(ms + eps);
    for (int p = 0; p < hd / 2; ++p) {
        int axis, i, P;
        if (p < pt)           { axis = 0; i = p;           P = pt; }
        else if (p < pt + ph) { axis = 1; i = p - pt;      P = ph; }
        else                  { axis = 2; i = p - pt - ph; P = pw; }
        double omega = pow(theta, -2.0 * (double)i / (2.0 * (double)P));
        double phi = (double)p3[axis] * omega;
        double u0 = x[2 * p] * inv * w[2 * p];
        double u1 = x[2 * p + 1] * inv * w[2 * p + 1];
        out[2 * p]     = u0 * cos(phi) - u1 * sin(phi);
        out[2 * p + 1] = u0 * sin(phi) + u1 * cos(phi);
    }
}

/*
 * x: rows of B*N tokens, token i's H*hd values start at x + i*row_stride.
 * w: [hd] fp64.  pos: [B*N, 3] int32 (t, h, w) per token.  out: [B*N, H*hd]
 * fp64, dense.  work: hd doubles.  Requires pt+ph+pw == hd/2, each > 0.
 */
int dito_qk_rmsnorm_rope3d(const uint16_t* x, int64_t row_stride, const double* w,
                           int B, int64_t N, int H, int hd, const int32_t* pos,
                           int pt, int ph, int pw, double theta, double eps,
                           double* out, double* work)
{
    if (hd <= 0 || hd % 2 || pt <= 0 || ph <= 0 || pw <= 0 || pt + ph + pw != hd / 2)
        return -2;
    if (row_stride < (int64_t)H * hd) return -2;
    int64_t rows = (int64_t)B * N;
    for (int64_t i = 0; i < rows; ++i)
        for (int h = 0; h < H; ++h) {
            const uint16_t* src = x + i * row_stride + (int64_t)h * hd;
            for (int j = 0; j < hd; ++j) work[j] = dito_bf16_to_f64(src[j]);
            qk_head(work, w, hd, pos + 3 * i, pt, ph, pw, theta, eps,
                    out + i * (int64_t)H * hd + (int64_t)h * hd);
        }
    return 0;
}

/*
 * The same operator with two options the pages leave open.
 *   layout 0: rotation pairs (u_{2p}, u_{2p+1})        (interleaved)
 *   layout 1: rotation pairs (u_p, u_{p + hd/2})        (rotate-half)
 *   norm 0:   RMS over each head's hd values, weight w[hd]
 *   norm 1:   RMS over the token's whole row of H*hd values, weight w[H*hd]
 * Pair p's axis, frequency and angle are as in dito_qk_rmsnorm_rope3d.
 * work: H*hd doubles.
 */
int dito_qk_rmsnorm_rope3d_ex(const uint16_t* x, int64_t row_stride, const double* w,
                              int B, int64_t N, int H, int hd, const int32_t* pos,
                              int pt, int ph, int pw, double theta, double eps,
                              int layout, int norm, double* out, double* work)
{
    if (hd <= 0 || hd % 2 || pt <= 0 || ph <= 0 || pw <= 0 || pt + ph + pw != hd / 2)
        return -2;
    if (row_stride < (int64_t)H * hd || (layout != 0 && layout != 1) || (norm != 0 && norm != 1))
        return -2;
    int64_t rows = (int64_t)B * N;
    int width = H * hd;
    for (int64_t r = 0; r < rows; ++r) {
        for (int j = 0; j < width; ++j) work[j] = dito_bf16_to_f64(x[r * row_stride + j]);
        double inv_row = 0.0;
        if (norm == 1) {
            double ms = 0.0;
            for (int j = 0; j < width; ++j) ms += work[j] * work[j];
            ms /= (double)width;
            inv_row = 1.0 / sqrt(ms + eps);
        }
        const int32_t* p3 = pos + 3 * r;
        for (int h = 0; h < H; ++h) {
            const double* xh = work + (int64_t)h * hd;
            const double* wh = norm == 1 ? w + (int64_t)h * hd : w;
            double* oh = out + r * width + (int64_t)h * hd;
            double inv = inv_row;
            if (norm == 0) {
                double ms = 0.0;
                for (int j = 0; j < hd; ++j) ms += xh[j] * xh[j];
                ms /= (double)hd;
                inv = 1.0 / sqrt(ms + eps);
            }
            for (int q = 0; q < hd / 2; ++q) {
                int axis, i, P;
                if (q < pt)           { axis = 0; i = q;           P = pt; }
                else if (q < pt + ph) { axis = 1; i = q - pt;      P = ph; }
                else                  { axis = 2; i = q - pt - ph; P = pw; }
                double omega = pow(theta, -2.0 * (double)i / (2.0 * (double)P));
                double phi = (double)p3[axis] * omega;
                int a = layout == 0 ? 2 * q : q;
                int b = layout == 0 ? 2 * q + 1 : q + hd / 2;
                double u0 = xh[a] * inv * wh[a];
                double u1 = xh[b] * inv * wh[b];
                oh[a] = u0 * cos(phi) - u1 * sin(phi);
                oh[b] = u0 * sin(phi) + u1 * cos(phi);
            }
        }
    }
    return 0;
}

/* ----------------------------------------- Cache-DiT residual check (a5) */

/*
 * Sums over `count` elements: num = sum |cur - prev|, den = sum |prev|.
 * [REPORT] Cache-DiT paragraph: a residual-difference threshold decides reuse.
 */
void dito_cachedit_sums(const uint16_t* prev, const uint16_t* cur, int64_t count,
                        double* num, double* den)
{
    double s_num = 0.0, s_den = 0.0;
    for (int64_t i = 0; i < count; ++i) {
        double p = dito_bf16_to_f64(prev[i]);
        double c = dito_bf16_to_f64(cur[i]);
        s_num += fabs(c - p);
        s_den += fabs(p);
    }
    *num = s_num;
    *den = s_den;
}

/*
 * rel = num / den, with 0/0 read as 0 (identical residuals are reusable) and
 * x/0 as +inf; reuse = rel < threshold (strict).  Returns reuse (0 or 1).
 */
int dito_cachedit_decide(double num, double den, double threshold, double* rel)
{
    double q;
    if (den == 0.0) q = (num == 0.0) ? 0.0 : INFINITY;
    else q = num / den;
    *rel = q;
    return q < threshold ? 1 : 0;
}

/*
 * prev, cur: [B,N,D] bf16.  Per sample b: rel[b] = relative L1 difference of
 * its N*D elements, reuse[b] = rel[b] < threshold.
 */
int dito_cachedit_residual_diff(const uint16_t* prev, const uint16_t* cur,
                                int B, int64_t N, int D, double threshold,
                                double* rel, uint8_t* reuse)
{
    if (B < 0 || N < 0 || D <= 0) return -2;
    for (int b = 0; b < B; ++b) {
        double num, den;
        int64_t off = (int64_t)b * N * D;
        dito_cachedit_sums(prev + off, cur + off, N * (int64_t)D, &num, &den);
        reuse[b] = (uint8_t)dito_cachedit_decide(num, den, threshold, &rel[b]);
    }
    return 0;
}

/* --------------------------- Cache-DiT residual cache across steps (f3) */

/*
 * [REPORT], section "Só com três camadas de aceleração somadas chega-se a 6
 * vezes": Cache-DiT reuses results cached between neighbouring denoising
 * steps.  Reading: the cached result is the residual the skipped blocks add
 * to the hidden state, R = after - before, stored in bf16 like the hidden
 * state; a reusing step adds it back, out = h + R.  Each is the exact
 * rational value rounded once to bf16: fp64 holds the sum or difference of
 * two bf16 values exactly unless their exponents differ by more than 44,
 * and then the smaller one lies far below half a bf16 ulp of the larger, so
 * the single rounding of the fp64 value still gives the nearest bf16.
 */
void dito_residual_store(const uint16_t* before, const uint16_t* after, int64_t n,
                         uint16_t* residual)
{
    for (int64_t i = 0; i < n; ++i)
        residual[i] = dito_f64_to_bf16(dito_bf16_to_f64(after[i]) - dito_bf16_to_f64(before[i]));
}

void dito_residual_apply(const uint16_t* h, const uint16_t* residual, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = dito_f64_to_bf16(dito_bf16_to_f64(h[i]) + dito_bf16_to_f64(residual[i]));
}

/* ------------------------ SwiGLU fused into the up-projection GEMM (f2) */

/*
 * out[m, j] = silu(g) * u with
 *     g = sum_k x[m, k] * w[j, k],   u = sum_k x[m, k] * w[F + j, k]
 * x: [M, K] bf16 (the block's normalised input), w: [2F, K] bf16 (the
 * up-projection weight, one row per output feature: rows [0, F) the gate
 * half, rows [F, 2F) the linear half, the order read for a3).  [REPORT]
 * names SwiGLU among the fused operators and [CEVIU] says fusion cuts
 * memory traffic; fusing it into the GEMM that produces its input is the
 * reading here, with no rounding between the product and the activation.
 * Dot products in fp64 in the order k = 0 .. K-1.  rows (n_rows entries)
 * picks the rows of x to compute, or NULL for all M; out is [n_rows, F].
 * g_abs / u_abs (optional) receive sum_k |x w| for each output, from which
 * a test bounds the error of a lower-precision accumulation.
 */
int dito_swiglu_gemm(const uint16_t* x, const uint16_t* w, int64_t M, int K, int F,
                     const int64_t* rows, int64_t n_rows, double* out, double* g_abs,
                     double* u_abs)
{
    if (M < 0 || K <= 0 || F <= 0 || n_rows < 0) return -2;
    if (!rows) n_rows = M;
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t m = rows ? rows[r] : r;
        if (m < 0 || m >= M) return -3;
        const uint16_t* xr = x + m * (int64_t)K;
        for (int j = 0; j < F; ++j) {
            const uint16_t* wg = w + (int64_t)j * K;
            const uint16_t* wu = w + ((int64_t)F + j) * K;
            double g = 0.0, u = 0.0, ga = 0.0, ua = 0.0;
            for (int k = 0; k < K; ++k) {
                double xv = dito_bf16_to_f64(xr[k]);
                double tg = xv * dito_bf16_to_f64(wg[k]);
                double tu = xv * dito_bf16_to_f64(wu[k]);
                g += tg;
                u += tu;
                ga += fabs(tg);
                ua += fabs(tu);
            }
            out[r * F + j] = g / (1.0 + exp(-g)) * u;
            if (g_abs) g_abs[r * F + j] = ga;
            if (u_abs) u_abs[r * F + j] = ua;
        }
    }
    return 0;
}

/* ---------------- gated residual fused into the down-projection GEMM (f2) */

/*
 * x_out[m, n] = bf16(x[m, n] + gate_b[n] * sum_k h[m, k] * w[n, k])
 * h: [M, K] bf16 (the block's MLP activations), w: [D, K] bf16 (the
 * projection weight, one row per output feature), x: [M, D] bf16 (the
 * residual stream), gate: [B, D] (sample b = m / N of token row m, vectors
 * mod_batch_stride apart).  This is a2's residual update with its branch
 * r = h w^T taken straight from the product: [REPORT] names the gated
 * residual among the fused operators, and the fused form must give what the
 * unfused chain gives up to the rounding of r, which the fusion removes.
 * The dot product is summed in fp64 in the order k = 0 .. K-1 (the products
 * of two bf16 values are exact), then x + gate * dot in fp64 is rounded once
 * to bf16.  rows (n_rows entries) picks the token rows, or NULL for all M;
 * x_out is [n_rows, D] and dot (optional) receives the fp64 dot products,
 * abs_dot (optional) sum_k |h w| for each output.
 */
int dito_gemm_gated_residual(const uint16_t* h, const uint16_t* w, const uint16_t* x,
                             const double* gate, int64_t mod_batch_stride, int64_t M,
                             int64_t N, int K, int D, const int64_t* rows, int64_t n_rows,
                             uint16_t* x_out, double* dot, double* abs_dot)
{
    if (M < 0 || N <= 0 || K <= 0 || D <= 0 || n_rows < 0 || M % N) return -2;
    if (!rows) n_rows = M;
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t m = rows ? rows[r] : r;
        if (m < 0 || m >= M) return -3;
        const double* g = gate + (m / N) * mod_batch_stride;
        const uint16_t* hr = h + m * (int64_t)K;
        for (int n = 0; n < D; ++n) {
            const uint16_t* wn = w + (int64_t)n * K;
            double s = 0.0, a = 0.0;
            for (int k = 0; k < K; ++k) {
                double t = dito_bf16_to_f64(hr[k]) * dito_bf16_to_f64(wn[k]);
                s += t;
                a += fabs(t);
            }
            x_out[r * D + n] = dito_f64_to_bf16(dito_bf16_to_f64(x[m * (int64_t)D + n]) + g[n] * s);
            if (dot) dot[r * D + n] = s;
            if (abs_dot) abs_dot[r * D + n] = a;
        }
    }
    return 0;
}

/* -------------------------------------------- SubBlock sparse router (f4) */

/*
 * [REPORT], section "Só com três camadas de aceleração somadas chega-se a 6
 * vezes": a block-sparse router cuts, from the 10th denoising step on, the
 * KV blocks that take part in attention, at sparsity 0.75 or 0.80.  The pages
 * give no rule; the reading here is the plainest one:
 *   - the N tokens of a sample are cut into blocks of `block` consecutive
 *     tokens (the last one may be shorter): n_blocks = ceil(N / block);
 *   - per head, a block's summary is the mean of its rows (q for query
 *     blocks, k for key blocks);
 *   - query block i scores key block j by the dot product of the summaries;
 *   - each query block keeps the n_keep key blocks with the highest scores
 *     (ties: the lower block index first), n_keep = ceil((1 - sparsity) *
 *     n_blocks) and at least 1; the kept indices are written in increasing
 *     order.
 * q, k: rows of B*N tokens, `row_stride` elements apart, each H heads of hd
 * values (head h at offset h*hd).  kept: [B, H, n_blocks, n_keep] int32.
 * scores (optional): [B, H, n_blocks, n_blocks] fp64.  work: 2*n_blocks*hd
 * + 2*n_blocks doubles.  Returns n_keep, or a negative code.
 */
int dito_subblock_keep_count(int64_t n_blocks, double sparsity)
{
    if (n_blocks <= 0 || !(sparsity >= 0.0) || !(sparsity < 1.0)) return -2;
    double want = ceil((1.0 - sparsity) * (double)n_blocks - 1e-9);
    int64_t keep = (int64_t)want;
    if (keep < 1) keep = 1;
    if (keep > n_blocks) keep = n_blocks;
    return (int)keep;
}

int dito_subblock_router(const uint16_t* q, const uint16_t* k, int64_t row_stride, int B,
                         int64_t N, int H, int hd, int block, double sparsity, int32_t* kept,
                         double* scores, double* work)
{
    if (B < 0 || N <= 0 || H < 1 || hd < 1 || block < 1 || row_stride < (int64_t)H * hd)
        return -2;
    int64_t nb = (N + block - 1) / block;
    int n_keep = dito_subblock_keep_count(nb, sparsity);
    if (n_keep < 0) return n_keep;
    double* qm = work;                 /* [nb, hd] */
    double* km = qm + nb * hd;         /* [nb, hd] */
    double* sc = km + nb * hd;         /* [nb] */
    int64_t* order = (int64_t*)(sc + nb);   /* [nb], fits in the next nb doubles */
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            /* block means */
            for (int64_t j = 0; j < nb; ++j) {
                int64_t t0 = j * block, t1 = t0 + block < N ? t0 + block : N;
                for (int d = 0; d < hd; ++d) {
                    double sq = 0.0, sk = 0.0;
                    for (int64_t t = t0; t < t1; ++t) {
                        int64_t off = ((int64_t)b * N + t) * row_stride + (int64_t)h * hd + d;
                        sq += dito_bf16_to_f64(q[off]);
                        sk += dito_bf16_to_f64(k[off]);
                    }
                    qm[j * hd + d] = sq / (double)(t1 - t0);
                    km[j * hd + d] = sk / (double)(t1 - t0);
                }
            }
            for (int64_t i = 0; i < nb; ++i) {
                for (int64_t j = 0; j < nb; ++j) {
                    double s = 0.0;
                    for (int d = 0; d < hd; ++d) s += qm[i * hd + d] * km[j * hd + d];
                    sc[j] = s;
                    order[j] = j;
                    if (scores) scores[(((int64_t)b * H + h) * nb + i) * nb + j] = s;
                }
                /* selection: repeatedly take the best remaining block */
                int32_t* out = kept + (((int64_t)b * H + h) * nb + i) * n_keep;
                for (int r = 0; r < n_keep; ++r) {
                    int64_t best = r;
                    for (int64_t c = r + 1; c < nb; ++c) {
                        int64_t oc = order[c], ob = order[best];
                        if (sc[oc] > sc[ob] || (sc[oc] == sc[ob] && oc < ob)) best = c;
                    }
                    int64_t tmp = order[r];
                    order[r] = order[best];
                    order[best] = tmp;
                }
                /* the kept blocks in increasing order */
                for (int r = 0; r < n_keep; ++r) out[r] = (int32_t)order[r];
                for (int r = 1; r < n_keep; ++r)
                    for (int c = r; c > 0 && out[c - 1] > out[c]; --c) {
                        int32_t t = out[c];
                        out[c] = out[c - 1];
                        out[c - 1] = t;
                    }
            }
        }
    return n_keep;
}

/*
 * Block-sparse attention over the router's kept key blocks (f4): for token t
 * of query block i, head h,
 *     out[t, h] = sum_u softmax_u(scale * q[t, h] . k[u, h]) v[u, h]
 * with u over the tokens of the kept key blocks kept[b, h, i, 0..n_keep) of
 * the same sample (the last block may be shorter).  Non-causal.  fp64: the
 * scores, the max-shifted exponentials, the normaliser and the weighted sum.
 * q, k, v rows `row_stride` apart, H heads of hd.  rows (n_rows entries)
 * picks the query rows (b*N + t) to compute, or NULL for all B*N; out:
 * [n_rows, H*hd] fp64.  work: the scores of one query token (n_keep * block
 * doubles).
 */
int dito_block_sparse_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                int64_t row_stride, int B, int64_t N, int H, int hd, int block,
                                const int32_t* kept, int n_keep, double scale,
                                const int64_t* rows, int64_t n_rows, double* out, double* work)
{
    if (B < 0 || N <= 0 || H < 1 || hd < 1 || block < 1 || n_keep < 1 || n_rows < 0 ||
        row_stride < (int64_t)H * hd)
        return -2;
    int64_t nb = (N + block - 1) / block;
    if (!rows) n_rows = (int64_t)B * N;
    for (int64_t r_out = 0; r_out < n_rows; ++r_out)
        for (int h = 0; h < H; ++h) {
            int64_t row = rows ? rows[r_out] : r_out;
            if (row < 0 || row >= (int64_t)B * N) return -3;
            int b = (int)(row / N);
            int64_t t = row - (int64_t)b * N;
            int64_t i = t / block;
            const int32_t* kb = kept + (((int64_t)b * H + h) * nb + i) * n_keep;
            const uint16_t* qt = q + ((int64_t)b * N + t) * row_stride + (int64_t)h * hd;
            int64_t n = 0;
            double mx = -INFINITY;
            for (int r = 0; r < n_keep; ++r) {
                int64_t j = kb[r];
                if (j < 0 || j >= nb) return -3;
                int64_t u1 = (j + 1) * block < N ? (j + 1) * block : N;
                for (int64_t u = j * block; u < u1; ++u) {
                    const uint16_t* ku = k + ((int64_t)b * N + u) * row_stride + (int64_t)h * hd;
                    double s = 0.0;
                    for (int d = 0; d < hd; ++d)
                        s += dito_bf16_to_f64(qt[d]) * dito_bf16_to_f64(ku[d]);
                    s *= scale;
                    work[n++] = s;
                    if (s > mx) mx = s;
                }
            }
            double l = 0.0;
            for (int64_t e = 0; e < n; ++e) {
                work[e] = exp(work[e] - mx);
                l += work[e];
            }
            double* ot = out + r_out * ((int64_t)H * hd) + (int64_t)h * hd;
            for (int d = 0; d < hd; ++d) ot[d] = 0.0;
            n = 0;
            for (int r = 0; r < n_keep; ++r) {
                int64_t j = kb[r];
                int64_t u1 = (j + 1) * block < N ? (j + 1) * block : N;
                for (int64_t u = j * block; u < u1; ++u) {
                    const uint16_t* vu = v + ((int64_t)b * N + u) * row_stride + (int64_t)h * hd;
                    double pw = work[n++] / l;
                    for (int d = 0; d < hd; ++d) ot[d] += pw * dito_bf16_to_f64(vu[d]);
                }
            }
        }
    return 0;
}
