/*
 * qknr oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow CPU statement, in fp64, of what the fused Q/K RMSNorm + rotary
 * embedding transform computes. Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load it. The product library never calls it,
 * and the two share no code: no header, helper, table or constant.
 *
 * Sources (web pages, cited by title and section):
 *   [T] "vllm_omni.diffusion.layers.fused_qk_norm_rope" (vLLM-Omni API docs):
 *       the module description with its public-contract bullets, and the
 *       signature of fused_qk_norm_rope.
 *   [F] "flashinfer.norm.fused_qk_rmsnorm_rope" (FlashInfer API docs): the
 *       summary paragraph, "Parameters" and "Returns".
 *   [U] "vllm_omni.diffusion.models.sana_wm.ucpe" (vLLM-Omni API docs):
 *       cam_prep_func, its description, "Parameters" and "Returns".
 *
 * The pages give signatures and prose but print no formula. Where they leave a
 * step open this file takes the plainest reading and says so next to the step:
 *   R1  RMSNorm is y = x / sqrt(mean(x^2) + eps) * w (plain weight, not 1 + w).
 *   R2  Order: normalise, multiply by the weight (indexed by the channel before
 *       rotation), then rotate.
 *   R3  One rounding at the end: everything in fp64, then one rounding to the
 *       output type ([T]: no normalised or rotated intermediate is kept).
 *   R4  Rotation of a pair (a, b) by angle theta is the complex product
 *       (a + i b) e^{i theta}: a' = a cos - b sin, b' = b cos + a sin.
 *   R5  3D channel groups sit in the order frame, height, width (the order of
 *       the num_*_channels parameters in [F]).
 *   R6  3D frequency of pair i inside an axis group of C channels is
 *       base^(-2i/C), i < C/2; positions are integer patch coordinates from 0.
 *   R7  Token t of a 3D input has s = (t + pos_offset) mod (ppf*pph*ppw) and
 *       row-major patch coordinates f = s / (pph*ppw), h = (s / ppw) mod pph,
 *       w = s mod ppw; a batch flattened into tokens repeats the grid.
 *   R8  NeoX pairs in the 3D form are (j, j + D/2) over the whole head, with
 *       pair j taking the frequency of pair slot j in the frame/height/width
 *       order (the 3D analogue of the half-split pairs of [T]). The other
 *       reading, NeoX inside each axis group, is kept behind a flag
 *       (neox_per_axis); the library offers it behind the same flag, off by
 *       default. PARITY UNPINNED between the two readings: the pages cannot
 *       decide it (each is pinned to its own textbook form).
 *   R9  FP8 output is E4M3(value * scale): the quantisation scale multiplies.
 *       PARITY UNPINNED against the reading that divides.
 *   R10 E4M3 is the OCP E4M3FN format (bias 7, largest finite 448, no
 *       infinities) with round-to-nearest-even and saturation to +-448.
 *   R11 With is_qk_norm off, Q/K are only rotated (weights and eps unused).
 *   R12 Table form: channels at and beyond rotary_dim are normalised but not
 *       rotated.
 *   R13 Table form activations may be bf16 or IEEE binary16 ([T]: the table
 *       has the activation type or is float32, so the activation type is
 *       not fixed to bf16); weights share the activation type, outputs are
 *       rounded once to it.
 *
 * The camera prep of [U] lists its steps (ReLU, the K scale, the ray
 * projection, RoPE) and its shapes but no formula. Readings taken:
 *   U1  ReLU is the feature map of Q and K and comes first; V is not passed
 *       through it ([U] takes V un-normalised and names no V step but the
 *       projection).
 *   U2  The K scale multiplies K alone, after its ReLU.
 *   U3  The ray projection splits each head's channels into blocks of four
 *       consecutive channels and multiplies every block, as a column vector,
 *       by the token's 4x4 matrix read row by row: y_i = sum_j M[i][j] x_j.
 *       Q takes proj_q; K and V take proj_kv ([U] gives proj_kv for both).
 *   U4  RoPE follows the projection, on Q and K only, with adjacent pairs
 *       (2j, 2j+1) ([U]: the tables are for interleaved pairs and have D/2
 *       columns, so they cover the whole head), column j of the token's row of rope_cos
 *       and rope_sin, and the rotation of R4. V is not rotated, as in the
 *       other two contracts.
 *   U5  Outputs are laid out [B, H, D, N] ([U], "Returns"): the value for
 *       batch b, token n, head h, channel d is stored at [b][h][d][n], rounded
 *       once to the activation type (bf16 or binary16, as R13). Projection
 *       matrices and RoPE tables are float32, used as stored.
 *   U6  inflation_sq [B, H, N] is the factor by which the ray projection
 *       multiplies the squared norm of the scaled key: |M_kv k'|^2 / |k'|^2,
 *       k' = k_scale * ReLU(k) of that token and head (RoPE keeps the norm,
 *       so before or after the rotation is the same), and 1 where k' = 0.
 *       PARITY UNPINNED: [U] names this output but does not define it; the
 *       same ratio for Q is the other plain reading.
 *
 * Threads: the per-token loops run under OpenMP when it is enabled; every
 * token is computed independently, so the results do not depend on the
 * number of threads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

/* Round a non-negative value to the nearest integer, ties to the even one. */
static double round_half_even(double n)
{
    double fl = floor(n);
    double d = n - fl; /* exact: n carries at most 53 significant bits */
    if (d > 0.5) return fl + 1.0;
    if (d < 0.5) return fl;
    return fl + fmod(fl, 2.0);
}

/* Exponent of the leading bit: 2^e <= a < 2^(e+1), for a > 0. */
static int leading_exponent(double a)
{
    int e2;
    frexp(a, &e2); /* a = m 2^e2 with m in [0.5, 1) */
    return e2 - 1;
}

/* bfloat16 value of a 16-bit pattern, exactly (sign, 8 exponent bits with
 * bias 127, 7 fraction bits: the upper half of an IEEE binary32). */
double qknr_oracle_bf16_to_double(uint16_t b)
{
    uint32_t bits = (uint32_t)b << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* One round-to-nearest-even rounding of x to bfloat16 (8 significant bits,
 * normal exponents -126..127, subnormal spacing 2^-133; overflow gives inf). */
uint16_t qknr_oracle_bf16_from_double(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(x);
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0) return sign;
    int e = leading_exponent(a);
    if (e < -126) e = -126;
    double quantum = ldexp(1.0, e - 7);
    double v = round_half_even(a / quantum) * quantum;
    if (v >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
    /* v has at most 8 significant bits and lies in binary32 range: exact. */
    float f = (float)v;
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(sign | ((bits >> 16) & 0x7FFFu));
}

/* E4M3FN value of an 8-bit pattern (sign, 4 exponent bits with bias 7, 3
 * fraction bits; exponent 0 is subnormal m 2^-9; 0x7F/0xFF are NaN). */
double qknr_oracle_e4m3_to_double(uint8_t b)
{
    double s = (b & 0x80u) ? -1.0 : 1.0;
    int e = (b >> 3) & 0xF;
    int m = b & 0x7;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) return s * ldexp((double)m, -9);
    return s * ldexp(1.0 + m / 8.0, e - 7);
}

/* One round-to-nearest-even rounding of x to E4M3FN (4 significant bits,
 * normal exponents -6..8, subnormal spacing 2^-9), saturating to +-448. */
uint8_t qknr_oracle_e4m3_from_double(double x)
{
    uint8_t sign = signbit(x) ? 0x80u : 0u;
    if (isnan(x)) return 0x7Fu;
    double a = fabs(x);
    if (isinf(a)) return (uint8_t)(sign | 0x7Eu);
    if (a == 0.0) return sign;
    int e = leading_exponent(a);
    if (e < -6) e = -6;
    double quantum = ldexp(1.0, e - 3);
    double v = round_half_even(a / quantum) * quantum;
    if (v > 448.0) v = 448.0;
    if (v == 0.0) return sign;
    if (v < ldexp(1.0, -6)) return (uint8_t)(sign | (uint8_t)(v / ldexp(1.0, -9)));
    int E = leading_exponent(v);
    int m = (int)((v / ldexp(1.0, E) - 1.0) * 8.0);
    return (uint8_t)(sign | (uint8_t)(((E + 7) << 3) | m));
}

/* IEEE binary16 value of a 16-bit pattern, exactly (sign, 5 exponent bits with
 * bias 15, 10 fraction bits; exponent 0 is subnormal m 2^-24; 31 is inf/NaN). */
double qknr_oracle_f16_to_double(uint16_t b)
{
    double s = (b & 0x8000u) ? -1.0 : 1.0;
    int e = (b >> 10) & 0x1F;
    int m = b & 0x3FF;
    if (e == 31) return m ? NAN : s * INFINITY;
    if (e == 0) return s * ldexp((double)m, -24);
    return s * ldexp(1.0 + m / 1024.0, e - 15);
}

/* One round-to-nearest-even rounding of x to binary16 (11 significant bits,
 * normal exponents -14..15, subnormal spacing 2^-24; overflow gives inf). */
uint16_t qknr_oracle_f16_from_double(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return (uint16_t)(sign | 0x7E00u);
    double a = fabs(x);
    if (isinf(a)) return (uint16_t)(sign | 0x7C00u);
    if (a == 0.0) return sign;
    int e = leading_exponent(a);
    if (e < -14) e = -14;
    double quantum = ldexp(1.0, e - 10);
    double v = round_half_even(a / quantum) * quantum;
    if (v >= 65536.0) return (uint16_t)(sign | 0x7C00u);
    if (v == 0.0) return sign;
    if (v < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)(v / ldexp(1.0, -24)));
    int E = leading_exponent(v);
    int m = (int)((v / ldexp(1.0, E) - 1.0) * 1024.0);
    return (uint16_t)(sign | (uint16_t)(((E + 15) << 10) | m));
}

void qknr_oracle_f16_from_double_array(const double* x, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = qknr_oracle_f16_from_double(x[i]);
}

void qknr_oracle_bf16_from_double_array(const double* x, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = qknr_oracle_bf16_from_double(x[i]);
}

void qknr_oracle_e4m3_from_double_array(const double* x, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = qknr_oracle_e4m3_from_double(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Steps of the transform                                                   */
/* ------------------------------------------------------------------------ */

/* RMSNorm over n channels ([F] "across-heads RMSNorm": n = heads * head_dim;
 * [T]: n = head_dim per head). R1, R2. weight may be NULL (unit weight). */
void qknr_oracle_rmsnorm(const double* x, int64_t n, const double* weight, double eps, double* y)
{
    double ssq = 0.0;
    for (int64_t c = 0; c < n; ++c) ssq += x[c] * x[c];
    double r = 1.0 / sqrt(ssq / (double)n + eps);
    for (int64_t c = 0; c < n; ++c) y[c] = x[c] * r * (weight ? weight[c] : 1.0);
}

/* Rotate the listed channel pairs of one head (R4); other channels copy. */
void qknr_oracle_rotate(const double* y, int64_t n, int64_t npairs, const int32_t* pa,
                        const int32_t* pb, const double* cos_t, const double* sin_t,
                        double* out)
{
    for (int64_t c = 0; c < n; ++c) out[c] = y[c];
    for (int64_t j = 0; j < npairs; ++j) {
        double a = y[pa[j]], b = y[pb[j]];
        out[pa[j]] = a * cos_t[j] - b * sin_t[j];
        out[pb[j]] = b * cos_t[j] + a * sin_t[j];
    }
}

/* Pair map of the table form ([T] contract bullets): interleaved pairs are
 * (2j, 2j+1), half-split pairs are (j, j + rotary_dim/2), j < rotary_dim/2. */
void qknr_oracle_pairs_table(int32_t rotary_dim, int32_t interleaved, int32_t* pa, int32_t* pb)
{
    for (int32_t j = 0; j < rotary_dim / 2; ++j) {
        pa[j] = interleaved ? 2 * j : j;
        pb[j] = interleaved ? 2 * j + 1 : j + rotary_dim / 2;
    }
}

/* Pair map of the 3D form over a head of D = Cf + Ch + Cw channels.
 * interleave (non-NeoX): pair j = (2j, 2j+1). NeoX, R8: (j, j + D/2).
 * NeoX read per axis group (the alternative reading of R8): inside group a at
 * channel offset o_a with C_a channels, pair i = (o_a + i, o_a + i + C_a/2),
 * numbered j = o_a/2 + i so that it keeps pair slot j's frequency. */
void qknr_oracle_pairs_3d(int32_t Cf, int32_t Ch, int32_t Cw, int32_t interleave,
                          int32_t neox_per_axis, int32_t* pa, int32_t* pb)
{
    int32_t D = Cf + Ch + Cw;
    if (interleave) {
        qknr_oracle_pairs_table(D, 1, pa, pb);
    } else if (!neox_per_axis) {
        qknr_oracle_pairs_table(D, 0, pa, pb);
    } else {
        int32_t C[3] = {Cf, Ch, Cw};
        int32_t off = 0;
        for (int a = 0; a < 3; ++a) {
            for (int32_t i = 0; i < C[a] / 2; ++i) {
                pa[off / 2 + i] = off + i;
                pb[off / 2 + i] = off + i + C[a] / 2;
            }
            off += C[a];
        }
    }
}

/* Patch coordinates of token t (R7). */
void qknr_oracle_position_3d(int64_t t, int64_t pos_offset, int32_t ppf, int32_t pph,
                             int32_t ppw, int64_t* f, int64_t* h, int64_t* w)
{
    int64_t P = (int64_t)ppf * pph * ppw;
    int64_t s = (t + pos_offset) % P;
    *f = s / ((int64_t)pph * ppw);
    *h = (s / ppw) % pph;
    *w = s % ppw;
}

/* Rotation angle of every pair slot j < D/2 of a 3D token at patch (f, h, w)
 * ([F] num_frame/height/width_channels and base; R5, R6). Slots
 * [0, Cf/2) follow the frame axis, the next Ch/2 the height axis, the rest the
 * width axis; i counts slots from the start of the axis group. */
void qknr_oracle_angles_3d(int64_t f, int64_t h, int64_t w, int32_t Cf, int32_t Ch, int32_t Cw,
                           double base, double* theta)
{
    int32_t C[3] = {Cf, Ch, Cw};
    int64_t pos[3] = {f, h, w};
    int32_t j = 0;
    for (int a = 0; a < 3; ++a)
        for (int32_t i = 0; i < C[a] / 2; ++i)
            theta[j++] = (double)pos[a] * pow(base, -2.0 * i / C[a]);
}

/* ------------------------------------------------------------------------ */
/* Table form ([T] fused_qk_norm_rope)                                       */
/* ------------------------------------------------------------------------ */

/* Exact (pre-rounding) outputs of the table form for dense q [T, Hq, D] and
 * k [T, Hk, D] bf16 inputs, [D] bf16 weights and a [T, rotary_dim] table
 * holding cos(theta) in its first rotary_dim/2 columns and sin(theta) in the
 * rest, stored as fp32 (table_is_f32) or bf16. Outputs are fp64, same layout. */
/* 16-bit activation pattern -> value: bf16, or binary16 when act_is_f16. */
static double act_to_double(uint16_t b, int32_t act_is_f16)
{
    return act_is_f16 ? qknr_oracle_f16_to_double(b) : qknr_oracle_bf16_to_double(b);
}

int qknr_oracle_rope_table_exact_act(const uint16_t* q, const uint16_t* k,
                                     const uint16_t* q_weight, const uint16_t* k_weight,
                                     const void* table, int32_t table_is_f32, int32_t act_is_f16,
                                     int64_t num_tokens, int32_t heads_q, int32_t heads_k,
                                     int32_t head_dim, int32_t rotary_dim, double eps,
                                     int32_t interleaved, double* q_out, double* k_out)
{
    int32_t D = head_dim, R = rotary_dim;
    if (D <= 0 || D > 256 || R <= 0 || R > D || (R & 1)) return 1;
    double* wq = malloc(sizeof(double) * D);
    double* wk = malloc(sizeof(double) * D);
    int32_t* pa = malloc(sizeof(int32_t) * (R / 2));
    int32_t* pb = malloc(sizeof(int32_t) * (R / 2));
    for (int32_t d = 0; d < D; ++d) {
        wq[d] = act_to_double(q_weight[d], act_is_f16);
        wk[d] = act_to_double(k_weight[d], act_is_f16);
    }
    qknr_oracle_pairs_table(R, interleaved, pa, pb);

#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t t = 0; t < num_tokens; ++t) {
        double x[512], y[512], c[256], s[256];
        for (int32_t j = 0; j < R / 2; ++j) {
            if (table_is_f32) {
                const float* row = (const float*)table + t * R;
                c[j] = row[j];
                s[j] = row[R / 2 + j];
            } else {
                const uint16_t* row = (const uint16_t*)table + t * R;
                c[j] = act_to_double(row[j], act_is_f16);
                s[j] = act_to_double(row[R / 2 + j], act_is_f16);
            }
        }
        for (int pass = 0; pass < 2; ++pass) {
            int32_t H = pass ? heads_k : heads_q;
            const uint16_t* src = pass ? k : q;
            double* dst = pass ? k_out : q_out;
            const double* wt = pass ? wk : wq;
            for (int32_t hh = 0; hh < H; ++hh) {
                const uint16_t* xr = src + (t * H + hh) * D;
                for (int32_t d = 0; d < D; ++d) x[d] = act_to_double(xr[d], act_is_f16);
                qknr_oracle_rmsnorm(x, D, wt, eps, y);
                qknr_oracle_rotate(y, D, R / 2, pa, pb, c, s, dst + (t * H + hh) * D);
            }
        }
    }
    free(wq);
    free(wk);
    free(pa);
    free(pb);
    return 0;
}

int qknr_oracle_rope_table_exact(const uint16_t* q, const uint16_t* k, const uint16_t* q_weight,
                                 const uint16_t* k_weight, const void* table,
                                 int32_t table_is_f32, int64_t num_tokens, int32_t heads_q,
                                 int32_t heads_k, int32_t head_dim, int32_t rotary_dim,
                                 double eps, int32_t interleaved, double* q_out, double* k_out)
{
    return qknr_oracle_rope_table_exact_act(q, k, q_weight, k_weight, table, table_is_f32, 0,
                                            num_tokens, heads_q, heads_k, head_dim, rotary_dim,
                                            eps, interleaved, q_out, k_out);
}

/* Table form rounded to the activation type (R3): bf16, or binary16 when
 * act_is_f16 ([T] lets the table take the activation type or fp32, so the
 * activation type is not fixed to bf16; binary16 is the other 16-bit one). */
int qknr_oracle_rope_table_act(const uint16_t* q, const uint16_t* k, const uint16_t* q_weight,
                               const uint16_t* k_weight, const void* table, int32_t table_is_f32,
                               int32_t act_is_f16, int64_t num_tokens, int32_t heads_q,
                               int32_t heads_k, int32_t head_dim, int32_t rotary_dim, double eps,
                               int32_t interleaved, uint16_t* q_out, uint16_t* k_out)
{
    int64_t nq = num_tokens * heads_q * head_dim, nk = num_tokens * heads_k * head_dim;
    double* eq = malloc(sizeof(double) * (nq ? nq : 1));
    double* ek = malloc(sizeof(double) * (nk ? nk : 1));
    int rc = qknr_oracle_rope_table_exact_act(q, k, q_weight, k_weight, table, table_is_f32,
                                              act_is_f16, num_tokens, heads_q, heads_k, head_dim,
                                              rotary_dim, eps, interleaved, eq, ek);
    if (rc == 0 && act_is_f16) {
        qknr_oracle_f16_from_double_array(eq, q_out, nq);
        qknr_oracle_f16_from_double_array(ek, k_out, nk);
    } else if (rc == 0) {
        qknr_oracle_bf16_from_double_array(eq, q_out, nq);
        qknr_oracle_bf16_from_double_array(ek, k_out, nk);
    }
    free(eq);
    free(ek);
    return rc;
}

int qknr_oracle_rope_table(const uint16_t* q, const uint16_t* k, const uint16_t* q_weight,
                           const uint16_t* k_weight, const void* table, int32_t table_is_f32,
                           int64_t num_tokens, int32_t heads_q, int32_t heads_k,
                           int32_t head_dim, int32_t rotary_dim, double eps, int32_t interleaved,
                           uint16_t* q_out, uint16_t* k_out)
{
    return qknr_oracle_rope_table_act(q, k, q_weight, k_weight, table, table_is_f32, 0,
                                      num_tokens, heads_q, heads_k, head_dim, rotary_dim, eps,
                                      interleaved, q_out, k_out);
}

/* ------------------------------------------------------------------------ */
/* 3D form ([F] fused_qk_rmsnorm_rope)                                       */
/* ------------------------------------------------------------------------ */

/* Exact outputs of the 3D form for one token row of packed bf16 QKV
 * [(Hq + Hk + Hv) * D] (Q heads, then K heads, then V heads). q/k outputs are
 * the normalised, rotated values before any FP8 scale; v is copied. */
static void rope_3d_token(const uint16_t* row, const double* wq, const double* wk,
                          const double* theta, const int32_t* pa, const int32_t* pb,
                          int32_t Hq, int32_t Hk, int32_t Hv, int32_t D, double eps,
                          int32_t is_qk_norm, double* q_o, double* k_o, double* v_o,
                          double* x, double* y)
{
    double c[128], s[128];
    for (int32_t j = 0; j < D / 2; ++j) {
        c[j] = cos(theta[j]);
        s[j] = sin(theta[j]);
    }
    for (int pass = 0; pass < 2; ++pass) {
        int32_t H = pass ? Hk : Hq;
        const uint16_t* src = row + (pass ? (int64_t)Hq * D : 0);
        double* dst = pass ? k_o : q_o;
        int64_t n = (int64_t)H * D;
        for (int64_t ch = 0; ch < n; ++ch) x[ch] = qknr_oracle_bf16_to_double(src[ch]);
        if (is_qk_norm)
            qknr_oracle_rmsnorm(x, n, pass ? wk : wq, eps, y); /* across all H heads */
        else
            for (int64_t ch = 0; ch < n; ++ch) y[ch] = x[ch]; /* R11 */
        for (int32_t hh = 0; hh < H; ++hh)
            qknr_oracle_rotate(y + (int64_t)hh * D, D, D / 2, pa, pb, c, s, dst + (int64_t)hh * D);
    }
    const uint16_t* vsrc = row + (int64_t)(Hq + Hk) * D;
    for (int64_t ch = 0; ch < (int64_t)Hv * D; ++ch) v_o[ch] = qknr_oracle_bf16_to_double(vsrc[ch]);
}

static int check_3d(int32_t ppf, int32_t pph, int32_t ppw, int32_t Cf, int32_t Ch, int32_t Cw,
                    int32_t D)
{
    if (ppf <= 0 || pph <= 0 || ppw <= 0) return 1;
    if ((Cf & 1) || (Ch & 1) || (Cw & 1) || Cf < 0 || Ch < 0 || Cw < 0) return 1;
    if (Cf + Ch + Cw != D || D > 256 || D <= 0) return 1;
    return 0;
}

/* Exact (pre-rounding, pre-scale) outputs of the 3D form: q [T, Hq, D],
 * k [T, Hk, D], v [T, Hv, D] in fp64. Weights are [Hq*D] and [Hk*D] bf16
 * (ignored when is_qk_norm is 0; may then be NULL). */
int qknr_oracle_rope_3d_exact(const uint16_t* qkv, const uint16_t* q_weight,
                              const uint16_t* k_weight, int64_t num_tokens, int64_t pos_offset,
                              int32_t ppf, int32_t pph, int32_t ppw, int32_t Cf, int32_t Ch,
                              int32_t Cw, int32_t Hq, int32_t Hk, int32_t Hv, int32_t D,
                              double eps, double base, int32_t interleave,
                              int32_t neox_per_axis, int32_t is_qk_norm, double* q_out,
                              double* k_out, double* v_out)
{
    if (check_3d(ppf, pph, ppw, Cf, Ch, Cw, D)) return 1;
    int64_t row = (int64_t)(Hq + Hk + Hv) * D;
    double* wq = malloc(sizeof(double) * ((int64_t)Hq * D + 1));
    double* wk = malloc(sizeof(double) * ((int64_t)Hk * D + 1));
    int32_t pa[128], pb[128];
    for (int64_t c = 0; c < (int64_t)Hq * D; ++c)
        wq[c] = (is_qk_norm && q_weight) ? qknr_oracle_bf16_to_double(q_weight[c]) : 1.0;
    for (int64_t c = 0; c < (int64_t)Hk * D; ++c)
        wk[c] = (is_qk_norm && k_weight) ? qknr_oracle_bf16_to_double(k_weight[c]) : 1.0;
    qknr_oracle_pairs_3d(Cf, Ch, Cw, interleave, neox_per_axis, pa, pb);
    int64_t nmax = (int64_t)(Hq > Hk ? Hq : Hk) * D;

#pragma omp parallel
    {
        double* x = malloc(sizeof(double) * (nmax + 1));
        double* y = malloc(sizeof(double) * (nmax + 1));
        double theta[128];
#pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < num_tokens; ++t) {
            int64_t f, h, w;
            qknr_oracle_position_3d(t, pos_offset, ppf, pph, ppw, &f, &h, &w);
            qknr_oracle_angles_3d(f, h, w, Cf, Ch, Cw, base, theta);
            rope_3d_token(qkv + t * row, wq, wk, theta, pa, pb, Hq, Hk, Hv, D, eps, is_qk_norm,
                          q_out + t * Hq * D, k_out + t * Hk * D, v_out + t * Hv * D, x, y);
        }
        free(x);
        free(y);
    }
    free(wq);
    free(wk);
    return 0;
}

/* 3D form with its output rounding (R3): bf16 outputs, or, with output_fp8,
 * E4M3(q * q_scale), E4M3(k * q_scale), E4M3(v * v_scale) (R9, R10).
 * Outputs are uint16 bf16 patterns or uint8 E4M3 patterns. */
int qknr_oracle_rope_3d(const uint16_t* qkv, const uint16_t* q_weight, const uint16_t* k_weight,
                        int64_t num_tokens, int64_t pos_offset, int32_t ppf, int32_t pph,
                        int32_t ppw, int32_t Cf, int32_t Ch, int32_t Cw, int32_t Hq, int32_t Hk,
                        int32_t Hv, int32_t D, double eps, double base, int32_t interleave,
                        int32_t neox_per_axis, int32_t is_qk_norm, int32_t output_fp8,
                        double q_scale, double v_scale, void* q_out, void* k_out, void* v_out)
{
    int64_t nq = num_tokens * Hq * D, nk = num_tokens * Hk * D, nv = num_tokens * Hv * D;
    double* eq = malloc(sizeof(double) * (nq + 1));
    double* ek = malloc(sizeof(double) * (nk + 1));
    double* ev = malloc(sizeof(double) * (nv + 1));
    int rc = qknr_oracle_rope_3d_exact(qkv, q_weight, k_weight, num_tokens, pos_offset, ppf, pph,
                                       ppw, Cf, Ch, Cw, Hq, Hk, Hv, D, eps, base, interleave,
                                       neox_per_axis, is_qk_norm, eq, ek, ev);
    if (rc == 0) {
        if (output_fp8) {
            for (int64_t i = 0; i < nq; ++i)
                ((uint8_t*)q_out)[i] = qknr_oracle_e4m3_from_double(eq[i] * q_scale);
            for (int64_t i = 0; i < nk; ++i)
                ((uint8_t*)k_out)[i] = qknr_oracle_e4m3_from_double(ek[i] * q_scale);
            for (int64_t i = 0; i < nv; ++i)
                ((uint8_t*)v_out)[i] = qknr_oracle_e4m3_from_double(ev[i] * v_scale);
        } else {
            qknr_oracle_bf16_from_double_array(eq, (uint16_t*)q_out, nq);
            qknr_oracle_bf16_from_double_array(ek, (uint16_t*)k_out, nk);
            qknr_oracle_bf16_from_double_array(ev, (uint16_t*)v_out, nv);
        }
    }
    free(eq);
    free(ek);
    free(ev);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* UCPE camera prep ([U] cam_prep_func)                                      */
/* ------------------------------------------------------------------------ */

/* U1: the feature map of the camera branch, max(x, 0) per element. */
void qknr_oracle_relu(const double* x, int64_t n, double* y)
{
    for (int64_t i = 0; i < n; ++i) y[i] = x[i] > 0.0 ? x[i] : 0.0;
}

/* U3: ray projection of one head. Every block of four consecutive channels
 * (x[4b], ..., x[4b+3]) is replaced by m times it, m a 4x4 matrix stored row
 * by row: y[4b+i] = sum_j m[4i+j] x[4b+j]. n must be a multiple of 4. */
void qknr_oracle_ray_project(const double* m, const double* x, int64_t n, double* y)
{
    for (int64_t b = 0; b + 4 <= n; b += 4)
        for (int i = 0; i < 4; ++i) {
            double acc = 0.0;
            for (int j = 0; j < 4; ++j) acc += m[4 * i + j] * x[b + j];
            y[b + i] = acc;
        }
}

/* Exact (pre-rounding) results of the camera prep for dense inputs
 * q, k, v [B, N, H, D] (16-bit activation patterns, binary16 when act_is_f16),
 * fp32 projection matrices proj_q, proj_kv [B, N, 4, 4] and fp32 rope_cos,
 * rope_sin [N, D/2]. Outputs q_out, k_out, v_out are fp64 in [B, H, D, N]
 * layout (U5) and inflation_sq is fp64 [B, H, N] (U6). Per token n and head h:
 *   Q: ReLU (U1), projection by proj_q (U3), rotation (U4);
 *   K: ReLU (U1), times k_scale (U2), projection by proj_kv (U3), rotation (U4);
 *   V: projection by proj_kv only (U1, U4).
 * Returns 1, writing nothing, when head_dim is not a positive multiple of 4
 * up to 512 or a size is negative. */
int qknr_oracle_ucpe_exact(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const float* proj_q, const float* proj_kv, const float* rope_cos,
                           const float* rope_sin, int32_t act_is_f16, int64_t batch,
                           int64_t num_tokens, int32_t heads, int32_t head_dim, double k_scale,
                           double* q_out, double* k_out, double* v_out, double* inflation_sq)
{
    const int32_t D = head_dim;
    const int64_t B = batch, N = num_tokens, H = heads;
    if (B < 0 || N < 0 || H < 0 || D <= 0 || D > 512 || (D % 4)) return 1;
    int32_t* pa = malloc(sizeof(int32_t) * (D / 2));
    int32_t* pb = malloc(sizeof(int32_t) * (D / 2));
    qknr_oracle_pairs_table(D, 1, pa, pb); /* U4: adjacent pairs (2j, 2j+1) */

#pragma omp parallel for collapse(2) schedule(dynamic, 16)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t n = 0; n < N; ++n) {
            double mq[16], mkv[16], c[256], s[256];
            double x[512], r[512], y[512], o[512];
            for (int i = 0; i < 16; ++i) {
                mq[i] = proj_q[(b * N + n) * 16 + i];
                mkv[i] = proj_kv[(b * N + n) * 16 + i];
            }
            for (int32_t j = 0; j < D / 2; ++j) {
                c[j] = rope_cos[n * (D / 2) + j];
                s[j] = rope_sin[n * (D / 2) + j];
            }
            for (int64_t h = 0; h < H; ++h) {
                const int64_t in = ((b * N + n) * H + h) * D;
                const int64_t out = (b * H + h) * D * N + n; /* channel d at out + d * N */

                /* Q */
                for (int32_t d = 0; d < D; ++d) x[d] = act_to_double(q[in + d], act_is_f16);
                qknr_oracle_relu(x, D, r);
                qknr_oracle_ray_project(mq, r, D, y);
                qknr_oracle_rotate(y, D, D / 2, pa, pb, c, s, o);
                for (int32_t d = 0; d < D; ++d) q_out[out + (int64_t)d * N] = o[d];

                /* K, and the squared-norm gain of its projection */
                for (int32_t d = 0; d < D; ++d) x[d] = act_to_double(k[in + d], act_is_f16);
                qknr_oracle_relu(x, D, r);
                for (int32_t d = 0; d < D; ++d) r[d] *= k_scale;
                qknr_oracle_ray_project(mkv, r, D, y);
                double before = 0.0, after = 0.0;
                for (int32_t d = 0; d < D; ++d) {
                    before += r[d] * r[d];
                    after += y[d] * y[d];
                }
                inflation_sq[(b * H + h) * N + n] = before > 0.0 ? after / before : 1.0;
                qknr_oracle_rotate(y, D, D / 2, pa, pb, c, s, o);
                for (int32_t d = 0; d < D; ++d) k_out[out + (int64_t)d * N] = o[d];

                /* V */
                for (int32_t d = 0; d < D; ++d) x[d] = act_to_double(v[in + d], act_is_f16);
                qknr_oracle_ray_project(mkv, x, D, y);
                for (int32_t d = 0; d < D; ++d) v_out[out + (int64_t)d * N] = y[d];
            }
        }
    free(pa);
    free(pb);
    return 0;
}

/* Camera prep with its output rounding (U5): q/k/v results rounded once to
 * the activation type (bf16, or binary16 when act_is_f16); inflation_sq is
 * returned in fp64. */
int qknr_oracle_ucpe(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     const float* proj_q, const float* proj_kv, const float* rope_cos,
                     const float* rope_sin, int32_t act_is_f16, int64_t batch, int64_t num_tokens,
                     int32_t heads, int32_t head_dim, double k_scale, uint16_t* q_out,
                     uint16_t* k_out, uint16_t* v_out, double* inflation_sq)
{
    int64_t n = batch * num_tokens * heads * head_dim;
    if (n < 0) return 1;
    double* eq = malloc(sizeof(double) * (n + 1));
    double* ek = malloc(sizeof(double) * (n + 1));
    double* ev = malloc(sizeof(double) * (n + 1));
    int rc = qknr_oracle_ucpe_exact(q, k, v, proj_q, proj_kv, rope_cos, rope_sin, act_is_f16,
                                    batch, num_tokens, heads, head_dim, k_scale, eq, ek, ev,
                                    inflation_sq);
    if (rc == 0) {
        void (*round_to)(const double*, uint16_t*, int64_t) =
            act_is_f16 ? qknr_oracle_f16_from_double_array : qknr_oracle_bf16_from_double_array;
        round_to(eq, q_out, n);
        round_to(ek, k_out, n);
        round_to(ev, v_out, n);
    }
    free(eq);
    free(ek);
    free(ev);
    return rc;
}

/* OpenMP thread count used by the loops above (1 without OpenMP). */
int qknr_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void qknr_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
