/*
 * bitnet_oracle.c -- plain, slow CPU oracle for the BitNet b1.58 BitLinear
 * projection (W1.58A8) and the two FFN compositions built from it.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path (the
 * CUDA library) never calls it and shares no code, header or table with it.
 *
 * Every function follows one stated definition, in the order the pages give
 * it, with no blocking, fusion or reordering.  Sources (web pages):
 *   [NN]  nnterp encyclopedia "bitnet" (ndif-team.github.io/nnterp):
 *         "The projections quantize their inputs and weights",
 *         "The block, in order", "Scaling inside a sublayer is undone by the
 *         sub-norm", "The MLP gates with a squared ReLU", "Config".
 *   [AZ]  "BitNet b1.58 2B4T - Scaling Native 1-bit LLM" (Azure AI catalog),
 *         "Model Details" (absmean ternary weights, per-token absmax int8
 *         activations, ReLU^2, subln, no bias).
 *   [H1]  "bitnetv2-model" README: "Architecture Overview",
 *         "Special Features", "Technical Details" (H-BitLinear: a Hadamard
 *         transform on power-of-two widths, 512 -> 2048 -> 512 FFN, SiLU).
 *
 * Numeric conventions (readings where the pages are silent; each is listed
 * with its reason in the design notes):
 *   - fp32 arithmetic is IEEE round-to-nearest-even; build with
 *     -ffp-contract=off and no fast-math so no FMA contraction happens.
 *   - rounding to an integer code is rintf (half to even).
 *   - gamma and the RMS mean-square are accumulated in fp64 and rounded once.
 *   - dequantisation and SiLU are evaluated in fp64 and rounded once to fp32.
 *
 * Packed ternary layout (the pages say only "four to a byte"; this bit order
 * is this library's own convention): a packed row holds ldw = 16*ceil(K/64)
 * bytes.  Weight k of row n lives in byte n*ldw + 4*(k/16) + (k%4), at bits
 * 2*((k%16)/4) .. +1, as the code c = t + 1 in {0,1,2}.  Positions k >= K in
 * the padded tail hold code 1 (t = 0).  Code 3 is never written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_OVERFLOW 1
#define ORC_ERR_ARG 2

enum { ORC_PRELUDE_NONE = 0, ORC_PRELUDE_RMSNORM = 1, ORC_PRELUDE_FWHT = 2 };

/* ---------------------------------------------------------------- weights */

/* gamma = mean |W| over the whole tensor.  [NN] "rounded to {-1,0,1} *
 * mean|W|"; [AZ] "absmean quantization".  Sum in fp64 in row-major order,
 * divide by the element count in fp64, round once to fp32. */
float orc_absmean(const float *w, int64_t count)
{
    if (count <= 0) return 0.0f;
    double acc = 0.0;
    for (int64_t i = 0; i < count; ++i) acc += fabs((double)w[i]);
    return (float)(acc / (double)count);
}

/* t = clamp(rint(W / gamma), -1, 1); gamma == 0 gives t = 0 everywhere.
 * [NN] "rounded to {-1, 0, 1} * mean|W| in every forward". */
void orc_ternarize(const float *w, int64_t count, float gamma, int8_t *t)
{
    for (int64_t i = 0; i < count; ++i) {
        if (gamma == 0.0f) { t[i] = 0; continue; }
        float r = w[i] / gamma;          /* IEEE fp32 division */
        float v = rintf(r);              /* half to even */
        if (v > 1.0f) v = 1.0f;
        if (v < -1.0f) v = -1.0f;
        t[i] = (int8_t)v;
    }
}

/* Bytes per packed row: 16-byte aligned rows of 64 weights per 16 bytes. */
int64_t orc_packed_row_bytes(int K)
{
    return 16 * (int64_t)((K + 63) / 64);
}

/* Four ternary codes to a byte ([NN] "stored ternary, four to a byte"), in
 * the layout stated in the file header. */
void orc_pack(const int8_t *t, int N, int K, uint8_t *packed)
{
    int64_t ldw = orc_packed_row_bytes(K);
    /* every position starts as code 1 (t = 0) so the padded tail reads as 0 */
    memset(packed, 0x55, (size_t)(ldw * N));
    for (int n = 0; n < N; ++n) {
        for (int k = 0; k < K; ++k) {
            int64_t byte = (int64_t)n * ldw + 4 * (k / 16) + (k % 4);
            int shift = 2 * ((k % 16) / 4);
            unsigned code = (unsigned)(t[(int64_t)n * K + k] + 1);
            packed[byte] = (uint8_t)((packed[byte] & ~(3u << shift)) | (code << shift));
        }
    }
}

/* Inverse of orc_pack.  Returns ORC_ERR_ARG if any code is 3. */
int orc_unpack(const uint8_t *packed, int N, int K, int8_t *t)
{
    int64_t ldw = orc_packed_row_bytes(K);
    for (int n = 0; n < N; ++n) {
        for (int k = 0; k < K; ++k) {
            int64_t byte = (int64_t)n * ldw + 4 * (k / 16) + (k % 4);
            int shift = 2 * ((k % 16) / 4);
            unsigned code = (packed[byte] >> shift) & 3u;
            if (code == 3u) return ORC_ERR_ARG;
            t[(int64_t)n * K + k] = (int8_t)((int)code - 1);
        }
    }
    return ORC_OK;
}

/* The canonical exchange layout TW2: row n occupies bytes [n K/4, (n+1) K/4)
 * and weight k of row n is the code c = t + 1 at bits 2 (k mod 4) of byte
 * n K/4 + floor(k / 4) (four to a byte, [NN] "stored ternary, four to a
 * byte"; the low-bits-first order is this library's stated convention).
 * K must be a multiple of 4. */
void orc_pack_tw2(const int8_t *t, int N, int K, uint8_t *tw2)
{
    int64_t rb = K / 4;
    memset(tw2, 0, (size_t)(rb * N));
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            unsigned code = (unsigned)(t[(int64_t)n * K + k] + 1);
            tw2[(int64_t)n * rb + k / 4] |= (uint8_t)(code << (2 * (k % 4)));
        }
}

/* Inverse of orc_pack_tw2.  Returns ORC_ERR_ARG if any code is 3. */
int orc_unpack_tw2(const uint8_t *tw2, int N, int K, int8_t *t)
{
    int64_t rb = K / 4;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            unsigned code = (tw2[(int64_t)n * rb + k / 4] >> (2 * (k % 4))) & 3u;
            if (code == 3u) return ORC_ERR_ARG;
            t[(int64_t)n * K + k] = (int8_t)((int)code - 1);
        }
    return ORC_OK;
}

/* ------------------------------------------------------------- preludes */

/* RMSNorm with gain, no bias, eps 1e-5 in the model ([NN] "Config":
 * rms_norm_eps; "The block, in order": the four RMSNorms; [AZ] "No bias
 * terms").  ms = sum(x^2)/K accumulated in fp64 and rounded once;
 * r = 1/sqrt(ms + eps) in fp32; out = (x * r) * g in fp32. */
void orc_rmsnorm_row(const float *x, int K, const float *gain, float eps, float *out)
{
    double ss = 0.0;
    for (int k = 0; k < K; ++k) ss += (double)x[k] * (double)x[k];
    float ms = (float)(ss / (double)K);
    float r = 1.0f / sqrtf(ms + eps);
    for (int k = 0; k < K; ++k) {
        float v = x[k] * r;
        out[k] = v * (gain ? gain[k] : 1.0f);
    }
}

/* Normalised fast Walsh-Hadamard transform in natural (Sylvester) order on a
 * power-of-two width ([H1] "H-BitLinear: Uses Hadamard transforms", "power of
 * 2 for H-BitLinear").  Butterfly stages h = 1, 2, 4, ..., n/2 in that order,
 * (a, b) -> (a + b, a - b) on the pair (j, j + h); then one multiply by
 * c = 1/sqrt(n) computed in fp64 and rounded to fp32.  Returns ORC_ERR_ARG
 * when n is not a power of two. */
int orc_fwht_row(const float *x, int n, float *out)
{
    if (n <= 0 || (n & (n - 1)) != 0) return ORC_ERR_ARG;
    for (int k = 0; k < n; ++k) out[k] = x[k];
    for (int h = 1; h < n; h <<= 1) {
        for (int i = 0; i < n; i += 2 * h) {
            for (int j = i; j < i + h; ++j) {
                float a = out[j], b = out[j + h];
                out[j] = a + b;
                out[j + h] = a - b;
            }
        }
    }
    float c = (float)(1.0 / sqrt((double)n));
    for (int k = 0; k < n; ++k) out[k] = out[k] * c;
    return ORC_OK;
}

/* ------------------------------------------------------- activation quant */

/* Per-token absmax int8: s = 127 / max|x| (fp32 division), q = clamp(rint(x *
 * s), -128, 127) ([NN] "rounds its input per token to 255 levels (round(x *
 * 127 / max|x|))"; [AZ] "8-bit integers using absmax quantization
 * (per-token)").  A row whose max is 0, or whose scale is not finite, gets
 * q = 0 and s = 1.  rowsum (may be NULL) receives sum(q). */
void orc_quant_row(const float *x, int K, int8_t *q, float *s, int32_t *rowsum)
{
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) {
        float a = fabsf(x[k]);
        if (a > amax) amax = a;
    }
    float scale = 127.0f / amax;
    int32_t sum = 0;
    if (amax == 0.0f || !isfinite(scale)) {
        for (int k = 0; k < K; ++k) q[k] = 0;
        scale = 1.0f;
    } else {
        for (int k = 0; k < K; ++k) {
            float v = rintf(x[k] * scale);
            if (v > 127.0f) v = 127.0f;
            if (v < -128.0f) v = -128.0f;
            q[k] = (int8_t)v;
            sum += q[k];
        }
    }
    *s = scale;
    if (rowsum) *rowsum = sum;
}

/* Prelude (none / RMSNorm / FWHT) then per-token quant, row by row. */
int orc_quant_act(const float *X, int M, int K, int prelude, const float *gain,
                  float eps, int8_t *Xq, float *scale, int32_t *rowsum)
{
    if (prelude == ORC_PRELUDE_FWHT && (K <= 0 || (K & (K - 1)) != 0)) return ORC_ERR_ARG;
    int err = ORC_OK;
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m) {
        const float *x = X + (int64_t)m * K;
        float *tmp = (float *)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
        if (prelude == ORC_PRELUDE_RMSNORM) orc_rmsnorm_row(x, K, gain, eps, tmp);
        else if (prelude == ORC_PRELUDE_FWHT) orc_fwht_row(x, K, tmp);
        else memcpy(tmp, x, sizeof(float) * (size_t)K);
        orc_quant_row(tmp, K, Xq + (int64_t)m * K, scale + m, rowsum ? rowsum + m : NULL);
        free(tmp);
    }
    return err;
}

/* ------------------------------------------------------------ contraction */

/* acc[m,n] = sum_k q[m,k] * t[n,k] in int64, then checked to fit int32.
 * [NN] "q_proj.output equals the linear map of the rounded input by the
 * ternarized weight exactly". */
int orc_contract(const int8_t *Xq, const int8_t *T, int M, int N, int K, int32_t *acc)
{
    int overflow = 0;
#pragma omp parallel for schedule(static) reduction(|:overflow)
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            int64_t a = 0;
            for (int k = 0; k < K; ++k)
                a += (int64_t)Xq[(int64_t)m * K + k] * (int64_t)T[(int64_t)n * K + k];
            if (a > INT32_MAX || a < INT32_MIN) overflow = 1;
            acc[(int64_t)m * N + n] = (int32_t)a;
        }
    }
    return overflow ? ORC_ERR_OVERFLOW : ORC_OK;
}

/* y = acc * gamma / s[m], in fp64, rounded once to fp32. */
void orc_dequant(const int32_t *acc, const float *scale, float gamma, int M, int N, float *Y)
{
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            int64_t i = (int64_t)m * N + n;
            Y[i] = (float)((double)acc[i] * (double)gamma / (double)scale[m]);
        }
}

/* ------------------------------------------------------ scalar epilogues */

/* Round fp32 to bf16 (round to nearest, ties to even) and widen back. */
float orc_round_bf16(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) {      /* inf or NaN: truncate */
        u &= 0xffff0000u;
        if ((x != x)) u |= 0x00400000u;
    } else {
        uint32_t lsb = (u >> 16) & 1u;
        u += 0x7fffu + lsb;
        u &= 0xffff0000u;
    }
    float r;
    memcpy(&r, &u, 4);
    return r;
}

/* relu(g)^2 * u in fp32 ([NN] "The MLP gates with a squared ReLU": a neuron
 * is relu(gate)^2 * up, exactly zero wherever the gate is negative). */
float orc_relu2_glu(float g, float u)
{
    float a = g > 0.0f ? g * g : 0.0f;
    return a * u;
}

/* silu(y) = y / (1 + exp(-y)) in fp64, rounded once ([H1] "Activation
 * function: silu"). */
float orc_silu(float y)
{
    double d = (double)y;
    return (float)(d / (1.0 + exp(-d)));
}

/* --------------------------------------------------------- compositions */

/* One BitLinear: prelude -> quant -> contraction -> dequant, with t given as
 * ternary codes [N][K].  Optional fp32 residual added after the dequant. */
int orc_bitlinear(const float *X, int M, int K, int prelude, const float *gain, float eps,
                  const int8_t *T, float gamma, int N, const float *residual, float *Y)
{
    int8_t *q = (int8_t *)malloc((size_t)M * (size_t)K + 1);
    float *s = (float *)malloc(sizeof(float) * (size_t)(M + 1));
    int32_t *acc = (int32_t *)malloc(sizeof(int32_t) * ((size_t)M * (size_t)N + 1));
    int err = orc_quant_act(X, M, K, prelude, gain, eps, q, s, NULL);
    if (!err) err = orc_contract(q, T, M, N, K, acc);
    if (!err) {
        orc_dequant(acc, s, gamma, M, N, Y);
        if (residual)
            for (int64_t i = 0; i < (int64_t)M * N; ++i) Y[i] = residual[i] + Y[i];
    }
    free(q); free(s); free(acc);
    return err;
}

/* The W1.58A8 FFN half of a block ([NN] "The block, in order"):
 *   z   = post_attention_layernorm(x)            (RMSNorm, gain pre_gain)
 *   m   = relu(gate_proj(z))^2 * up_proj(z)      (each a BitLinear of z)
 *   out = x + down_proj(ffn_sub_norm(m))         (RMSNorm gain sub_gain)
 * x [M][H] fp32 (bf16 inputs are widened exactly by the caller); Tg, Tu
 * [I][H], Td [H][I] ternary codes.  Intermediates are kept for inspection
 * when the pointers are non-NULL: m [M][I], qm [M][I], sm [M]. */
int orc_ffn_relu2(const float *x, int M, int H, int I,
                  const int8_t *Tg, float gg, const int8_t *Tu, float gu,
                  const int8_t *Td, float gd, const float *pre_gain, const float *sub_gain,
                  float eps, int add_residual, float *out,
                  float *m_out, int8_t *qm_out, float *sm_out)
{
    int64_t MI = (int64_t)M * I, MH = (int64_t)M * H;
    int8_t *qx = (int8_t *)malloc((size_t)MH + 1);
    float *sx = (float *)malloc(sizeof(float) * (size_t)(M + 1));
    int32_t *acc = (int32_t *)malloc(sizeof(int32_t) * (size_t)(MI > MH ? MI : MH) + 4);
    float *G = (float *)malloc(sizeof(float) * (size_t)MI + 4);
    float *U = (float *)malloc(sizeof(float) * (size_t)MI + 4);
    int8_t *qm = (int8_t *)malloc((size_t)MI + 1);
    float *sm = (float *)malloc(sizeof(float) * (size_t)(M + 1));
    int err = orc_quant_act(x, M, H, ORC_PRELUDE_RMSNORM, pre_gain, eps, qx, sx, NULL);
    if (!err) err = orc_contract(qx, Tg, M, I, H, acc);
    if (!err) { orc_dequant(acc, sx, gg, M, I, G); err = orc_contract(qx, Tu, M, I, H, acc); }
    if (!err) {
        orc_dequant(acc, sx, gu, M, I, U);
        for (int64_t i = 0; i < MI; ++i) G[i] = orc_relu2_glu(G[i], U[i]);   /* G now holds m */
        if (m_out) memcpy(m_out, G, sizeof(float) * (size_t)MI);
        err = orc_quant_act(G, M, I, ORC_PRELUDE_RMSNORM, sub_gain, eps, qm, sm, NULL);
    }
    if (!err) {
        if (qm_out) memcpy(qm_out, qm, (size_t)MI);
        if (sm_out) memcpy(sm_out, sm, sizeof(float) * (size_t)M);
        err = orc_contract(qm, Td, M, H, I, acc);
    }
    if (!err) {
        orc_dequant(acc, sm, gd, M, H, out);
        if (add_residual)
            for (int64_t i = 0; i < MH; ++i) out[i] = x[i] + out[i];
    }
    free(qx); free(sx); free(acc); free(G); free(U); free(qm); free(sm);
    return err;
}

/* The block after attention ([NN] "The block, in order"):
 *   h   = x + o_proj(attn_sub_norm(a))          (a = attention output)
 *   out = h + down_proj(ffn_sub_norm(relu(gate_proj(z))^2 * up_proj(z))),
 *         z = post_attention_layernorm(h)
 * a, x [M][H] fp32 (bf16 inputs widened exactly by the caller); To [H][H],
 * Tg, Tu [I][H], Td [H][I] ternary codes; gains [H] / [I] or NULL; h is
 * kept in fp32 (written to h_out when non-NULL); out [M][H] fp32. */
int orc_block_tail(const float *a, const float *x, int M, int H, int I,
                   const int8_t *To, float go, const int8_t *Tg, float gg,
                   const int8_t *Tu, float gu, const int8_t *Td, float gd,
                   const float *attn_gain, const float *post_gain, const float *sub_gain,
                   float eps, float *h_out, float *out)
{
    int64_t MH = (int64_t)M * H;
    float *h = (float *)malloc(sizeof(float) * (size_t)MH + 4);
    int err = orc_bitlinear(a, M, H, ORC_PRELUDE_RMSNORM, attn_gain, eps, To, go, H, x, h);
    if (!err) {
        if (h_out) memcpy(h_out, h, sizeof(float) * (size_t)MH);
        err = orc_ffn_relu2(h, M, H, I, Tg, gg, Tu, gu, Td, gd, post_gain, sub_gain, eps, 1,
                            out, NULL, NULL, NULL);
    }
    free(h);
    return err;
}

/* The H-BitLinear FFN ([H1] "H-BitLinear Feed-Forward Network: 512 -> 2048
 * -> 512", "Activation function: silu", "Hadamard transform-based linear
 * layers"): y = W2 . silu(W1 . x), each projection an H-BitLinear, i.e. a
 * normalised FWHT of its input before the per-token int8 quant.  x [M][D]
 * fp32, T1 [F][D], T2 [D][F] ternary codes; out [M][D] fp32.  The hidden
 * activation (post-SiLU, pre-transform) is kept when h_out != NULL. */
int orc_hffn(const float *x, int M, int D, int F,
             const int8_t *T1, float g1, const int8_t *T2, float g2,
             float *out, float *h_out)
{
    int64_t MF = (int64_t)M * F;
    float *Hh = (float *)malloc(sizeof(float) * (size_t)MF + 4);
    int err = orc_bitlinear(x, M, D, ORC_PRELUDE_FWHT, NULL, 0.0f, T1, g1, F, NULL, Hh);
    if (!err) {
        for (int64_t i = 0; i < MF; ++i) Hh[i] = orc_silu(Hh[i]);
        if (h_out) memcpy(h_out, Hh, sizeof(float) * (size_t)MF);
        err = orc_bitlinear(Hh, M, F, ORC_PRELUDE_FWHT, NULL, 0.0f, T2, g2, D, NULL, out);
    }
    free(Hh);
    return err;
}

/* ------------------------------------------------- array forms (bindings) */

void orc_round_bf16_array(const float *x, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_round_bf16(x[i]);
}

void orc_relu2_glu_array(const float *g, const float *u, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_relu2_glu(g[i], u[i]);
}

void orc_silu_array(const float *y, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_silu(y[i]);
}

void orc_rmsnorm(const float *X, int M, int K, const float *gain, float eps, float *out)
{
    for (int m = 0; m < M; ++m)
        orc_rmsnorm_row(X + (int64_t)m * K, K, gain, eps, out + (int64_t)m * K);
}

int orc_fwht(const float *X, int M, int n, float *out)
{
    for (int m = 0; m < M; ++m) {
        int err = orc_fwht_row(X + (int64_t)m * n, n, out + (int64_t)m * n);
        if (err) return err;
    }
    return ORC_OK;
}

/* ------------------------------------------------------ threading (plumbing) */

/* Threads the OpenMP loops above use (1 when built without OpenMP). */
void orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int orc_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
