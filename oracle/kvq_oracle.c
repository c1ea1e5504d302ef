/*
 * kvq_oracle.c -- plain, slow CPU reference of the NVFP4 attention cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * bench's CPU-baseline leg load this file (through the oracle package's
 * ctypes loader).  The
 * CUDA library never links, calls or includes it, and it includes nothing of
 * the library: the two share no code.
 *
 * Sources (web pages; cited by title and section):
 *   [P1] "NVFP4 attention cache on W4A4 Qwen3-8B: static key smoothing is
 *        near-lossless, key rotations hurt" (rstation.ai post) -- setup
 *        paragraph, results table, observations.
 *   [P3] "QServe SmoothAttention (4-bit KV cache with an accuracy-preserving
 *        correction)" -- Activation scheme / Kernels fields.
 *   [P4] "OSFP4: Joint Optimization of Diagonal Smoothing and Block Scales for
 *        NVFP4 Quantization" (paperlayer.ai summary) -- Problem bullet, sec. 1,
 *        sec. 3, sec. D.1.
 *   [P5] "QuaRot KV cache 4-bit (rotated KV, no retained outlier channels)".
 *
 * Precision.  The pages fix the formats but not the arithmetic of the
 * quantiser; it is computed here as a fixed sequence of IEEE fp32 operations,
 * each rounded to nearest-even (compiled with -ffp-contract=off, no fast-math,
 * so no fused multiply-add and no reassociation).  Everything after
 * dequantisation -- the query transform, scores, softmax and P.V -- is fp64.
 *
 * Readings of points the pages leave open:
 *   - FP32 per-tensor scale: static, one per (layer, K|V), g = amax / (6*448)
 *     over the transformed calibration tensor including position 0.
 *   - E4M3 block scale: round-to-nearest-even with saturation at 448.
 *   - A negative value that rounds to zero keeps its sign (code 0x8).
 *   - Hadamard: Sylvester order, butterfly stages h = 1, 2, ..., 64, then one
 *     multiply by fp32(1/sqrt(128)); keys only, queries rotated to match.
 *   - Softmax scale 1/sqrt(head_dim), no soft-cap.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define HD 128      /* head_dim: [P1] setup, Qwen3-8B heads of 128 channels */
#define BLK 16      /* NVFP4 block length along head_dim: [P1] setup; [P4] sec. D.1 */

/* ------------------------------------------------------------------------- */
/* E2M1 element format.  [P4] sec. D.1 names E2M1 values; [P4] sec. 1 gives 6
 * as the largest FP4 value.  Bit layout: s e1 e0 m, exponent bias 1; exponent
 * field 0 is subnormal (0 or 0.5). */
double oracle_e2m1_value(uint32_t code)
{
    uint32_t s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -mag : mag;
}

/* Round one fp32 value to E2M1: nearest of {0, .5, 1, 1.5, 2, 3, 4, 6},
 * ties to the even code (mantissa bit 0), magnitudes beyond 6 saturate to 6,
 * sign kept (so -0 and small negatives give 0x8). */
uint32_t oracle_e2m1_encode(float x)
{
    /* the decision points between consecutive magnitudes are their midpoints */
    static const double mid[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
    uint32_t sign = signbit(x) ? 8u : 0u;
    double a = fabs((double)x);
    uint32_t mag = 7;                        /* saturate by default */
    for (uint32_t i = 0; i < 7; ++i) {
        if (a < mid[i]) { mag = i; break; }
        if (a == mid[i]) {                   /* tie: pick the even code of the two */
            mag = (i & 1u) ? i + 1 : i;
            break;
        }
    }
    return sign | mag;
}

/* ------------------------------------------------------------------------- */
/* E4M3 scale format ([P4] sec. D.1: "E4M3 scales per 16").  OCP E4M3FN:
 * s eeee mmm, bias 7, no infinities, largest finite 448, S.1111.111 is NaN. */
double oracle_e4m3_value(uint32_t code)
{
    uint32_t s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    double mag;
    if (e == 15 && m == 7) mag = NAN;
    else if (e == 0) mag = ldexp((double)m, -9);              /* m/8 * 2^-6 */
    else mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

/* Round one fp32 value to E4M3, nearest-even, saturating at 448. */
uint32_t oracle_e4m3_encode(float x)
{
    uint32_t sign = signbit(x) ? 0x80u : 0u;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7Eu;
    /* quantum of the binade holding a; subnormal binade below 2^-6 */
    int e;
    if (a < ldexp(1.0, -6)) e = -6;
    else { (void)frexp(a, &e); e -= 1; }                  /* a in [2^e, 2^(e+1)) */
    double q = ldexp(1.0, e - 3);                          /* 3 mantissa bits */
    double n = a / q;                                      /* exact: power-of-two divide */
    double fl = floor(n), fr = n - fl;
    double r = (fr > 0.5 || (fr == 0.5 && fmod(fl, 2.0) != 0.0)) ? fl + 1.0 : fl;
    double v = r * q;
    if (v >= 448.0) return sign | 0x7Eu;
    /* encode the exact value v */
    if (v < ldexp(1.0, -6)) return sign | (uint32_t)(v / ldexp(1.0, -9));
    int ev; (void)frexp(v, &ev); ev -= 1;
    uint32_t m = (uint32_t)((v / ldexp(1.0, ev) - 1.0) * 8.0);
    return sign | ((uint32_t)(ev + 7) << 3) | m;
}

void oracle_e2m1_encode_n(const float* x, uint8_t* out, int64_t n)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)oracle_e2m1_encode(x[i]);
}

void oracle_e4m3_encode_n(const float* x, uint8_t* out, int64_t n)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)oracle_e4m3_encode(x[i]);
}

/* ------------------------------------------------------------------------- */
/* Key pre-transform T.  [P1] results table rows "static per-channel
 * smoothing, sqrt(absmax)" and observation 2 (SmoothAttention, [P3]): each key
 * channel is divided by its smoothing factor s_c -- here multiplied by the
 * stored reciprocal inv_s_c, one fp32 rounding.  Optional normalised
 * Hadamard-128 on head_dim ([P1] rows "Hadamard-128 on head_dim" and
 * "Hadamard-128 + smoothing"; QuaRot's rotation, [P5]) after smoothing. */
static const float kInvSqrt128 = 0.08838834764831845f;   /* fp32 nearest 1/sqrt(128) */

static void transform_row(const float* k, const float* inv_s, int hadamard, float* y)
{
    for (int c = 0; c < HD; ++c) y[c] = k[c] * inv_s[c];
    if (!hadamard) return;
    for (int h = 1; h < HD; h <<= 1)                     /* Sylvester butterflies */
        for (int j = 0; j < HD; ++j)
            if ((j & h) == 0) {
                float a = y[j], b = y[j + h];
                y[j] = a + b;
                y[j + h] = a - b;
            }
    for (int c = 0; c < HD; ++c) y[c] = y[c] * kInvSqrt128;
}

/* keys [n][H][D] (fp32) -> transformed [n][H][D]; inv_s is [H][D] */
void oracle_transform_keys(const float* k, const float* inv_s, int64_t n, int H, int hadamard, float* y)
{
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t)
        for (int h = 0; h < H; ++h)
            transform_row(k + ((size_t)t * H + h) * HD, inv_s + (size_t)h * HD, hadamard,
                          y + ((size_t)t * H + h) * HD);
}

/* Static per-head KLT ([P1] results table, rows "K: static per-head KLT" and
 * "K: static KLT + smoothing"): y' = U^T y for a 128 x 128 orthogonal U per
 * (layer, kv head), U[c][i] = component c of basis vector i.  Each output is
 * one fp32 fused multiply-add chain over c = 0, 1, ..., 127 starting from 0:
 * the library applies the transform in exactly this order, so the codes
 * that follow are reproducible bit for bit.
 *
 * y, out: [n][128] fp32; U: [128][128] fp32. */
void oracle_klt_apply(const float* y, const float* U, int64_t n, float* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        const float* yr = y + (size_t)r * HD;
        float* o = out + (size_t)r * HD;
        for (int i = 0; i < HD; ++i) {
            float acc = 0.0f;
            for (int c = 0; c < HD; ++c) acc = fmaf(U[(size_t)c * HD + i], yr[c], acc);
            o[i] = acc;
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Calibration ([P1] results table row 4 and observation 2): the smoothing
 * factor of each (layer, kv head, channel) is sqrt of the absolute maximum of
 * the post-RoPE key over the calibration windows, position 0 of each window
 * excluded (exclude_pos0 = 1) or included (row 5 of the table).
 * The FP32 per-tensor scale follows the "global calibration-based scale" of
 * [P4] sec. 3, fitted so the tensor's absmax maps to 6 * 448: one per layer
 * for K (after the transform) and one for V.
 *
 * k, v: [L][W][T][H][D] fp32.  s, inv_s: [L][H][D].  gk, gv: [L]. */
/* smooth = 0: keys kept in their native basis ([P1] results table, row
 * "NVFP4 K only, native basis"): s = 1, and the tensor scale is taken over
 * the unsmoothed (optionally rotated) keys. */
void oracle_calibrate(const float* k, const float* v, int L, int W, int T, int H,
                      int exclude_pos0, int hadamard, int smooth,
                      float* s, float* inv_s, float* gk, float* gv)
{
    const size_t per_tok = (size_t)H * HD, per_win = (size_t)T * per_tok,
                 per_layer = (size_t)W * per_win;
    for (int l = 0; l < L; ++l) {
        const float* kl = k + l * per_layer;
        const float* vl = v + l * per_layer;
        float* sl = s + (size_t)l * per_tok;
        float* il = inv_s + (size_t)l * per_tok;
        for (int h = 0; h < H; ++h)
            for (int c = 0; c < HD; ++c) {
                float A = 0.0f;
                for (int w = 0; w < W; ++w)
                    for (int t = exclude_pos0 ? 1 : 0; t < T; ++t) {
                        float a = fabsf(kl[w * per_win + (size_t)t * per_tok + (size_t)h * HD + c]);
                        if (a > A) A = a;
                    }
                float sc = (smooth && A > 0.0f) ? sqrtf(A) : 1.0f;
                sl[h * HD + c] = sc;
                il[h * HD + c] = 1.0f / sc;
            }
        float amax_k = 0.0f, amax_v = 0.0f, y[HD];
        for (size_t r = 0; r < (size_t)W * T; ++r)
            for (int h = 0; h < H; ++h) {
                transform_row(kl + r * per_tok + (size_t)h * HD, il + (size_t)h * HD, hadamard, y);
                for (int c = 0; c < HD; ++c) {
                    if (fabsf(y[c]) > amax_k) amax_k = fabsf(y[c]);
                    float a = fabsf(vl[r * per_tok + (size_t)h * HD + c]);
                    if (a > amax_v) amax_v = a;
                }
            }
        gk[l] = (amax_k > 0.0f) ? amax_k / 2688.0f : 1.0f;
        gv[l] = (amax_v > 0.0f) ? amax_v / 2688.0f : 1.0f;
    }
}

/* ------------------------------------------------------------------------- */
/* NVFP4 quantisation of one 16-entry block ([P4] Problem bullet and sec. 1:
 * absmax mapped to 6, the largest FP4 value; [P4] sec. D.1: E2M1 values, an
 * E4M3 scale per 16 entries and an FP32 tensor scale g).
 *   a   = max |y_i|
 *   enc = 1 / (6 g)                   (per tensor)
 *   sf  = E4M3(a * enc)               block scale, RNE, saturating
 *   d   = val(sf) * g                 effective block step
 *   r   = 1 / d   (0 when d = 0)
 *   q_i = E2M1(y_i * r)
 * Every product and quotient is one fp32 rounding. */
static void quantize_block(const float* y, float enc, float g, uint8_t* codes, uint8_t* sf)
{
    float a = 0.0f;
    for (int i = 0; i < BLK; ++i) if (fabsf(y[i]) > a) a = fabsf(y[i]);
    uint32_t s = oracle_e4m3_encode(a * enc);
    float d = (float)oracle_e4m3_value(s) * g;
    float r = (d == 0.0f) ? 0.0f : 1.0f / d;
    for (int i = 0; i < BLK; ++i) codes[i] = (uint8_t)oracle_e2m1_encode(y[i] * r);
    *sf = (uint8_t)s;
}

/* rows [n][D] (fp32, already transformed) -> codes [n][D] (one 4-bit code per
 * byte, element order) and scales [n][D/16] */
void oracle_quantize_rows(const float* y, int64_t n, float g, uint8_t* codes, uint8_t* sf)
{
    const float six_g = 6.0f * g;
    const float enc = 1.0f / six_g;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r)
        for (int b = 0; b < HD / BLK; ++b)
            quantize_block(y + (size_t)r * HD + b * BLK, enc, g,
                           codes + (size_t)r * HD + b * BLK, sf + (size_t)r * (HD / BLK) + b);
}

/* Query rows quantised to NVFP4 for a Q.K product taken on FP4 tensor cores
 * with block scales ([P1] setup: W4A4, activations in NVFP4; [P4] Problem
 * bullet, sec. 1 and sec. D.1: absmax of each 16-entry block mapped to 6,
 * an E4M3 scale per block, an FP32 scale above it).  The pages fix no
 * static scale for queries, so the FP32 scale is taken online per row, the
 * same way the static tensor scale is fitted: g = amax(row) / (6 * 448)
 * (1 for an all-zero row); the blocks are then quantised exactly as the
 * cache's (quantize_block above).
 *   y:     [n][D] fp32, already transformed (smoothing, rotation)
 *   codes: [n][D] one code per byte;  sf: [n][D/16];  g: [n] */
void oracle_quantize_query_rows(const float* y, int64_t n, uint8_t* codes, uint8_t* sf, float* g)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        const float* yr = y + (size_t)r * HD;
        float a = 0.0f;
        for (int c = 0; c < HD; ++c) if (fabsf(yr[c]) > a) a = fabsf(yr[c]);
        const float gr = (a > 0.0f) ? a / 2688.0f : 1.0f;
        const float six_g = 6.0f * gr;
        const float enc = 1.0f / six_g;
        for (int b = 0; b < HD / BLK; ++b)
            quantize_block(yr + b * BLK, enc, gr, codes + (size_t)r * HD + b * BLK, sf + (size_t)r * (HD / BLK) + b);
        g[r] = gr;
    }
}

/* Dequantisation, exact in fp64: x = val(code) * val(sf) * g. */
void oracle_dequantize_rows(const uint8_t* codes, const uint8_t* sf, int64_t n, float g, double* x)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r)
        for (int c = 0; c < HD; ++c)
            x[(size_t)r * HD + c] = oracle_e2m1_value(codes[(size_t)r * HD + c])
                                  * oracle_e4m3_value(sf[(size_t)r * (HD / BLK) + c / BLK]) * (double)g;
}

/* ------------------------------------------------------------------------- */
/* Query transform, fp64: the smoothing factor is folded into the query
 * (q~ = q * s), [P1] observation 2 / [P3] SmoothAttention, so that
 * q~ . (k / s) = q . k; with the rotation, q~ <- H q~ / sqrt(128) ([P5]). */
static void query_transform(const float* q, const float* s, int hadamard, double* out)
{
    for (int c = 0; c < HD; ++c) out[c] = (double)q[c] * (double)s[c];
    if (!hadamard) return;
    double tmp[HD];
    for (int i = 0; i < HD; ++i) {
        double acc = 0.0;
        for (int j = 0; j < HD; ++j)
            acc += (__builtin_popcount((unsigned)(i & j)) & 1) ? -out[j] : out[j];
        tmp[i] = acc / sqrt((double)HD);
    }
    memcpy(out, tmp, sizeof tmp);
}

/* Exact softmax attention of one transformed query row qt (fp64) against the
 * first n cached positions of kv head h: scores qt . k_j / sqrt(D), softmax
 * over j < n, output sum_j p_j v_j.  kx, vx: [T][Hkv][D] fp64. */
static void attend_row(const double* qt, int h, int n, int Hkv, const double* kx, const double* vx, double* o)
{
    const double scale = 1.0 / sqrt((double)HD);
    for (int c = 0; c < HD; ++c) o[c] = 0.0;
    if (n <= 0) return;
    double* sc = (double*)malloc(sizeof(double) * (size_t)n);
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        const double* kj = kx + ((size_t)j * Hkv + h) * HD;
        double acc = 0.0;
        for (int c = 0; c < HD; ++c) acc += qt[c] * kj[c];
        sc[j] = acc * scale;
        if (sc[j] > m) m = sc[j];
    }
    double l = 0.0;
    for (int j = 0; j < n; ++j) { sc[j] = exp(sc[j] - m); l += sc[j]; }
    for (int j = 0; j < n; ++j) {
        const double* vj = vx + ((size_t)j * Hkv + h) * HD;
        double p = sc[j] / l;
        for (int c = 0; c < HD; ++c) o[c] += p * vj[c];
    }
    free(sc);
}

/* Causal GQA attention of Tq queries of one sequence and one layer against its
 * dequantised cache, exact softmax in fp64.
 *   q:    [Tq][Hq][D] fp32 (post-RoPE, untransformed)
 *   s:    [Hkv][D] smoothing factors
 *   kx:   [T][Hkv][D] dequantised transformed keys (fp64)
 *   vx:   [T][Hkv][D] dequantised values (fp64)
 *   query i attends cached positions j < min(T, q_start + i + 1); a decode
 *   step is Tq = 1, q_start = T - 1.
 *   out:  [Tq][Hq][D] fp64 */
void oracle_attention(const float* q, int Tq, int q_start, int Hq, int Hkv,
                      const float* s, int hadamard,
                      const double* kx, const double* vx, int T, double* out)
{
    const int G = Hq / Hkv;
    #pragma omp parallel for collapse(2) schedule(dynamic)
    for (int i = 0; i < Tq; ++i)
        for (int hq = 0; hq < Hq; ++hq) {
            int h = hq / G;
            int n = q_start + i + 1;
            if (n > T) n = T;
            double qt[HD];
            query_transform(q + ((size_t)i * Hq + hq) * HD, s + (size_t)h * HD, hadamard, qt);
            attend_row(qt, h, n, Hkv, kx, vx, out + ((size_t)i * Hq + hq) * HD);
        }
}

/* The same attention for queries given already in the keys' basis, in fp64
 * (the dequantised NVFP4 queries of an FP4 Q.K product).
 *   qx: [Tq][Hq][D] fp64; the rest as oracle_attention. */
void oracle_attention_x(const double* qx, int Tq, int q_start, int Hq, int Hkv,
                        const double* kx, const double* vx, int T, double* out)
{
    const int G = Hq / Hkv;
    #pragma omp parallel for collapse(2) schedule(dynamic)
    for (int i = 0; i < Tq; ++i)
        for (int hq = 0; hq < Hq; ++hq) {
            int n = q_start + i + 1;
            if (n > T) n = T;
            attend_row(qx + ((size_t)i * Hq + hq) * HD, hq / G, n, Hkv, kx, vx, out + ((size_t)i * Hq + hq) * HD);
        }
}
