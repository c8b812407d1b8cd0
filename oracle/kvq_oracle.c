/*
 * kvq_oracle.c -- plain, slow CPU oracle for the fused KV-cache
 * rotate-and-quantize path (lambda smooth scale -> random signs ->
 * normalised Walsh-Hadamard transform -> per-group abs-max int4 with fp16
 * group scales -> nibble packing) and its inverse.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file.  It is used by the tests, by the package's smoke check and
 * by the benchmark's CPU-baseline leg, and by nothing else.  It shares no
 * code, header, table or constant with the CUDA path.
 *
 * Sources (the method is described on these pages; no code is printed there):
 *   [P3]  "When Quantization Is Free: An int4 KV Cache That Outruns fp16 on
 *         Apple Silicon" (arXiv 2605.05699), Abstract: one fused kernel does
 *         sign-randomised transform + per-channel lambda + per-group abs-max +
 *         int4 nibble pack; SRFT and SRHT give indistinguishable quality.
 *   [P5]  Same title, technical summary ("Technische Samenvatting"),
 *         Methodologie 1 (fixed random sign vector s, transform of diag(s) x),
 *         Methodologie 2 (kernel steps: load & sign-multiply, transform,
 *         per-channel lambda rescale, per-group absolute-max reduction, round
 *         to signed int4, pack two int4 values per byte),
 *         Methodologie 3 (per-channel + per-group scaling, groups of 16).
 *   [P1]  "The Kernel That Finally Did Something -- And Didn't Quite Agree
 *         With Itself" (VeloxQuant-MLX blog), "What VecInfer does" and "The
 *         kernel toggle": smooth scale is applied before the Hadamard
 *         transform, and the inverse runs dequantize -> inverse transform ->
 *         unscale.
 *
 * Readings taken where the pages are silent (each is also listed in the
 * design notes):
 *   - lambda multiplies x BEFORE the rotation; the inverse divides by lambda
 *     last (order of [P1]; [P5] puts lambda after the transform).
 *   - rotation = SRHT: y = H_D diag(s) (lambda . x) / sqrt(D), H_D the
 *     Sylvester Hadamard matrix H_ij = (-1)^popcount(i & j), s in {+1,-1}^D
 *     ([P3] reports SRHT indistinguishable from the paper's SRFT).
 *   - the unnormalised transform runs radix-2 butterflies with ascending
 *     half-width h = 1, 2, ..., D/2; 1/sqrt(D) is one fp32 multiply after it.
 *   - quantiser: symmetric, scale S = fp16_rne(max|y| / 7), codes
 *     q = clamp(rint(y * (1/S)), -8, 7), rint = round half to even; S = 0
 *     (all codes 0) when the fp16 scale is zero; a scale above the largest
 *     finite fp16 saturates to 65504.
 *   - nibble order: element 2b in the low nibble of byte b, element 2b+1 in
 *     the high nibble, 4-bit two's complement.
 *   - precision: the quantiser's decisions (codes, fp16 scale) are taken in
 *     fp32 with the fixed operation order below, the precision the GPU kernel
 *     uses; the double-precision functions exist to pin the fp32 ones.
 *
 * Compile with -O2 -ffp-contract=off and without -ffast-math: every line
 * below is one IEEE operation with one rounding, in the order written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define KVQO_DMAX 4096

/* ------------------------------------------------------------------ */
/* IEEE binary16 <-> binary32 conversion (round to nearest even).       */
/* ------------------------------------------------------------------ */

uint16_t kvqo_f32_to_f16(float f)
{
    _Float16 h = (_Float16)f;
    uint16_t bits;
    memcpy(&bits, &h, sizeof bits);
    return bits;
}

float kvqo_f16_to_f32(uint16_t bits)
{
    _Float16 h;
    memcpy(&h, &bits, sizeof h);
    return (float)h;
}

/* The normalisation constant: the fp32 value nearest 1/sqrt(D). */
float kvqo_norm_const(int D)
{
    return (float)(1.0 / sqrt((double)D));
}

static int is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

/* Shapes the oracle accepts: D a power of two in [2, KVQO_DMAX],
 * G a power of two with 2 <= G <= D.  Returns 0 if valid. */
static int check_shape(int D, int G)
{
    if (!is_pow2(D) || D < 2 || D > KVQO_DMAX) return -3;
    if (!is_pow2(G) || G < 2 || G > D) return -4;
    return 0;
}

/* ------------------------------------------------------------------ */
/* Unnormalised fast Walsh-Hadamard transform, Sylvester (natural)     */
/* order, radix-2 butterflies with ascending half-width h.             */
/* [P3] Abstract (SRHT); [P5] Methodologie 1.                          */
/* ------------------------------------------------------------------ */

void kvqo_fwht_f64(double *v, int D)
{
    for (int h = 1; h < D; h <<= 1)
        for (int i = 0; i < D; i += 2 * h)
            for (int k = i; k < i + h; ++k) {
                double a = v[k];
                double b = v[k + h];
                v[k] = a + b;
                v[k + h] = a - b;
            }
}

void kvqo_fwht_f32(float *v, int D)
{
    for (int h = 1; h < D; h <<= 1)
        for (int i = 0; i < D; i += 2 * h)
            for (int k = i; k < i + h; ++k) {
                float a = v[k];
                float b = v[k + h];
                v[k] = a + b;
                v[k + h] = a - b;
            }
}

/* ------------------------------------------------------------------ */
/* Double-precision rotation and its inverse, the definitions that pin */
/* the fp32 path:  y = H diag(s) (lambda . x) / sqrt(D)                 */
/*                 x = (diag(s) H y / sqrt(D)) / lambda                */
/* ------------------------------------------------------------------ */

void kvqo_rotate_f64(const double *x, const double *lam, const int8_t *s,
                     int D, double *y)
{
    double inv = 1.0 / sqrt((double)D);
    for (int i = 0; i < D; ++i) y[i] = x[i] * lam[i] * (double)s[i];
    kvqo_fwht_f64(y, D);
    for (int i = 0; i < D; ++i) y[i] *= inv;
}

void kvqo_unrotate_f64(const double *y, const double *lam, const int8_t *s,
                       int D, double *x)
{
    double inv = 1.0 / sqrt((double)D);
    for (int i = 0; i < D; ++i) x[i] = y[i];
    kvqo_fwht_f64(x, D);
    for (int i = 0; i < D; ++i) x[i] = x[i] * inv * (double)s[i] / lam[i];
}

/* ------------------------------------------------------------------ */
/* fp32 forward rotation of one fp16 row (steps: load, lambda & sign,  */
/* transform, normalise).  [P5] Methodologie 2, first two steps;       */
/* lambda before the transform per [P1].                                */
/* ------------------------------------------------------------------ */

static void rotate_row_f32(const uint16_t *x, const float *lam,
                           const int8_t *s, int D, float c, float *y)
{
    for (int i = 0; i < D; ++i) {
        float t = kvqo_f16_to_f32(x[i]) * lam[i];   /* one rounding  */
        y[i] = (s[i] < 0) ? -t : t;                 /* exact         */
    }
    kvqo_fwht_f32(y, D);
    for (int i = 0; i < D; ++i) y[i] = y[i] * c;
}

int kvqo_rotate_f32(const uint16_t *x, const float *lam, const int8_t *s,
                    int64_t n, int D, float *y)
{
    if (!is_pow2(D) || D < 2 || D > KVQO_DMAX || n < 0) return -3;
    float c = kvqo_norm_const(D);
    for (int64_t r = 0; r < n; ++r)
        rotate_row_f32(x + r * D, lam, s, D, c, y + r * D);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Per-group abs-max int4 quantisation of one rotated row.              */
/* [P5] Methodologie 2 ("per-group absolute-max reduction, round to    */
/* signed int4"), Methodologie 3 (per-group scaling).                  */
/* ------------------------------------------------------------------ */

static void quantize_rotated_row(const float *y, int D, int G,
                                 int8_t *q, uint16_t *scales)
{
    for (int j = 0; j < D / G; ++j) {
        const float *yg = y + j * G;
        float a = 0.0f;
        for (int i = 0; i < G; ++i) {
            float m = fabsf(yg[i]);
            if (m > a) a = m;
        }
        uint16_t sb = kvqo_f32_to_f16(a / 7.0f);
        if (sb == 0x7C00u) sb = 0x7BFFu;            /* saturate to 65504 */
        scales[j] = sb;
        float sf = kvqo_f16_to_f32(sb);
        if (sf == 0.0f) {
            for (int i = 0; i < G; ++i) q[j * G + i] = 0;
            continue;
        }
        float r = 1.0f / sf;
        for (int i = 0; i < G; ++i) {
            float t = rintf(yg[i] * r);              /* half to even  */
            if (t > 7.0f) t = 7.0f;
            if (t < -8.0f) t = -8.0f;
            q[j * G + i] = (int8_t)t;
        }
    }
}

/* Codes unpacked, one int8 per element: codes[n][D], scales[n][D/G]
 * (fp16 bit patterns). */
int kvqo_quantize_codes(const uint16_t *x, const float *lam, const int8_t *s,
                        int64_t n, int D, int G, int8_t *codes,
                        uint16_t *scales)
{
    int rc = check_shape(D, G);
    if (rc) return rc;
    if (n < 0) return -5;
    float c = kvqo_norm_const(D);
    float y[KVQO_DMAX];
    for (int64_t r = 0; r < n; ++r) {
        rotate_row_f32(x + r * D, lam, s, D, c, y);
        quantize_rotated_row(y, D, G, codes + r * D, scales + r * (D / G));
    }
    return 0;
}

/* Two int4 codes per byte: element 2b in the low nibble, 2b+1 in the high
 * nibble ([P5] Methodologie 2, last step). */
void kvqo_pack(const int8_t *codes, int64_t count, uint8_t *packed)
{
    for (int64_t b = 0; b < count / 2; ++b) {
        unsigned lo = (unsigned)codes[2 * b] & 0xFu;
        unsigned hi = (unsigned)codes[2 * b + 1] & 0xFu;
        packed[b] = (uint8_t)(lo | (hi << 4));
    }
}

void kvqo_unpack(const uint8_t *packed, int64_t count, int8_t *codes)
{
    for (int64_t b = 0; b < count / 2; ++b) {
        int lo = packed[b] & 0xF;
        int hi = (packed[b] >> 4) & 0xF;
        codes[2 * b] = (int8_t)(lo >= 8 ? lo - 16 : lo);
        codes[2 * b + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
    }
}

/* The whole forward path: packed[n][D/2] bytes, scales[n][D/G] fp16 bits. */
int kvqo_quantize(const uint16_t *x, const float *lam, const int8_t *s,
                  int64_t n, int D, int G, uint8_t *packed, uint16_t *scales)
{
    int rc = check_shape(D, G);
    if (rc) return rc;
    if (n < 0) return -5;
    float c = kvqo_norm_const(D);
    float y[KVQO_DMAX];
    int8_t q[KVQO_DMAX];
    for (int64_t r = 0; r < n; ++r) {
        rotate_row_f32(x + r * D, lam, s, D, c, y);
        quantize_rotated_row(y, D, G, q, scales + r * (D / G));
        kvqo_pack(q, D, packed + r * (D / 2));
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Inverse path: unpack -> times scale -> inverse rotation -> / lambda. */
/* H/sqrt(D) is symmetric and orthogonal, so it is its own inverse, and */
/* diag(s) is its own inverse.  Order per [P1] ("dequantize, inverse    */
/* transform, unscale").  Division by lambda is a multiply by the fp32  */
/* reciprocal 1/lambda.                                                 */
/* ------------------------------------------------------------------ */

static void dequantize_row(const int8_t *q, const uint16_t *scales,
                           const float *lam, const int8_t *s, int D, int G,
                           float c, float *w)
{
    for (int i = 0; i < D; ++i)
        w[i] = (float)q[i] * kvqo_f16_to_f32(scales[i / G]);   /* exact */
    kvqo_fwht_f32(w, D);
    for (int i = 0; i < D; ++i) {
        float z = w[i] * c;
        float zs = (s[i] < 0) ? -z : z;                         /* exact */
        float il = 1.0f / lam[i];
        w[i] = zs * il;
    }
}

int kvqo_dequantize(const uint8_t *packed, const uint16_t *scales,
                    const float *lam, const int8_t *s, int64_t n, int D,
                    int G, uint16_t *out)
{
    int rc = check_shape(D, G);
    if (rc) return rc;
    if (n < 0) return -5;
    float c = kvqo_norm_const(D);
    int8_t q[KVQO_DMAX];
    float w[KVQO_DMAX];
    for (int64_t r = 0; r < n; ++r) {
        kvqo_unpack(packed + r * (D / 2), D, q);
        dequantize_row(q, scales + r * (D / G), lam, s, D, G, c, w);
        for (int i = 0; i < D; ++i) out[r * D + i] = kvqo_f32_to_f16(w[i]);
    }
    return 0;
}

/* The inverse without the final fp16 rounding (fp32 output), from codes. */
int kvqo_dequantize_f32(const int8_t *codes, const uint16_t *scales,
                        const float *lam, const int8_t *s, int64_t n, int D,
                        int G, float *out)
{
    int rc = check_shape(D, G);
    if (rc) return rc;
    if (n < 0) return -5;
    float c = kvqo_norm_const(D);
    for (int64_t r = 0; r < n; ++r)
        dequantize_row(codes + r * D, scales + r * (D / G), lam, s, D, G, c,
                       out + r * D);
    return 0;
}

/* fp32 inverse rotation of rotated rows (no quantisation): y -> x. */
int kvqo_unrotate_f32(const float *y, const float *lam, const int8_t *s,
                      int64_t n, int D, float *x)
{
    if (!is_pow2(D) || D < 2 || D > KVQO_DMAX || n < 0) return -3;
    float c = kvqo_norm_const(D);
    for (int64_t r = 0; r < n; ++r) {
        float *w = x + r * D;
        for (int i = 0; i < D; ++i) w[i] = y[r * D + i];
        kvqo_fwht_f32(w, D);
        for (int i = 0; i < D; ++i) {
            float z = w[i] * c;
            float zs = (s[i] < 0) ? -z : z;
            w[i] = zs * (1.0f / lam[i]);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Textbook cross-check form of the quantiser: codes = rint(y / S) with */
/* an IEEE division per element instead of a multiply by 1/S.  Used    */
/* only to show that the two forms disagree at near-ties alone.        */
/* ------------------------------------------------------------------ */

int kvqo_quantize_codes_divform(const uint16_t *x, const float *lam,
                                const int8_t *s, int64_t n, int D, int G,
                                int8_t *codes)
{
    int rc = check_shape(D, G);
    if (rc) return rc;
    float c = kvqo_norm_const(D);
    float y[KVQO_DMAX];
    for (int64_t r = 0; r < n; ++r) {
        rotate_row_f32(x + r * D, lam, s, D, c, y);
        for (int j = 0; j < D / G; ++j) {
            float a = 0.0f;
            for (int i = 0; i < G; ++i) {
                float m = fabsf(y[j * G + i]);
                if (m > a) a = m;
            }
            uint16_t sb = kvqo_f32_to_f16(a / 7.0f);
            if (sb == 0x7C00u) sb = 0x7BFFu;
            float sf = kvqo_f16_to_f32(sb);
            for (int i = 0; i < G; ++i) {
                float t = (sf == 0.0f) ? 0.0f : rintf(y[j * G + i] / sf);
                if (t > 7.0f) t = 7.0f;
                if (t < -8.0f) t = -8.0f;
                codes[r * D + j * G + i] = (int8_t)t;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Decode attention over the int4 cache: one query token per sequence.  */
/* [P1] "Fused group-affine (KIVI-style) attention": the quantised K    */
/* and V are reconstructed and attended with a numerically stable       */
/* softmax in place of a dequantize -> memory -> SDPA round trip.  This */
/* is the plain definition the fused kernel has to reproduce, in double */
/* precision and without rounding the reconstructed rows to fp16:       */
/*   K_t = (diag(s_K) H (codes_t . S_t) / sqrt(D)) / lambda_K, V_t      */
/*   likewise with (lambda_V, s_V);                                     */
/*   z_t = sm_scale <q, K_t>;  p = softmax(z) over t < len;             */
/*   o = sum_t p_t V_t.                                                 */
/* Query head h reads KV head h / (Hq / Hkv) (grouped-query attention). */
/* An empty context (len = 0) gives o = 0.                               */
/* Layouts: q fp16 [B][Hq][D]; packed u8 [B][Hkv][T][D/2]; scales fp16  */
/* [B][Hkv][T][D/G]; seq_len [B]; out double [B][Hq][D].                */
/* ------------------------------------------------------------------ */

void kvqo_isrft_f64(const double *y, int D, double *v);   /* below */
static int srft_len_ok(int D);

/* One reconstructed row in double: codes times scales, then the exact   */
/* inverse of the row's rotation (flags as for the codec variants: bit 0 */
/* lambda after the rotation, bit 1 the SRFT):                           */
/*   lambda before: x = (diag(s) R^T y) / lambda,                        */
/*   lambda after:  x = diag(s) R^T (y / lambda),                        */
/* R^T = H / sqrt(D) (Walsh-Hadamard) or P^T (the SRFT's packed unitary  */
/* DFT, transposed).                                                     */
static void reconstruct_row_f64(const uint8_t *packed, const uint16_t *scales,
                                const double *lam, const int8_t *s, int D,
                                int G, int flags, double *x)
{
    int8_t q[KVQO_DMAX];
    double y[KVQO_DMAX];
    kvqo_unpack(packed, D, q);
    for (int i = 0; i < D; ++i)
        y[i] = (double)q[i] * (double)kvqo_f16_to_f32(scales[i / G]);
    if (flags == 0) {
        kvqo_unrotate_f64(y, lam, s, D, x);
        return;
    }
    if (flags & 1)
        for (int i = 0; i < D; ++i) y[i] /= lam[i];
    if (flags & 2) {
        kvqo_isrft_f64(y, D, x);
    } else {
        double inv = 1.0 / sqrt((double)D);
        for (int i = 0; i < D; ++i) x[i] = y[i];
        kvqo_fwht_f64(x, D);
        for (int i = 0; i < D; ++i) x[i] *= inv;
    }
    for (int i = 0; i < D; ++i) {
        x[i] *= (double)s[i];
        if (!(flags & 1)) x[i] /= lam[i];
    }
}

int kvqo_attention_decode_ex(const uint16_t *q, const uint8_t *k_packed,
                             const uint16_t *k_scales, const uint8_t *v_packed,
                             const uint16_t *v_scales, const int32_t *seq_len,
                             const float *lam_k, const int8_t *s_k,
                             const float *lam_v, const int8_t *s_v, int B,
                             int Hq, int Hkv, int T, int D, int G, int flags,
                             double sm_scale, double *out)
{
    int rc = (flags & 2) ? (srft_len_ok(D) ? 0 : -3) : check_shape(D, G);
    if (rc) return rc;
    if (!is_pow2(G) || G < 2 || G > D || D % G != 0) return -4;
    if (flags & ~3) return -4;
    if (B < 0 || T < 0 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0) return -5;
    for (int b = 0; b < B; ++b)
        if (seq_len[b] < 0 || seq_len[b] > T) return -5;
    int R = Hq / Hkv;
    double lk[KVQO_DMAX], lv[KVQO_DMAX], qd[KVQO_DMAX], row[KVQO_DMAX];
    for (int i = 0; i < D; ++i) {
        lk[i] = (double)lam_k[i];
        lv[i] = (double)lam_v[i];
    }
    double *z = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (z == NULL) return -6;
    for (int b = 0; b < B; ++b) {
        int len = seq_len[b];
        for (int h = 0; h < Hq; ++h) {
            int kv = h / R;
            int64_t base = ((int64_t)b * Hkv + kv) * T;
            double *o = out + ((int64_t)b * Hq + h) * D;
            for (int i = 0; i < D; ++i) {
                qd[i] = (double)kvqo_f16_to_f32(q[((int64_t)b * Hq + h) * D + i]);
                o[i] = 0.0;
            }
            if (len == 0) continue;
            double m = -INFINITY;
            for (int t = 0; t < len; ++t) {
                reconstruct_row_f64(k_packed + (base + t) * (D / 2),
                                    k_scales + (base + t) * (D / G), lk, s_k,
                                    D, G, flags, row);
                double dot = 0.0;
                for (int i = 0; i < D; ++i) dot += qd[i] * row[i];
                z[t] = sm_scale * dot;
                if (z[t] > m) m = z[t];
            }
            double l = 0.0;
            for (int t = 0; t < len; ++t) {
                double p = exp(z[t] - m);
                l += p;
                reconstruct_row_f64(v_packed + (base + t) * (D / 2),
                                    v_scales + (base + t) * (D / G), lv, s_v,
                                    D, G, flags, row);
                for (int i = 0; i < D; ++i) o[i] += p * row[i];
            }
            for (int i = 0; i < D; ++i) o[i] /= l;
        }
    }
    free(z);
    return 0;
}

/* The base cache format: Walsh-Hadamard rows, lambda before the rotation. */
int kvqo_attention_decode(const uint16_t *q, const uint8_t *k_packed,
                          const uint16_t *k_scales, const uint8_t *v_packed,
                          const uint16_t *v_scales, const int32_t *seq_len,
                          const float *lam_k, const int8_t *s_k,
                          const float *lam_v, const int8_t *s_v, int B, int Hq,
                          int Hkv, int T, int D, int G, double sm_scale,
                          double *out)
{
    return kvqo_attention_decode_ex(q, k_packed, k_scales, v_packed, v_scales,
                                    seq_len, lam_k, s_k, lam_v, s_v, B, Hq, Hkv,
                                    T, D, G, 0, sm_scale, out);
}

/* ------------------------------------------------------------------ */
/* The SRFT rotation: SRFT(x) = pack(F diag(s) x), F the unitary DFT    */
/* of length D ([P5] Methodologie 1), computed as the paper's kernel    */
/* does ([P5] Methodologie 2): the length-N = D/2 complex FFT of        */
/* z_n = v_2n + i v_2n+1 in Stockham stages, then the Hermitian         */
/* unpacking to a real representation.  [P3] picks the SRFT for mixed  */
/* radix, so N is a power of two (log2 N radix-2 stages) or three times */
/* one (radix-2 stages, then one radix-3 stage).  The packing read      */
/* here (orthonormal, so the inverse is the transpose):                 */
/*   y0 = X_0 / sqrt(D),  y1 = X_N / sqrt(D),                            */
/*   (y_2k, y_2k+1) = sqrt(2) (Re, Im) X_k / sqrt(D),  k = 1 .. N-1,     */
/* X = DFT(v).  Readings of the arithmetic:                             */
/*  - twiddles are the fp32 values nearest the exact roots of unity;    */
/*    a product by 1, -1, i or -i is exact (the operand, negated or     */
/*    with its parts swapped); in any other complex product each part   */
/*    is one rounded product and one fused multiply-add:                */
/*    re = fma(dr, wr, -rn(di wi)), im = fma(di, wr, rn(dr wi));        */
/*  - the unpacking forms 2 X_k (its factor 1/2 goes into the           */
/*    normalisation), scaled by fp32(1/sqrt(2D)); X_0 and X_N are       */
/*    scaled by fp32(1/sqrt(D));                                        */
/*  - the inverse is the transpose of the forward, step by step in      */
/*    reverse order: the scaling, the adjoint of the unpacking, then    */
/*    the adjoint (decimation-in-time) Stockham stages with conjugate   */
/*    twiddles.                                                         */
/* ------------------------------------------------------------------ */

/* omega_M^k = (cos(2 pi k / M), -sin(2 pi k / M)) as the fp32 values
 * nearest the exact ones.  The angle is reduced by exact symmetries to a
 * base angle (pi/2) r / M with 0 <= r <= M/2 (at most pi/4), whose cosine
 * and sine are taken in double and rounded once; quadrant and complement
 * are exact swaps and negations.  So omega^0 = 1, omega^(M/4) = -i and
 * omega^(M/2) = -1 exactly, the table keeps every symmetry of the exact
 * roots, and its zero parts are +0. */
void kvqo_twiddle(int k, int M, float *wr, float *wi)
{
    long j = ((long)k % M + M) % M;
    long q = (4 * j) / M;                       /* quadrant */
    long r = 4 * j - q * M;                     /* angle = q pi/2 + (pi/2) r / M */
    int comp = 2 * r > M;
    if (comp) r = M - r;
    double a = 1.57079632679489661923 * (double)r / (double)M;
    float c = (float)cos(a), s = (float)sin(a);
    if (comp) { float t = c; c = s; s = t; }    /* cos, sin of (pi/2) r_0 / M */
    float cr, sn;                               /* cos, sin of the whole angle */
    switch (q) {
    case 0: cr = c; sn = s; break;
    case 1: cr = -s; sn = c; break;
    case 2: cr = -c; sn = -s; break;
    default: cr = s; sn = -c; break;
    }
    *wr = cr + 0.0f;                            /* -0 -> +0 */
    *wi = -sn + 0.0f;
}

/* d * w for a table twiddle w (readings above). */
static void cmul(float dr, float di, float wr, float wi, float *pr, float *pi_)
{
    if (wi == 0.0f && fabsf(wr) == 1.0f) {              /* w = +-1 */
        *pr = (wr > 0.0f) ? dr : -dr;
        *pi_ = (wr > 0.0f) ? di : -di;
    } else if (wr == 0.0f && fabsf(wi) == 1.0f) {       /* w = +-i: (dr + i di)(i wi) */
        *pr = (wi > 0.0f) ? -di : di;
        *pi_ = (wi > 0.0f) ? dr : -dr;
    } else {
        float b = di * wi, c = dr * wi;                 /* rounded products */
        *pr = fmaf(dr, wr, -b);                         /* dr wr - di wi */
        *pi_ = fmaf(di, wr, c);                         /* di wr + dr wi */
    }
}

/* Radices of a length-N transform, first stage first: 2 while the remaining
 * length is even, then 3 if it is 3.  Returns the number of stages, or -1
 * for another N. */
static int fft_radices(int N, int *rad)
{
    int n = N, ns = 0;
    if (N < 1) return -1;
    while (n % 2 == 0) { rad[ns++] = 2; n /= 2; }
    if (n == 3) { rad[ns++] = 3; n = 1; }
    return n == 1 ? ns : -1;
}

/* One forward (decimation-in-frequency) Stockham stage of radix r on
 * sub-transforms of length n, stride s = N / n, m = n / r:
 *   a_j = x[q + s (p + j m)],  j < r,
 *   y[q + s (r p + t)] = (a_0 + omega_r^t a_1 + ... ) omega_n^(p t),
 * the sum taken left to right over j.  At r = 2 that is a + b and
 * (a - b) omega_n^p. */
static void dif_stage(const float *xr, const float *xi, float *yr, float *yi,
                      int N, int n, int r)
{
    int s = N / n, m = n / r;
    for (int p = 0; p < m; ++p)
        for (int q = 0; q < s; ++q)
            for (int t = 0; t < r; ++t) {
                float br = xr[q + s * p], bi = xi[q + s * p];
                for (int j = 1; j < r; ++j) {
                    float wr, wi, tr, ti;
                    kvqo_twiddle((N / r) * j * t, N, &wr, &wi);     /* omega_r^(j t) */
                    cmul(xr[q + s * (p + j * m)], xi[q + s * (p + j * m)], wr, wi, &tr, &ti);
                    br = br + tr;
                    bi = bi + ti;
                }
                float wr, wi;
                kvqo_twiddle(s * p * t, N, &wr, &wi);               /* omega_n^(p t) */
                cmul(br, bi, wr, wi, &yr[q + s * (r * p + t)], &yi[q + s * (r * p + t)]);
            }
}

/* The transpose of dif_stage: c_t = y[q + s (r p + t)] conj(omega_n^(p t)),
 * x[q + s (p + j m)] = c_0 + conj(omega_r^j) c_1 + ..., left to right over
 * t.  At r = 2 that is x = c_0 + c_1 and c_0 - c_1 with
 * c_1 = y_odd conj(omega_n^p). */
static void dit_stage(const float *yr, const float *yi, float *xr, float *xi,
                      int N, int n, int r)
{
    int s = N / n, m = n / r;
    for (int p = 0; p < m; ++p)
        for (int q = 0; q < s; ++q) {
            float cr[3], ci[3];
            for (int t = 0; t < r; ++t) {
                float wr, wi;
                kvqo_twiddle(s * p * t, N, &wr, &wi);
                cmul(yr[q + s * (r * p + t)], yi[q + s * (r * p + t)], wr, -wi, &cr[t], &ci[t]);
            }
            for (int j = 0; j < r; ++j) {
                float ar = cr[0], ai = ci[0];
                for (int t = 1; t < r; ++t) {
                    float wr, wi, tr, ti;
                    kvqo_twiddle((N / r) * j * t, N, &wr, &wi);
                    cmul(cr[t], ci[t], wr, -wi, &tr, &ti);
                    ar = ar + tr;
                    ai = ai + ti;
                }
                xr[q + s * (p + j * m)] = ar;
                xi[q + s * (p + j * m)] = ai;
            }
        }
}

/* Length-N complex FFT in place (through a scratch copy), N a power of two
 * or three times one.  inverse = 0: the forward DIF stages (the unnormalised
 * DFT X_k = sum_n z_n omega_N^(n k)); inverse = 1: its transpose, the
 * adjoint stages in reverse order (the unnormalised conjugate DFT).
 * Returns 0, or -3 for an unsupported N. */
int kvqo_fft_f32(float *re, float *im, int N, int inverse)
{
    int rad[32], len[33];
    int ns = fft_radices(N, rad);
    if (ns < 0 || N > KVQO_DMAX / 2) return -3;
    len[0] = N;
    for (int i = 0; i < ns; ++i) len[i + 1] = len[i] / rad[i];
    float tr[KVQO_DMAX / 2], ti[KVQO_DMAX / 2];
    float *xr = re, *xi = im, *yr = tr, *yi = ti;
    for (int i = 0; i < ns; ++i) {
        int st = inverse ? ns - 1 - i : i;
        if (inverse)
            dit_stage(xr, xi, yr, yi, N, len[st], rad[st]);
        else
            dif_stage(xr, xi, yr, yi, N, len[st], rad[st]);
        float *t;
        t = xr; xr = yr; yr = t;
        t = xi; xi = yi; yi = t;
    }
    if (xr != re) {
        for (int i = 0; i < N; ++i) { re[i] = xr[i]; im[i] = xi[i]; }
    }
    return 0;
}

/* 2 X_k and 2 X_(N-k) of the real input from its half-length spectrum Z,
 * for a pair 1 <= k <= N/2 (one bin at k = N/2):  A = Z_k, B = conj Z_(N-k),
 * E = A + B, O = (A - B) / i (exact), T = omega_D^k O,
 *   2 X_k = E + T,   2 X_(N-k) = conj(E - T)
 * (the Hermitian symmetry of a real input's spectrum: both bins of a pair
 * share E, O and T).  x[0..3] = re, im of 2 X_k, then of 2 X_(N-k). */
static void real_pair2(const float *zr, const float *zi, int N, int k, float *x)
{
    float Ar = zr[k], Ai = zi[k], Br = zr[N - k], Bi = -zi[N - k];
    float Er = Ar + Br, Ei = Ai + Bi;
    float Dr = Ar - Br, Di = Ai - Bi;
    float Or = Di, Oi = -Dr;
    float wr, wi, Tr, Ti;
    kvqo_twiddle(k, 2 * N, &wr, &wi);
    cmul(Or, Oi, wr, wi, &Tr, &Ti);
    x[0] = Er + Tr;
    x[1] = Ei + Ti;
    float Wr = Er - Tr, Wi = Ei - Ti;
    x[2] = Wr;
    x[3] = -Wi;
}

/* Is D an SRFT length: even, D/2 a power of two or three times one. */
static int srft_len_ok(int D)
{
    int rad[32];
    return D >= 2 && D % 2 == 0 && D <= KVQO_DMAX && fft_radices(D / 2, rad) >= 0;
}

/* Normalisation of packed position i: fp32(1/sqrt(D)) on y0, y1 (X_0, X_N),
 * fp32(1/sqrt(2D)) on the rest (which hold 2 Re X_k, 2 Im X_k). */
static float srft_norm(int i, int D)
{
    return (i < 2) ? (float)(1.0 / sqrt((double)D)) : (float)(1.0 / sqrt(2.0 * (double)D));
}

/* Forward SRFT of one sign-flipped row v[D] with per-position factors f:
 * y0 = (Z0.re + Z0.im) f0, y1 = (Z0.re - Z0.im) f1 (X_0 and X_N),
 * (y_2k, y_2k+1) = 2 X_k . (f_2k, f_2k+1), the bins formed in pairs. */
static void srft_scaled(const float *v, int D, const float *f, float *y)
{
    int N = D / 2;
    float zr[KVQO_DMAX / 2], zi[KVQO_DMAX / 2];
    for (int n = 0; n < N; ++n) { zr[n] = v[2 * n]; zi[n] = v[2 * n + 1]; }
    kvqo_fft_f32(zr, zi, N, 0);
    y[0] = (zr[0] + zi[0]) * f[0];
    y[1] = (zr[0] - zi[0]) * f[1];
    for (int k = 1; 2 * k <= N; ++k) {
        float x[4];
        real_pair2(zr, zi, N, k, x);
        y[2 * k] = x[0] * f[2 * k];
        y[2 * k + 1] = x[1] * f[2 * k + 1];
        if (2 * k < N) {
            y[2 * (N - k)] = x[2] * f[2 * (N - k)];
            y[2 * (N - k) + 1] = x[3] * f[2 * (N - k) + 1];
        }
    }
}

/* Transpose of srft_scaled: U_i = y_i f_i; the adjoint of the unpacking,
 * z_0 = (U_0 + U_1, U_0 - U_1) and, for a pair 1 <= k <= N/2 (one bin at
 * k = N/2), A = U_k, B = conj U_(N-k), E = A + B, T = (A - B) conj(omega_D^k),
 *   Z_k = E + i T,   Z_(N-k) = conj(E - i T);
 * then the transposed FFT. */
static void isrft_scaled(const float *y, int D, const float *f, float *v)
{
    int N = D / 2;
    float zr[KVQO_DMAX / 2], zi[KVQO_DMAX / 2];
    float u0 = y[0] * f[0], un = y[1] * f[1];
    zr[0] = u0 + un;
    zi[0] = u0 - un;
    for (int k = 1; 2 * k <= N; ++k) {
        float Ar = y[2 * k] * f[2 * k], Ai = y[2 * k + 1] * f[2 * k + 1];
        float Br = y[2 * (N - k)] * f[2 * (N - k)];
        float Bi = -(y[2 * (N - k) + 1] * f[2 * (N - k) + 1]);
        float Er = Ar + Br, Ei = Ai + Bi;
        float Dr = Ar - Br, Di = Ai - Bi;
        float wr, wi, Tr, Ti;
        kvqo_twiddle(k, D, &wr, &wi);
        cmul(Dr, Di, wr, -wi, &Tr, &Ti);                 /* conj(omega_D^k) */
        zr[k] = Er - Ti;                                  /* E + i T */
        zi[k] = Ei + Tr;
        if (2 * k < N) {
            float Wr = Er + Ti, Wi = Ei - Tr;             /* E - i T */
            zr[N - k] = Wr;
            zi[N - k] = -Wi;
        }
    }
    kvqo_fft_f32(zr, zi, N, 1);
    for (int n = 0; n < N; ++n) { v[2 * n] = zr[n]; v[2 * n + 1] = zi[n]; }
}

/* fp32 SRFT of one sign-flipped row v[D] -> y[D] (normalised). */
int kvqo_srft_f32(const float *v, int D, float *y)
{
    float f[KVQO_DMAX];
    if (!srft_len_ok(D)) return -3;
    for (int i = 0; i < D; ++i) f[i] = srft_norm(i, D);
    srft_scaled(v, D, f, y);
    return 0;
}

/* fp32 inverse SRFT (the transpose): y[D] -> v[D] = P^T y. */
int kvqo_isrft_f32(const float *y, int D, float *v)
{
    float f[KVQO_DMAX];
    if (!srft_len_ok(D)) return -3;
    for (int i = 0; i < D; ++i) f[i] = srft_norm(i, D);
    isrft_scaled(y, D, f, v);
    return 0;
}

/* Definitions in double, for the pins: the packed unitary DFT and its
 * transpose, by direct sums. */
void kvqo_srft_f64(const double *v, int D, double *y)
{
    int N = D / 2;
    for (int k = 0; k <= N; ++k) {
        double xr = 0.0, xi = 0.0;
        for (int n = 0; n < D; ++n) {
            double a = 2.0 * 3.14159265358979323846 * (double)k * (double)n / (double)D;
            xr += v[n] * cos(a);
            xi -= v[n] * sin(a);
        }
        if (k == 0) y[0] = xr / sqrt((double)D);
        else if (k == N) y[1] = xr / sqrt((double)D);
        else { y[2 * k] = xr * sqrt(2.0 / D); y[2 * k + 1] = xi * sqrt(2.0 / D); }
    }
}

void kvqo_isrft_f64(const double *y, int D, double *v)
{
    int N = D / 2;
    for (int n = 0; n < D; ++n) {
        double acc = y[0] / sqrt((double)D) + y[1] * ((n & 1) ? -1.0 : 1.0) / sqrt((double)D);
        for (int k = 1; k < N; ++k) {
            double a = 2.0 * 3.14159265358979323846 * (double)k * (double)n / (double)D;
            acc += sqrt(2.0 / D) * (y[2 * k] * cos(a) - y[2 * k + 1] * sin(a));
        }
        v[n] = acc;
    }
}

/* ------------------------------------------------------------------ */
/* Format variants of the codec: lambda after the rotation, the SRFT,  */
/* 8-bit codes, and one lambda table per range of rows.  flags:         */
/*   bit 0 (lambda after) 0: y = R (lambda . x), as above;              */
/*                        1: y = lambda . (R x), the paper's order      */
/*                   ([P5] Methodologie 2: transform of diag(s) x,      */
/*                   then the per-channel lambda rescale);              */
/*   bit 1 (SRFT)  R = H diag(s) / sqrt(D) (0) or the SRFT pack(F       */
/*                 diag(s) .) above (1);                                */
/*   bits 4: codes in [-8, 7], S = fp16(max|y| / 7), nibbles packed     */
/*           as kvqo_pack;                                              */
/*   bits 8: codes in [-128, 127], S = fp16(max|y| / 127), one two's-   */
/*           complement byte per code;                                  */
/*   row r uses lambda table (r / lambda_rows) % n_lambda, a table      */
/*   being D floats (per-(layer, head) smoothing).                      */
/* With lambda after the rotation, the rescale after the transform is   */
/* the only scaling step ([P5] Methodologie 2 lists no other): channel  */
/* i is multiplied by fp32(lambda_i c_i), c_i the normalisation of that */
/* position (1/sqrt(D), or the SRFT's), one product per channel; the    */
/* inverse multiplies q S by fp32(c_i / lambda_i) before its transform  */
/* and applies the signs last.  With lambda before it the transform is  */
/* followed by c_i, and the inverse mirrors that (c_i, transform, signs,*/
/* 1/lambda).                                                            */
/* ------------------------------------------------------------------ */

/* D a power of two in [2, KVQO_DMAX] (an SRFT length with the SRFT),
 * G a power of two with 2 <= G <= D dividing D.  Returns 0 if valid. */
static int check_ex(int D, int G, int bits, int64_t lambda_rows, int n_lambda, int srft)
{
    if (srft ? !srft_len_ok(D) : (!is_pow2(D) || D < 2 || D > KVQO_DMAX)) return -3;
    if (!is_pow2(G) || G < 2 || G > D || D % G != 0) return -4;
    if (bits != 4 && bits != 8) return -4;
    if (lambda_rows < 1 || n_lambda < 1) return -5;
    return 0;
}

static const float *table_of(const float *lam, int64_t r, int64_t lambda_rows,
                             int n_lambda, int D)
{
    return lam + ((r / lambda_rows) % n_lambda) * (int64_t)D;
}

/* Normalisation of position i of a rotated row. */
static float norm_of(int i, int D, int srft)
{
    return srft ? srft_norm(i, D) : kvqo_norm_const(D);
}

int kvqo_quantize_ex(const uint16_t *x, const float *lam, const int8_t *s,
                     int64_t n, int D, int G, int bits, int flags,
                     int64_t lambda_rows, int n_lambda, uint8_t *codes,
                     uint16_t *scales)
{
    const int lambda_after = flags & 1, srft = (flags >> 1) & 1;
    int rc = check_ex(D, G, bits, lambda_rows, n_lambda, srft);
    if (rc) return rc;
    if (n < 0) return -5;
    float c = kvqo_norm_const(D);
    float qmax = (bits == 4) ? 7.0f : 127.0f;
    float qmin = (bits == 4) ? -8.0f : -128.0f;
    int row_bytes = (bits == 4) ? D / 2 : D;
    float y[KVQO_DMAX];
    int8_t q[KVQO_DMAX];
    for (int64_t r = 0; r < n; ++r) {
        const uint16_t *xr = x + r * D;
        const float *lr = table_of(lam, r, lambda_rows, n_lambda, D);
        if (!lambda_after && !srft) {
            rotate_row_f32(xr, lr, s, D, c, y);
        } else {
            float v[KVQO_DMAX], f[KVQO_DMAX];
            for (int i = 0; i < D; ++i) {
                float t = kvqo_f16_to_f32(xr[i]);
                if (!lambda_after) t = t * lr[i];              /* lambda */
                v[i] = (s[i] < 0) ? -t : t;                    /* exact  */
                f[i] = lambda_after ? lr[i] * norm_of(i, D, srft)   /* lambda c_i */
                                    : norm_of(i, D, srft);
            }
            if (srft) {
                srft_scaled(v, D, f, y);
            } else {
                kvqo_fwht_f32(v, D);
                for (int i = 0; i < D; ++i) y[i] = v[i] * f[i];
            }
        }
        uint16_t *sc = scales + r * (D / G);
        for (int j = 0; j < D / G; ++j) {
            const float *yg = y + j * G;
            float a = 0.0f;
            for (int i = 0; i < G; ++i) {
                float m = fabsf(yg[i]);
                if (m > a) a = m;
            }
            uint16_t sb = kvqo_f32_to_f16(a / qmax);
            if (sb == 0x7C00u) sb = 0x7BFFu;
            sc[j] = sb;
            float sf = kvqo_f16_to_f32(sb);
            float rcp = (sf == 0.0f) ? 0.0f : 1.0f / sf;
            for (int i = 0; i < G; ++i) {
                float t = (sf == 0.0f) ? 0.0f : rintf(yg[i] * rcp);
                if (t > qmax) t = qmax;
                if (t < qmin) t = qmin;
                q[j * G + i] = (int8_t)t;
            }
        }
        uint8_t *cr = codes + r * row_bytes;
        if (bits == 4)
            kvqo_pack(q, D, cr);
        else
            for (int i = 0; i < D; ++i) cr[i] = (uint8_t)q[i];
    }
    return 0;
}

int kvqo_dequantize_ex(const uint8_t *codes, const uint16_t *scales,
                       const float *lam, const int8_t *s, int64_t n, int D,
                       int G, int bits, int flags, int64_t lambda_rows,
                       int n_lambda, uint16_t *out)
{
    const int lambda_after = flags & 1, srft = (flags >> 1) & 1;
    int rc = check_ex(D, G, bits, lambda_rows, n_lambda, srft);
    if (rc) return rc;
    if (n < 0) return -5;
    float c = kvqo_norm_const(D);
    int row_bytes = (bits == 4) ? D / 2 : D;
    int8_t q[KVQO_DMAX];
    float w[KVQO_DMAX];
    for (int64_t r = 0; r < n; ++r) {
        const uint8_t *cr = codes + r * row_bytes;
        const float *lr = table_of(lam, r, lambda_rows, n_lambda, D);
        if (bits == 4)
            kvqo_unpack(cr, D, q);
        else
            for (int i = 0; i < D; ++i) q[i] = (int8_t)cr[i];
        const uint16_t *sc = scales + r * (D / G);
        if (!lambda_after && !srft) {
            dequantize_row(q, sc, lr, s, D, G, c, w);
        } else {
            float u[KVQO_DMAX], f[KVQO_DMAX];
            for (int i = 0; i < D; ++i) {
                u[i] = (float)q[i] * kvqo_f16_to_f32(sc[i / G]);      /* exact */
                f[i] = lambda_after ? norm_of(i, D, srft) / lr[i]     /* c_i / lambda */
                                    : norm_of(i, D, srft);
            }
            if (srft) {
                isrft_scaled(u, D, f, w);
            } else {
                for (int i = 0; i < D; ++i) w[i] = u[i] * f[i];
                kvqo_fwht_f32(w, D);
            }
            for (int i = 0; i < D; ++i) {
                float z = (s[i] < 0) ? -w[i] : w[i];                   /* exact */
                w[i] = lambda_after ? z : z * (1.0f / lr[i]);
            }
        }
        for (int i = 0; i < D; ++i) out[r * D + i] = kvqo_f32_to_f16(w[i]);
    }
    return 0;
}
