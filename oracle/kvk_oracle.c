/*
 * kvk_oracle.c -- CPU oracle for the KV-Kaizen compressed MLA cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or constant with the CUDA library in
 * compressed_decode_attention_kvk_b200/csrc, and it never reads anything the
 * CUDA library produced: it quantises the original inputs itself.
 *
 * It is deliberately plain: one token, one element, one head at a time, in the
 * order the method states it.  Built with -O2 -ffp-contract=off (no fused
 * multiply-add, no fast-math) so that every float operation below is one IEEE
 * binary32 or binary64 operation with round-to-nearest-even.
 *
 * What it follows (KV-Kaizen: Learning Context-Adaptive Cache Compression
 * Choices, picx.dev whiteboard summary):
 *   - "Three Non-Eviction Compression Axes", item 2 (rank): the cached MLA
 *     vector is the latent c^KV truncated to its first d coordinates plus the
 *     decoupled RoPE key k^R of width d_R.
 *   - same section, item 3 (precision): symmetric uniform quantisation to
 *     b <= 16 bits with one scale per token.
 *   - same section, item 1 (depth): inheriting layers read the nearest
 *     anchor's cache (handled by the caller: it passes the anchor's rows).
 *   - "Action Space and Cost Model": c(inherit)=0, c(d,b)=(d+d_R)*b bits per
 *     token, C_0 = L * 2 * n_kv * d_h * 16.
 *   - "Background: The KV Cache Bottleneck": every decoded token reads the
 *     whole cache -> decode attention over all cached (or kept) tokens.
 * Where the pages are silent the readings below are used (each is listed with
 * its reason in the design notes of this repository):
 *   R1  one scale per token per anchor layer, shared by c[:d] and k^R;
 *   R2  scale = fp16( fp32(absmax) / fp32(2^(b-1)-1) ) rounded toward +inf,
 *       codes use the stored (fp16) scale;
 *   R3  codes = clamp(round_half_even(fp32(v / s)), -q, q), q = 2^(b-1)-1;
 *       a zero scale (all-zero token) gives all-zero codes;
 *   R4  stored field u = code + 2^(b-1) (offset binary), element i at bit
 *       i*b of the row read as a little-endian bit stream, rows zero-padded
 *       to a multiple of 16 bytes, scales in a separate fp16 plane;
 *   R5  decode uses the absorbed MLA form: z_t = sigma * (q_lat . c_hat_t[:d]
 *       + q_rope . kR_hat_t), p = softmax(z), out = sum_t p_t c_hat_t[:d],
 *       lse = log sum_t exp(z_t); an empty token set gives out = 0,
 *       lse = -inf;
 *   R6  bits per token = sum over anchor layers of ((d+d_R)*b + 16): the +16
 *       is the fp16 scale of R1/R2.
 */
#include <stdint.h>
#include <stddef.h>
#include <math.h>
#include <fenv.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* IEEE binary16 helpers written from the format's definition:               */
/* 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits; exponent field 0  */
/* holds subnormals with quantum 2^-24; field 31 holds inf/NaN.               */
/* ------------------------------------------------------------------------ */

double kvko_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int f = h & 1023;
    double mag;
    if (e == 0) {
        mag = ldexp((double)f, -24);
    } else if (e == 31) {
        mag = (f == 0) ? INFINITY : NAN;
    } else {
        mag = ldexp(1.0 + (double)f / 1024.0, e - 15);
    }
    return sign ? -mag : mag;
}

/* Encode a non-negative double that is exactly representable in binary16
 * (or is +inf) into its bit pattern. */
static uint16_t encode_f16_exact(double v)
{
    if (isinf(v)) return 0x7C00;
    if (v == 0.0) return 0;
    if (v < ldexp(1.0, -14)) {
        /* subnormal: v = f * 2^-24 */
        return (uint16_t)(v / ldexp(1.0, -24));
    }
    int ex;
    double m = frexp(v, &ex);       /* v = m * 2^ex, m in [0.5, 1) */
    int e = ex - 1;                 /* v = (2m) * 2^e, 2m in [1, 2) */
    double frac = 2.0 * m - 1.0;    /* in [0, 1) */
    return (uint16_t)(((e + 15) << 10) | (int)(frac * 1024.0));
}

/* Quantum (spacing of binary16 values) in the binade containing |x|. */
static double f16_quantum(double ax)
{
    if (ax < ldexp(1.0, -14)) return ldexp(1.0, -24);
    int ex;
    frexp(ax, &ex);
    return ldexp(1.0, (ex - 1) - 10);
}

/* float -> binary16 rounded toward +infinity (R2): the smallest binary16
 * value >= x.  Exact: every step is a power-of-two scaling or ceil/floor of a
 * double that holds the float exactly. */
uint16_t kvko_f32_to_f16_ru(float xf)
{
    double x = (double)xf;
    const double max16 = 65504.0;
    if (isnan(x)) return 0x7E00;
    if (x == 0.0) return signbit(x) ? 0x8000 : 0;
    if (x > 0) {
        if (x > max16) return 0x7C00;                  /* +inf */
        double qn = f16_quantum(x);
        double up = ceil(x / qn) * qn;                 /* may reach next binade: still exact */
        return encode_f16_exact(up);
    } else {
        double ax = -x;
        if (isinf(ax)) return 0xFC00;                  /* -inf stays -inf */
        if (ax > max16) return 0x8000 | encode_f16_exact(max16);
        double qn = f16_quantum(ax);
        double dn = floor(ax / qn) * qn;               /* toward +inf = magnitude down */
        return 0x8000 | encode_f16_exact(dn);
    }
}

/* ------------------------------------------------------------------------ */
/* bfloat16, for the uncompressed cache the compressed one is measured        */
/* against: 1 sign bit, 8 exponent bits, 7 fraction bits, i.e. exactly the     */
/* binary32 values whose low 16 bits are zero.                                */
/* ------------------------------------------------------------------------ */

double kvko_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* binary32 -> bfloat16, round to nearest, ties to even: of the two bf16 values
 * that bracket x (truncation of the low 16 bits, and the next one away from
 * zero), take the nearer in exact arithmetic; on a tie the one whose last
 * fraction bit is 0.  The next value past the largest finite one is +-inf,
 * reached (as in IEEE arithmetic) from half an ulp beyond the largest. */
uint16_t kvko_f32_to_bf16_rne(float x)
{
    if (isnan(x)) return 0x7FC0;
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    if ((u & 0x7FFFFFFFu) >= 0x7F800000u) return (uint16_t)(u >> 16);   /* +-inf */
    uint32_t lo_bits = u & 0xFFFF0000u, hi_bits = lo_bits + 0x10000u;
    float lo, hi;
    memcpy(&lo, &lo_bits, sizeof lo);
    double dlo = (double)lo, dhi;
    if ((hi_bits & 0x7FFFFFFFu) == 0x7F800000u) {
        dhi = ldexp(1.0, 128);                   /* where +-inf sits in the rounding rule */
        if (signbit(x)) dhi = -dhi;
    } else {
        memcpy(&hi, &hi_bits, sizeof hi);
        dhi = (double)hi;
    }
    double dx = (double)x;
    double elo = fabs(dx - dlo), ehi = fabs(dhi - dx);
    if (elo < ehi) return (uint16_t)(lo_bits >> 16);
    if (ehi < elo) return (uint16_t)(hi_bits >> 16);
    return ((lo_bits >> 16) & 1u) ? (uint16_t)(hi_bits >> 16) : (uint16_t)(lo_bits >> 16);
}

void kvko_bf16_round(const float* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = kvko_f32_to_bf16_rne(v[i]);
}

/* ------------------------------------------------------------------------ */
/* Quantiser (R1-R3): one token vector v[0..n) -> fp16 scale + integer codes  */
/* ------------------------------------------------------------------------ */

void kvko_quantize_token(const float* v, int n, int b, uint16_t* scale_out, int32_t* codes)
{
    const int q = (1 << (b - 1)) - 1;
    float A = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > A) A = a;
    }
    volatile float qf = (float)q;
    volatile float s32 = A / qf;                 /* IEEE binary32 division */
    uint16_t sh = kvko_f32_to_f16_ru(s32);
    float s = (float)kvko_f16_to_f64(sh);
    *scale_out = sh;
    for (int i = 0; i < n; ++i) {
        if (s == 0.0f) { codes[i] = 0; continue; }
        volatile float t = v[i] / s;             /* IEEE binary32 division */
        float r = nearbyintf(t);                 /* round half to even (default mode) */
        long c = (long)r;
        if (c > q) c = q;
        if (c < -q) c = -q;
        codes[i] = (int32_t)c;
    }
}

void kvko_quantize(const float* v, int64_t n_tok, int n, int b, uint16_t* scales, int32_t* codes)
{
    fesetround(FE_TONEAREST);
    for (int64_t t = 0; t < n_tok; ++t)
        kvko_quantize_token(v + t * n, n, b, scales + t, codes + t * n);
}

/* ------------------------------------------------------------------------ */
/* Packing (R4)                                                              */
/* ------------------------------------------------------------------------ */

int kvko_row_bytes(int n, int b)
{
    int raw = (n * b + 7) / 8;
    return (raw + 15) / 16 * 16;
}

void kvko_pack(const int32_t* codes, int64_t n_tok, int n, int b, int row_bytes, uint8_t* rows)
{
    const int off = 1 << (b - 1);
    memset(rows, 0, (size_t)(n_tok * row_bytes));
    for (int64_t t = 0; t < n_tok; ++t) {
        uint8_t* row = rows + t * row_bytes;
        for (int i = 0; i < n; ++i) {
            uint32_t u = (uint32_t)(codes[t * n + i] + off);
            for (int k = 0; k < b; ++k) {
                int64_t bit = (int64_t)i * b + k;
                if ((u >> k) & 1u) row[bit / 8] |= (uint8_t)(1u << (bit % 8));
            }
        }
    }
}

void kvko_unpack(const uint8_t* rows, int64_t n_tok, int n, int b, int row_bytes, int32_t* codes)
{
    const int off = 1 << (b - 1);
    for (int64_t t = 0; t < n_tok; ++t) {
        const uint8_t* row = rows + t * row_bytes;
        for (int i = 0; i < n; ++i) {
            uint32_t u = 0;
            for (int k = 0; k < b; ++k) {
                int64_t bit = (int64_t)i * b + k;
                u |= (uint32_t)((row[bit / 8] >> (bit % 8)) & 1u) << k;
            }
            codes[t * n + i] = (int32_t)u - off;
        }
    }
}

/* Dequantise: c_hat = code * s, exact in binary64. */
void kvko_dequant(const int32_t* codes, const uint16_t* scales, int64_t n_tok, int n, double* out)
{
    for (int64_t t = 0; t < n_tok; ++t) {
        double s = kvko_f16_to_f64(scales[t]);
        for (int i = 0; i < n; ++i) out[t * n + i] = (double)codes[t * n + i] * s;
    }
}

/* ------------------------------------------------------------------------ */
/* Decode attention for one sequence (R5), binary64 throughout.              */
/*   q_lat  [H][d]       query projected into latent space                    */
/*   q_rope [H][d_R]     RoPE part of the query                               */
/*   rows   [T][d+d_R]   dequantised cache rows of the anchor layer           */
/*   tok    [nt]         token indices attended (all tokens, or a keep list)  */
/*   out    [H][d], lse [H]                                                   */
/* ------------------------------------------------------------------------ */

void kvko_attend(const double* q_lat, const double* q_rope, const double* rows,
                 const int32_t* tok, int nt, int H, int d, int d_R, double sigma,
                 double* out, double* lse)
{
    const int n = d + d_R;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int h = 0; h < H; ++h) {
        double* o = out + (size_t)h * d;
        for (int j = 0; j < d; ++j) o[j] = 0.0;
        if (nt == 0) { lse[h] = -INFINITY; continue; }
        /* scores */
        double m = -INFINITY;
        for (int i = 0; i < nt; ++i) {
            const double* c = rows + (size_t)tok[i] * n;
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += q_lat[(size_t)h * d + j] * c[j];
            for (int j = 0; j < d_R; ++j) acc += q_rope[(size_t)h * d_R + j] * c[d + j];
            double z = sigma * acc;
            if (z > m) m = z;
        }
        /* softmax weights relative to the max, then the weighted sum */
        double l = 0.0;
        for (int i = 0; i < nt; ++i) {
            const double* c = rows + (size_t)tok[i] * n;
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += q_lat[(size_t)h * d + j] * c[j];
            for (int j = 0; j < d_R; ++j) acc += q_rope[(size_t)h * d_R + j] * c[d + j];
            double w = exp(sigma * acc - m);
            l += w;
            for (int j = 0; j < d; ++j) o[j] += w * c[j];
        }
        for (int j = 0; j < d; ++j) o[j] /= l;
        lse[h] = m + log(l);
    }
}

/* ------------------------------------------------------------------------ */
/* Cost model ("Action Space and Cost Model", plus R6)                        */
/* ------------------------------------------------------------------------ */

/* Bits per token of a plan: anchors pay (d+d_R)*b (+16 for the fp16 scale
 * when with_scale != 0); inheriting layers pay 0.  b = 0 marks an anchor kept
 * uncompressed in bfloat16 (the cache C_0's 16 bits per element, no scale): it
 * pays (d+d_R)*16. */
int64_t kvko_bits_per_token(int n_layers, const int32_t* anchor, const int32_t* d,
                            const int32_t* b, int d_R, int with_scale)
{
    int64_t s = 0;
    for (int l = 0; l < n_layers; ++l) {
        if (anchor[l] != l) continue;
        if (b[l] == 0)
            s += (int64_t)(d[l] + d_R) * 16;
        else
            s += (int64_t)(d[l] + d_R) * b[l] + (with_scale ? 16 : 0);
    }
    return s;
}

/* Bits per token of a plan whose anchors carry one fp16 scale per group of G
 * consecutive elements of [c[:d] || k^R] instead of one per token (the group-scale
 * comparison point: a b-bit cache with a scale per G elements costs b + 16/G bits
 * per element, e.g. 4.5 at b = 4, G = 32): anchors pay (d+d_R)*b + 16*(d+d_R)/G;
 * an uncompressed (b = 0) anchor pays (d+d_R)*16. */
int64_t kvko_bits_per_token_grouped(int n_layers, const int32_t* anchor, const int32_t* d,
                                    const int32_t* b, int d_R, int G)
{
    int64_t s = 0;
    for (int l = 0; l < n_layers; ++l) {
        if (anchor[l] != l) continue;
        const int n = d[l] + d_R;
        if (b[l] == 0)
            s += (int64_t)n * 16;
        else
            s += (int64_t)n * b[l] + (int64_t)16 * (n / G);
    }
    return s;
}

/* Uncompressed bf16 non-MLA cost: C_0 = L * 2 * n_kv * d_h * 16. */
int64_t kvko_c0_bits(int n_layers, int n_kv, int d_h)
{
    return (int64_t)n_layers * 2 * n_kv * d_h * 16;
}

int kvko_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
