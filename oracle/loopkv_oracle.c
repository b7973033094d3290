/*
 * loopkv_oracle.c -- plain, slow, single-threaded CPU oracle for the LoopKV
 * decode hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline / reference arm may load this library.  It shares no code, header,
 * constant or table with the CUDA library; every rule below is restated here from
 * the LoopKV paper (arXiv 2611.04137) and the readings listed in the design notes.
 *
 * What it computes, and where each step comes from:
 *   - KIVI-style asymmetric quantization with an fp16 scale and an fp16 zero per
 *     group of 32: keys grouped per channel over 32 tokens, values per token over
 *     32 channels (LoopKV paper, §5.1 "Baselines and ablations": groups of 32;
 *     Appendix "History reader": per-channel key scale constant over a page,
 *     per-token value scale).  The exact rounding rule is not printed anywhere;
 *     the reading used here: zero = largest fp16 <= min, scale = smallest fp16 >=
 *     (max - zero) / L computed in fp64, code = round-half-even of the fp32
 *     quotient fl32(fl32(x - zero) / scale), clamped to [0, L].
 *   - Bit-plane value layout: a 4-bit value code q = 4h + l is kept as a hi plane
 *     h = q >> 2 and a lo plane l = q & 3; keys stay one 4-bit plane (LoopKV paper,
 *     §3.3 "Bit-plane V layout").
 *   - Read-time V precision: a history token is hot when its softmax weight is at
 *     least tau times the largest weight in its row (LoopKV paper, §3.3, "Read-time
 *     V precision at no extra read cost"; the "ideal" test with the exact row
 *     maximum).  A hot token reads both planes (full INT4 value); a cold token
 *     reads only the hi plane and decodes to the middle of its 4-code bucket,
 *     z + s * (4h + 1.5).  Scores always come from the full 4-bit keys (LoopKV
 *     paper, Appendix "Proof of Proposition 1").
 *   - An INT2 cell stores its own 2-bit codes, read in full (LoopKV paper, §3.4
 *     "Layout"; §2.4 P1 "KIVI-style INT2").
 *   - Exact softmax attention in fp64 over history (dequantized) and the BF16/fp32
 *     tail (raw), o = sum_t r_t v_t / sum_t r_t with r_t = exp(s_t - m).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -shared -fPIC (no -ffast-math): the
 * fp32 steps of the quantizer must be plain IEEE binary32 operations.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* status codes of this oracle (its own numbering) */
#define ORC_OK 0
#define ORC_NONFINITE 1
#define ORC_RANGE 2
#define ORC_BADARG 3

#define ORC_GROUP 32        /* quantization group (LoopKV paper, §5.1: groups of 32) */
#define ORC_F16_MAX 65504.0 /* largest finite IEEE binary16 value */

/* ------------------------------------------------------------------------- */
/* IEEE 754 binary16, written out from the format definition.                */
/* ------------------------------------------------------------------------- */

/* Value of a binary16 bit pattern. */
double orc_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24); /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* Bit pattern of a finite value that is exactly representable in binary16. */
static uint16_t f16_encode_exact(double v)
{
    uint16_t sign = 0;
    if (signbit(v)) {
        sign = 0x8000;
        v = -v;
    }
    if (v == 0.0)
        return sign;
    if (v < ldexp(1.0, -14)) /* subnormal range */
        return (uint16_t)(sign | (uint16_t)(v * ldexp(1.0, 24)));
    int e2;
    double f = frexp(v, &e2); /* v = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;           /* v = (2f) * 2^E, 2f in [1, 2) */
    uint16_t mant = (uint16_t)((2.0 * f - 1.0) * 1024.0);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | mant);
}

/* Spacing of binary16 values in the binade of |x| (x finite, nonzero). */
static double f16_ulp(double x)
{
    double a = fabs(x);
    if (a < ldexp(1.0, -14))
        return ldexp(1.0, -24);
    int e2;
    frexp(a, &e2);
    return ldexp(1.0, (e2 - 1) - 10);
}

/*
 * Round a double to binary16.  dir = -1: toward -inf (largest fp16 <= x);
 * dir = +1: toward +inf (smallest fp16 >= x); dir = 0: nearest, ties to even.
 * Overflow follows IEEE 754: a result beyond the largest finite value becomes
 * infinity unless the rounding direction points back toward zero.
 */
uint16_t orc_f64_to_f16(double x, int dir)
{
    if (isnan(x))
        return 0x7e00;
    if (isinf(x)) {
        if (x > 0)
            return dir < 0 ? f16_encode_exact(ORC_F16_MAX) : 0x7c00;
        return dir > 0 ? f16_encode_exact(-ORC_F16_MAX) : 0xfc00;
    }
    if (x == 0.0)
        return signbit(x) ? 0x8000 : 0x0000;
    double u = f16_ulp(x);
    double t = x / u; /* exact: division by a power of two */
    double k;
    if (dir < 0)
        k = floor(t);
    else if (dir > 0)
        k = ceil(t);
    else
        k = nearbyint(t); /* default rounding mode: ties to even */
    double y = k * u;
    if (y > ORC_F16_MAX)
        return dir < 0 ? f16_encode_exact(ORC_F16_MAX) : 0x7c00;
    if (y < -ORC_F16_MAX)
        return dir > 0 ? f16_encode_exact(-ORC_F16_MAX) : 0xfc00;
    if (y == 0.0)
        return signbit(x) ? 0x8000 : 0x0000;
    return f16_encode_exact(y);
}

/* ------------------------------------------------------------------------- */
/* Quantization of one group (KIVI-style asymmetric, LoopKV paper §5.1).     */
/* ------------------------------------------------------------------------- */

/*
 * Quantize n values x[0], x[stride], ... at L = 2^bits - 1 levels.
 *   1. mn, mx = min and max (fp32); any non-finite value -> NONFINITE.
 *   2. zero  = largest fp16 <= mn.
 *   3. r     = ((double)mx - (double)zero) / L, in fp64.
 *   4. scale = smallest fp16 >= r.  zero or scale infinite -> RANGE.
 *   5. scale == 0 -> every code is 0.
 *   6. code_i = clamp(round_half_even(fl32(fl32(x_i - zero) / scale)), 0, L).
 * On an error the group is written as zero = scale = 0 and all codes 0.
 */
int orc_quantize_group(const float *x, int stride, int n, int bits, uint16_t *zero_out,
                       uint16_t *scale_out, uint8_t *codes, int code_stride)
{
    int L = (1 << bits) - 1;
    float mn = x[0], mx = x[0];
    int bad = 0;
    for (int i = 0; i < n; ++i) {
        float v = x[(size_t)i * stride];
        if (!isfinite(v))
            bad = 1;
        if (v < mn)
            mn = v;
        if (v > mx)
            mx = v;
    }
    int status = ORC_OK;
    uint16_t zh = 0, sh = 0;
    if (bad) {
        status = ORC_NONFINITE;
    } else {
        zh = orc_f64_to_f16((double)mn, -1);
        double z = orc_f16_to_f64(zh);
        if (isinf(z)) {
            status = ORC_RANGE;
        } else {
            double r = ((double)mx - z) / (double)L;
            sh = orc_f64_to_f16(r, +1);
            if (isinf(orc_f16_to_f64(sh)))
                status = ORC_RANGE;
        }
    }
    if (status != ORC_OK) {
        *zero_out = 0;
        *scale_out = 0;
        for (int i = 0; i < n; ++i)
            codes[(size_t)i * code_stride] = 0;
        return status;
    }
    float zf = (float)orc_f16_to_f64(zh);
    float sf = (float)orc_f16_to_f64(sh);
    for (int i = 0; i < n; ++i) {
        int c = 0;
        if (sf != 0.0f) {
            float d = x[(size_t)i * stride] - zf; /* fp32 subtract, round to nearest */
            float qf = d / sf;                    /* fp32 divide, round to nearest */
            double rq = nearbyint((double)qf);    /* ties to even (exact on a float) */
            c = (int)(rq < 0 ? 0 : (rq > L ? L : rq));
        }
        codes[(size_t)i * code_stride] = (uint8_t)c;
    }
    *zero_out = zh;
    *scale_out = sh;
    return ORC_OK;
}

/*
 * Keys of one (request, head): k[T][D] row-major, T a multiple of 32.  Group g
 * covers tokens 32g..32g+31 of one channel.  codes[T][D]; scale/zero[T/32][D].
 * Returns the first non-OK status met (every group is still written).
 */
int orc_quantize_k(const float *k, int T, int D, int bits, uint8_t *codes, uint16_t *scale,
                   uint16_t *zero)
{
    if (T % ORC_GROUP)
        return ORC_BADARG;
    int status = ORC_OK;
    for (int g = 0; g < T / ORC_GROUP; ++g)
        for (int c = 0; c < D; ++c) {
            int st = orc_quantize_group(k + (size_t)g * ORC_GROUP * D + c, D, ORC_GROUP, bits,
                                        &zero[(size_t)g * D + c], &scale[(size_t)g * D + c],
                                        codes + (size_t)g * ORC_GROUP * D + c, D);
            if (st && !status)
                status = st;
        }
    return status;
}

/*
 * Values of one (request, head): v[T][D].  Group j of token t covers channels
 * 32j..32j+31.  codes[T][D]; scale/zero[T][D/32].
 */
int orc_quantize_v(const float *v, int T, int D, int bits, uint8_t *codes, uint16_t *scale,
                   uint16_t *zero)
{
    if (D % ORC_GROUP)
        return ORC_BADARG;
    int G = D / ORC_GROUP, status = ORC_OK;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < G; ++j) {
            int st = orc_quantize_group(v + (size_t)t * D + j * ORC_GROUP, 1, ORC_GROUP, bits,
                                        &zero[(size_t)t * G + j], &scale[(size_t)t * G + j],
                                        codes + (size_t)t * D + j * ORC_GROUP, 1);
            if (st && !status)
                status = st;
        }
    return status;
}

/* ------------------------------------------------------------------------- */
/* Packed storage of one 16-token block of one head.                          */
/* ------------------------------------------------------------------------- */
/*
 * The paper fixes only that keys are "interleaved 4-bit codes", that an INT4
 * value is kept as two 2-bit planes hi and lo followed by scales and zeros, and
 * that an INT2 page holds its own 2-bit codes (LoopKV paper, §3.3 and §3.4
 * "Layout").  The byte order below is this implementation's reading, stated in
 * words so that the CUDA side can be checked against it byte for byte:
 *
 *   4-bit row (D channels, D/2 bytes): 32-bit word w holds channels 8w..8w+7;
 *     in byte b of that word the low nibble is channel 8w+b and the high nibble
 *     channel 8w+4+b.
 *   2-bit row (D/4 bytes): word w holds channels 16w..16w+15; in byte b, bits
 *     2i..2i+1 are channel 16w+4i+b.
 *   Block = 16 tokens of one (cell, request); a K group of 32 tokens is two
 *   consecutive blocks.  Per head, the main region of a 4-bit block is
 *     [K codes 16 x D/2][K meta D x fp16][V meta 16 x (D/32) x (scale,zero)]
 *     [V hi plane 16 x D/4]
 *   where K meta is the group's K scales in the even block and its K zeros in
 *   the odd block; the V lo plane (16 x D/4) is a separate array.  A 2-bit
 *   block per head is [K codes 16 x D/4][K meta D x fp16][V meta][V codes
 *   16 x D/4].  fp16 values are little-endian.
 */

static void put_u16(uint8_t *p, uint16_t v)
{
    p[0] = (uint8_t)(v & 0xff);
    p[1] = (uint8_t)(v >> 8);
}

/* one 4-bit row of D codes */
void orc_pack_row4(const uint8_t *codes, int D, uint8_t *out)
{
    memset(out, 0, (size_t)D / 2);
    for (int c = 0; c < D; ++c) {
        int w = c / 8, r = c % 8, b = r % 4;
        int byte = 4 * w + b;
        if (r < 4)
            out[byte] |= (uint8_t)(codes[c] & 0xf);
        else
            out[byte] |= (uint8_t)((codes[c] & 0xf) << 4);
    }
}

/* one 2-bit row of D codes */
void orc_pack_row2(const uint8_t *codes, int D, uint8_t *out)
{
    memset(out, 0, (size_t)D / 4);
    for (int c = 0; c < D; ++c) {
        int w = c / 16, r = c % 16, b = r % 4, i = r / 4;
        out[4 * w + b] |= (uint8_t)((codes[c] & 3) << (2 * i));
    }
}

/* bytes of one head's main region / lo region of a block */
int orc_head_main_bytes(int bits, int D)
{
    int kc = bits == 4 ? 16 * D / 2 : 16 * D / 4;
    return kc + 2 * D + 16 * (D / ORC_GROUP) * 4 + 16 * D / 4;
}
int orc_head_lo_bytes(int bits, int D) { return bits == 4 ? 16 * D / 4 : 0; }

static void put_u32(uint8_t *p, uint32_t v)
{
    p[0] = (uint8_t)(v & 0xff);
    p[1] = (uint8_t)((v >> 8) & 0xff);
    p[2] = (uint8_t)((v >> 16) & 0xff);
    p[3] = (uint8_t)(v >> 24);
}

/*
 * One word of a value plane: 4 tokens x 4 channels of 2-bit values plane[16][D].
 * Byte b holds token 4*tau + b; in it, bits 2i..2i+1 hold channel 4*kappa + i.
 * (The pages fix two 2-bit planes, not their bit order; this is the reading.)
 */
static uint32_t plane_word(const uint8_t *plane, int D, int kappa, int tau)
{
    uint32_t w = 0;
    for (int b = 0; b < 4; ++b)
        for (int i = 0; i < 4; ++i)
            w |= (uint32_t)(plane[(size_t)(4 * tau + b) * D + 4 * kappa + i] & 3) << (8 * b + 2 * i);
    return w;
}

/*
 * Pack one head of one block.  kcodes[16][D], kmeta[D] (scales if the block is
 * even in its group, zeros if odd), vcodes[16][D] (4-bit or 2-bit codes),
 * vscale/vzero[16][D/32].  main_out gets orc_head_main_bytes, lo_out (4-bit
 * only) orc_head_lo_bytes.
 *   K rows: token-major, orc_pack_row4 / orc_pack_row2 per token.
 *   V meta: (scale, zero) fp16 pairs ordered [channel group j][token t].
 *   V planes: words of plane_word; the hi plane (or the 2-bit codes) ordered
 *   [channel quad kappa][token quad tau], the lo plane [tau][kappa].
 */
void orc_pack_head_block(int bits, int D, const uint8_t *kcodes, const uint16_t *kmeta,
                         const uint8_t *vcodes, const uint16_t *vscale, const uint16_t *vzero,
                         uint8_t *main_out, uint8_t *lo_out)
{
    int G = D / ORC_GROUP;
    uint8_t *p = main_out;
    for (int t = 0; t < 16; ++t) {
        if (bits == 4) {
            orc_pack_row4(kcodes + (size_t)t * D, D, p);
            p += D / 2;
        } else {
            orc_pack_row2(kcodes + (size_t)t * D, D, p);
            p += D / 4;
        }
    }
    for (int c = 0; c < D; ++c, p += 2)
        put_u16(p, kmeta[c]);
    for (int j = 0; j < G; ++j)
        for (int t = 0; t < 16; ++t) {
            put_u16(p, vscale[t * G + j]);
            put_u16(p + 2, vzero[t * G + j]);
            p += 4;
        }
    uint8_t *hi = (uint8_t *)malloc((size_t)16 * D), *lo = (uint8_t *)malloc((size_t)16 * D);
    for (int i = 0; i < 16 * D; ++i) {
        hi[i] = bits == 4 ? (uint8_t)(vcodes[i] >> 2) : vcodes[i];
        lo[i] = (uint8_t)(vcodes[i] & 3);
    }
    for (int kappa = 0; kappa < D / 4; ++kappa)
        for (int tau = 0; tau < 4; ++tau)
            put_u32(p + 4 * (kappa * 4 + tau), plane_word(hi, D, kappa, tau));
    if (bits == 4)
        for (int tau = 0; tau < 4; ++tau)
            for (int kappa = 0; kappa < D / 4; ++kappa)
                put_u32(lo_out + 4 * (tau * (D / 4) + kappa), plane_word(lo, D, kappa, tau));
    free(hi);
    free(lo);
}

/* ------------------------------------------------------------------------- */
/* Decode attention for one (request, head) row, fp64, exact row maximum.   */
/* ------------------------------------------------------------------------- */

#define ORC_TAU_REL_MAX 0 /* hot iff r_t = exp(s_t - m) >= tau        (LoopKV paper, §3.3) */
#define ORC_TAU_ABS_PROB 1 /* hot iff r_t / sum_u r_u >= tau           (normalised weight) */

/*
 * Inputs (one row; history length n_hist is a multiple of 32):
 *   q[D]                 query, already widened to double
 *   kc[n_hist][D]        key codes, ks/kz[n_hist/32][D] fp16 scale/zero
 *   vc[n_hist][D]        value codes (4-bit code q, or 2-bit code), vs/vz[n_hist][D/32]
 *   bits                 4 or 2 (storage of the cell whose history is read)
 *   tk/tv[n_tail][D]     raw tail keys/values (BF16 or fp32 inputs widened)
 *   tau, tau_mode        threshold of the refine set
 *   s_force              if not NULL: use this refine-set bitmap instead of
 *                        computing it (re-evaluation with another reader's set)
 * Outputs:
 *   o[D]                 attention output (fp64)
 *   m_out, l_out         row max of the scores, sum_t exp(s_t - m)
 *   s_bits[n_hist/32]    refine set S: bit (t % 32) of word t/32 set iff t is hot
 *   r_out[n_hist+n_tail] exp(s_t - m) (history first), may be NULL
 * Returns ORC_BADARG if no token is attended.
 */
int orc_decode_row_from(int D, int bits, int n_hist, int hist_first, const double *q, const uint8_t *kc,
                        const uint16_t *ks, const uint16_t *kz, const uint8_t *vc, const uint16_t *vs,
                        const uint16_t *vz, int n_tail, const double *tk, const double *tv, double tau,
                        int tau_mode, const uint32_t *s_force, double *o, double *m_out, double *l_out,
                        uint32_t *s_bits, double *r_out);

int orc_decode_row(int D, int bits, int n_hist, const double *q, const uint8_t *kc,
                   const uint16_t *ks, const uint16_t *kz, const uint8_t *vc,
                   const uint16_t *vs, const uint16_t *vz, int n_tail, const double *tk,
                   const double *tv, double tau, int tau_mode, const uint32_t *s_force,
                   double *o, double *m_out, double *l_out, uint32_t *s_bits, double *r_out)
{
    return orc_decode_row_from(D, bits, n_hist, 0, q, kc, ks, kz, vc, vs, vz, n_tail, tk, tv, tau, tau_mode,
                               s_force, o, m_out, l_out, s_bits, r_out);
}

/*
 * orc_decode_row for a layer with a sliding attention window (the Dory model's
 * sliding-window layers, LoopKV paper §2.1): history tokens t < hist_first lie before the
 * window and are not attended (weight 0, never in S, r_out 0); the caller passes only the
 * attended tail tokens.  hist_first = 0 is plain orc_decode_row.  The history is still
 * quantized in its 32-token groups from token 0, as it is stored.
 */
int orc_decode_row_from(int D, int bits, int n_hist, int hist_first, const double *q, const uint8_t *kc,
                        const uint16_t *ks, const uint16_t *kz, const uint8_t *vc, const uint16_t *vs,
                        const uint16_t *vz, int n_tail, const double *tk, const double *tv, double tau,
                        int tau_mode, const uint32_t *s_force, double *o, double *m_out, double *l_out,
                        uint32_t *s_bits, double *r_out)
{
    int n = n_hist + n_tail, G = D / ORC_GROUP;
    if (hist_first < 0 || hist_first > n_hist)
        return ORC_BADARG;
    if (n - hist_first <= 0 || n_hist % ORC_GROUP || (bits != 4 && bits != 2))
        return ORC_BADARG;
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    double *r = (double *)malloc(sizeof(double) * (size_t)n);
    double inv_sqrt_d = 1.0 / sqrt((double)D);

    /* 1. scores from dequantized keys k = z + s * code (history) or raw keys (tail) */
    for (int t = 0; t < n; ++t) {
        double acc = 0.0;
        for (int c = 0; c < D; ++c) {
            double kv;
            if (t < n_hist) {
                int g = t / ORC_GROUP;
                kv = orc_f16_to_f64(kz[(size_t)g * D + c]) +
                     orc_f16_to_f64(ks[(size_t)g * D + c]) * (double)kc[(size_t)t * D + c];
            } else {
                kv = tk[(size_t)(t - n_hist) * D + c];
            }
            acc += q[c] * kv;
        }
        s[t] = acc * inv_sqrt_d;
    }
    /* 2. exact row maximum over the attended tokens and weights r_t = exp(s_t - m) */
    double m = s[hist_first];
    for (int t = hist_first + 1; t < n; ++t)
        if (s[t] > m)
            m = s[t];
    double l = 0.0;
    for (int t = 0; t < n; ++t) {
        r[t] = t < hist_first ? 0.0 : exp(s[t] - m);
        l += r[t];
    }
    /* 3. refine set S (history tokens of a 4-bit cell only) */
    int W = n_hist / ORC_GROUP;
    for (int w = 0; w < W; ++w)
        s_bits[w] = 0;
    for (int t = hist_first; t < n_hist; ++t) {
        int hot;
        if (s_force)
            hot = (s_force[t / 32] >> (t % 32)) & 1;
        else if (bits != 4)
            hot = 0;
        else if (tau_mode == ORC_TAU_ABS_PROB)
            hot = r[t] / l >= tau;
        else
            hot = r[t] >= tau;
        if (hot && bits == 4)
            s_bits[t / 32] |= 1u << (t % 32);
    }
    /* 4. output: hot -> z + s*q, cold -> z + s*(4h + 1.5), 2-bit -> z + s*code, tail raw */
    for (int c = 0; c < D; ++c) {
        double acc = 0.0;
        for (int t = hist_first; t < n; ++t) {
            double vv;
            if (t < n_hist) {
                int j = c / ORC_GROUP;
                double z = orc_f16_to_f64(vz[(size_t)t * G + j]);
                double sc = orc_f16_to_f64(vs[(size_t)t * G + j]);
                int code = vc[(size_t)t * D + c];
                if (bits == 2) {
                    vv = z + sc * (double)code;
                } else if ((s_bits[t / 32] >> (t % 32)) & 1) {
                    vv = z + sc * (double)code;
                } else {
                    vv = z + sc * (4.0 * (double)(code >> 2) + 1.5);
                }
            } else {
                vv = tv[(size_t)(t - n_hist) * D + c];
            }
            acc += r[t] * vv;
        }
        o[c] = acc / l;
    }
    *m_out = m;
    *l_out = l;
    if (r_out)
        for (int t = 0; t < n; ++t)
            r_out[t] = r[t];
    free(s);
    free(r);
    return ORC_OK;
}

/*
 * Refine set of the streaming reader (LoopKV §3.3 "Read-time V precision", §3.4 launch
 * grid): instead of the row's exact maximum, the reader tests each token against a
 * maximum that starts at a seed m0 (the published sink maximum; when it does not arrive
 * in time the seed is chosen so that every token is hot).  The pages leave open whether
 * that maximum also grows with the scores the reader has already computed; both
 * readings are provided:
 *   running = 1: the history is read in 32-token groups in the order order[0..ng-1]; a
 *                group's scores are known before its values are read, so the running
 *                maximum takes the group's largest score before its tokens are tested;
 *   running = 0: every token is tested against the seed alone (m0 = -infinity then
 *                marks every token hot, the fallback of §3.4).
 * Token t is hot iff exp(s_t - m) >= tau for the maximum m it is tested against.  As
 * long as m0 does not exceed the exact row maximum, neither maximum does, and the set
 * contains the exact one (a superset).
 *   s[n_hist]            scores in natural-log units (q.k / sqrt(D))
 *   order[ng]            each group index 0..n_hist/32-1 exactly once
 *   s_bits[n_hist/32]    output, bit (t % 32) of word t/32 set iff t is hot
 * Returns ORC_BADARG on a malformed order.
 */
int orc_stream_refine(int n_hist, const double *s, const int *order, int ng, double m0, int running,
                      double tau, uint32_t *s_bits)
{
    if (n_hist < 0 || n_hist % ORC_GROUP || ng != n_hist / ORC_GROUP)
        return ORC_BADARG;
    unsigned char *seen = (unsigned char *)calloc((size_t)(ng > 0 ? ng : 1), 1);
    for (int i = 0; i < ng; ++i) {
        if (order[i] < 0 || order[i] >= ng || seen[order[i]]) {
            free(seen);
            return ORC_BADARG;
        }
        seen[order[i]] = 1;
    }
    free(seen);
    double m_run = m0;
    for (int i = 0; i < ng; ++i) {
        const int g = order[i];
        if (running)
            for (int j = 0; j < ORC_GROUP; ++j)
                if (s[g * ORC_GROUP + j] > m_run)
                    m_run = s[g * ORC_GROUP + j];
        uint32_t w = 0;
        for (int j = 0; j < ORC_GROUP; ++j)
            if (exp(s[g * ORC_GROUP + j] - m_run) >= tau)
                w |= 1u << j;
        s_bits[g] = w;
    }
    return ORC_OK;
}
