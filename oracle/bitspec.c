/*
 * fp32 operation sequence of the post-RoPE Q/K transform with dynamic KV4
 * quantisation, in plain C.
 *
 * TEST INFRASTRUCTURE ONLY.  It is loaded by oracle/bitspec.py, which only
 * tests/, __graft_entry__.smoke() and the CPU-baseline / reference legs of
 * bench.py import.  It shares no code with the CUDA library.
 *
 * Why an fp32 sequence beside the fp64 definition (oracle/definition.py): the
 * 4-bit codes are integers decided by floating point, and the decision has to
 * be taken in the same precision on both sides.  The kernel computes in fp32,
 * so this file fixes one fp32 order of operations, step by step in the order
 * the method applies them:
 *
 *   load      bf16 -> fp32 (exact)
 *   RoPE      pair (a, b), table entries c = fp32(cos(m w_k)), s = fp32(sin(m w_k)):
 *             a' = fma(a, c, -(b*s)),  b' = fma(a, s, b*c)
 *             (split tables: (c, s) = the high row (64 h) turned by the low row (l),
 *              m = 64 h + l, c = fma(c_h, c_l, -(s_h*s_l)), s = fma(c_h, s_l, s_h*c_l))
 *             (paper summary "When Local Variance Optimality Is Not Enough ...",
 *              "Problem statement": RoPE turns fixed two-dimensional frequency pairs)
 *   pairwise  after RoPE, the pair rotation by phi_k ("Methodology", item 2: the
 *             head-shared rotation of each post-RoPE frequency pair), its own step with
 *             the same two lines and cphi = fp32(cos(phi_k)), sphi = fp32(sin(phi_k))
 *             computed in fp64 from the fp32 angle:
 *             a'' = fma(a', cphi, -(b'*sphi)),  b'' = fma(a', sphi, b'*cphi)
 *   Hadamard  fast Walsh-Hadamard butterfly (u, v) -> (u + v, u - v) over blocks of
 *             n channels, strides 1, 2, 4, ..., n/2 in that order, then one
 *             multiply by kappa_n = fp32(1/sqrt(n)) ("LLM旋转量化笔记" §3.3, online
 *             FWHT; §2.2, normalisation 1/sqrt(K))
 *   Q store   fp32 -> bf16, round to nearest even
 *   K quant   per group: amax = max|x|; r = 7/amax (IEEE division);
 *             code = clamp(rint(x*r), -7, 7) where x*r is the EXACT product
 *             (rounded once, to the nearest integer, ties to even); s = amax/7
 *             (IEEE division); stored scale = fp16(s), round to nearest even
 *             ("LLM旋转量化笔记" §1.2 quantiser round(x/s), step from the group range)
 *   pack      byte j = (code[2j] & 0xF) | ((code[2j+1] & 0xF) << 4)
 *
 * Groups whose amax is below 2^-125 (zero included) get codes 0 and scale 0:
 * their fp16 scale would be 0 anyway, and 7/amax would overflow fp32.
 *
 * Status bits (OR-ed into *status): 1 = a transformed K value was NaN or Inf,
 * 2 = a stored fp16 scale overflowed to Inf, 4 = a position was outside
 * [0, max_pos) (the row is then computed at the clamped position).
 *
 * Build with -ffp-contract=off and without -ffast-math: every a*b + c below is
 * two roundings unless written as fmaf.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { MODE_HADAMARD = 0, MODE_PAIRWISE = 1, MODE_PAIRWISE_HADAMARD = 2,
       MODE_BLOCK_HADAMARD = 3, MODE_ROPE_ONLY = 4 };
enum { ROPE_HALF = 0, ROPE_INTERLEAVED = 1, STYLE_SPLIT_TABLE = 0x100 };
enum { ST_NONFINITE = 1, ST_SCALE_OVERFLOW = 2, ST_POS_RANGE = 4 };

/* ---- number formats ---------------------------------------------------- */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

float orc_bf16_to_f32(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

/* fp32 -> bfloat16, round to nearest, ties to even; NaN -> quiet NaN. */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u = f32_to_bits(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7fffu + lsb) >> 16);
}

/* fp32 -> IEEE binary16, round to nearest, ties to even. */
uint16_t orc_f32_to_f16(float f)
{
    uint32_t u = f32_to_bits(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t a = u & 0x7fffffffu;
    if (a > 0x7f800000u) return (uint16_t)(sign | 0x7e00u);        /* NaN */
    if (a >= 0x477ff000u) return (uint16_t)(sign | 0x7c00u);       /* >= 65520 -> Inf */
    if (a >= 0x38800000u) {                                         /* >= 2^-14: normal */
        uint32_t mant = a & 0x7fffffu;
        uint32_t e = (a >> 23) - 127u + 15u;
        uint32_t h = (e << 10) | (mant >> 13);
        uint32_t rem = mant & 0x1fffu;
        if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u;
        return (uint16_t)(sign | h);
    }
    if (a < 0x00800000u) return sign;                               /* fp32 subnormal: far below */
    /* half subnormal: value = M * 2^(E-150), unit 2^-24, so k = M * 2^(E-126) */
    uint32_t M = (a & 0x7fffffu) | 0x800000u;
    int shift = 126 - (int)(a >> 23);                               /* >= 14 here */
    if (shift >= 32) return sign;
    uint32_t k = M >> shift;
    uint32_t rem = M & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (k & 1u))) k += 1u;
    return (uint16_t)(sign | k);
}

float orc_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1fu, m = h & 0x3ffu;
    if (e == 0x1f) return bits_to_f32(sign | 0x7f800000u | (m << 13));
    if (e == 0) {
        float v = (float)m * 5.9604644775390625e-08f;               /* m * 2^-24, exact */
        return sign ? -v : v;
    }
    return bits_to_f32(sign | ((e - 15u + 127u) << 23) | (m << 13));
}

/* ---- RoPE table ---------------------------------------------------------- */

/* cos/sin table [max_pos][d_h/2]: fp32 of the fp64 cos/sin of m * w_k, with
 * w_k = theta^(-2k/d_h) in fp64 (or inv_freq[k] when given). */
int orc_rope_table(float *cos_t, float *sin_t, int max_pos, int d_h, double theta,
                   const double *inv_freq)
{
    int P = d_h / 2;
    if (max_pos < 0 || d_h < 2 || (d_h & 1)) return -1;
    for (int k = 0; k < P; ++k) {
        double w = inv_freq ? inv_freq[k] : pow(theta, -(2.0 * (double)k) / (double)d_h);
        for (int m = 0; m < max_pos; ++m) {
            double ang = (double)m * w;
            cos_t[(int64_t)m * P + k] = (float)cos(ang);
            sin_t[(int64_t)m * P + k] = (float)sin(ang);
        }
    }
    return 0;
}

/* Split table: rows [0, 64) hold cos/sin of l * w_k (l = 0..63), rows [64, 64 + n_high)
 * hold cos/sin of (64 h) * w_k, n_high = ceil(max_pos / 64); each entry fp32 of the fp64
 * value.  A position m = 64 h + l turns a pair by 64 h w_k and then by l w_k: plane
 * rotations of one pair add their angles (paper summary, "Problem statement": RoPE turns
 * fixed 2-D frequency pairs by a position-dependent angle).  Returns the row count used,
 * or -1. */
int orc_rope_table_split(float *cos_t, float *sin_t, int max_pos, int d_h, double theta,
                         const double *inv_freq)
{
    int P = d_h / 2;
    if (max_pos < 1 || d_h < 2 || (d_h & 1)) return -1;
    int rows = 64 + (max_pos + 63) / 64;
    for (int k = 0; k < P; ++k) {
        double w = inv_freq ? inv_freq[k] : pow(theta, -(2.0 * (double)k) / (double)d_h);
        for (int r = 0; r < rows; ++r) {
            double m = r < 64 ? (double)r : (double)(r - 64) * 64.0;
            double ang = m * w;
            cos_t[(int64_t)r * P + k] = (float)cos(ang);
            sin_t[(int64_t)r * P + k] = (float)sin(ang);
        }
    }
    return rows;
}

/* ---- steps of the transform ---------------------------------------------- */

static void pair_of(int k, int P, int style, int *ia, int *ib)
{
    if (style == ROPE_HALF) { *ia = k; *ib = k + P; }
    else                    { *ia = 2 * k; *ib = 2 * k + 1; }
}

/* (a, b) -> (a c - b s, a s + b c) on every pair, fp32 as documented above. */
static void rotate_pairs(float *x, int d_h, int style, const float *c, const float *s)
{
    int P = d_h / 2;
    for (int k = 0; k < P; ++k) {
        int ia, ib;
        pair_of(k, P, style, &ia, &ib);
        float a = x[ia], b = x[ib];
        float bs = b * s[k];
        float bc = b * c[k];
        x[ia] = fmaf(a, c[k], -bs);
        x[ib] = fmaf(a, s[k], bc);
    }
}

/* Unnormalised fast Walsh-Hadamard transform of n values, strides 1, 2, ..., n/2. */
void orc_fwht(float *x, int n)
{
    for (int h = 1; h < n; h *= 2)
        for (int i = 0; i < n; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                float u = x[j], v = x[j + h];
                x[j] = u + v;
                x[j + h] = u - v;
            }
}

static void hadamard_blocks(float *x, int d_h, int n)
{
    float kappa = (float)(1.0 / sqrt((double)n));
    for (int j = 0; j < d_h; j += n) orc_fwht(x + j, n);
    for (int i = 0; i < d_h; ++i) x[i] = x[i] * kappa;
}

/* A split table's entry for position m = 64 h + l: the high row's (c_h, s_h) turned by the
 * low row's (c_l, s_l) with the pair-rotation steps, c = fma(c_h, c_l, -(s_h*s_l)),
 * s = fma(c_h, s_l, s_h*c_l) (two plane rotations of one pair add their angles). */
static void split_table_entry(int P, const float *ch, const float *sh, const float *cl,
                              const float *sl, float *cc, float *ss)
{
    for (int k = 0; k < P; ++k) {
        float c = ch[k], s = sh[k];
        float ssl = s * sl[k];
        float scl = s * cl[k];
        cc[k] = fmaf(c, cl[k], -ssl);
        ss[k] = fmaf(c, sl[k], scl);
    }
}

/* One row in place, in the order of the method: RoPE with the table entries (ct, st); in
 * the pairwise modes the pair rotation by phi (cphi, sphi) after it; then the mode's
 * Hadamard mixing. */
static void transform_row(float *x, int d_h, int style, const float *ct, const float *st,
                          const float *cphi, const float *sphi, int mode, int b)
{
    rotate_pairs(x, d_h, style, ct, st);
    if (mode == MODE_PAIRWISE || mode == MODE_PAIRWISE_HADAMARD)
        rotate_pairs(x, d_h, style, cphi, sphi);
    if (mode == MODE_HADAMARD || mode == MODE_PAIRWISE_HADAMARD)
        hadamard_blocks(x, d_h, d_h);
    else if (mode == MODE_BLOCK_HADAMARD)
        hadamard_blocks(x, d_h, b);
}

/* Quantise one group of g transformed K values; returns status bits. */
static int quantize_group(const float *x, int g, int8_t *codes, uint16_t *scale)
{
    int st = 0;
    float amax = 0.0f;
    for (int i = 0; i < g; ++i) {
        if (!isfinite(x[i])) { st |= ST_NONFINITE; continue; }
        float v = fabsf(x[i]);
        if (v > amax) amax = v;
    }
    if (!(amax >= 0x1p-125f)) {
        for (int i = 0; i < g; ++i) codes[i] = 0;
        *scale = 0;
        return st;
    }
    float r = 7.0f / amax;
    for (int i = 0; i < g; ++i) {
        /* the product of two fp32 values is exact in fp64; round it once */
        double q = rint((double)x[i] * (double)r);
        if (!(q == q)) q = 0.0;                /* NaN element (flagged above) */
        if (q > 7.0) q = 7.0;
        if (q < -7.0) q = -7.0;
        codes[i] = (int8_t)q;
    }
    float s = amax / 7.0f;
    *scale = orc_f32_to_f16(s);
    if ((*scale & 0x7fffu) == 0x7c00u) st |= ST_SCALE_OVERFLOW;
    return st;
}

/* The quantiser alone, on fp32 rows x [rows][d_h] (already transformed): packed codes
 * [rows][d_h/2] and fp16 scales [rows][d_h/group], by the same rule as below.  Returns the
 * status bits, or -1 on a bad argument. */
int orc_quantize_rows(const float *x, int64_t rows, int d_h, int group, uint8_t *k_codes,
                      uint16_t *k_scales)
{
    int8_t codes[1024];
    int st = 0;
    if (d_h < 2 || (d_h & 1) || d_h > 1024 || group < 2 || d_h % group) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const float *row = x + r * d_h;
        for (int gi = 0; gi < d_h / group; ++gi)
            st |= quantize_group(row + gi * group, group, codes + gi * group,
                                 k_scales + r * (d_h / group) + gi);
        for (int j = 0; j < d_h / 2; ++j)
            k_codes[r * (d_h / 2) + j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));
    }
    return st;
}

/* Value rows: no RoPE; the full-head normalised Hadamard ("LLM旋转量化笔记" §3.2.2,
 * V~ = V H_head), then the K quantiser.  v [T][Hkv][d_h] bf16 bits; outputs as for K.
 * Returns the status bits, or -1 on a bad argument. */
int orc_value_quantize(const uint16_t *v, int64_t rows, int d_h, int group, uint8_t *v_codes,
                       uint16_t *v_scales, float *v_f32)
{
    float row[1024];
    int8_t codes[1024];
    int st = 0;
    if (d_h < 2 || d_h > 1024 || (d_h & (d_h - 1)) || group < 2 || d_h % group) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int i = 0; i < d_h; ++i) row[i] = orc_bf16_to_f32(v[r * d_h + i]);
        hadamard_blocks(row, d_h, d_h);
        if (v_f32) memcpy(v_f32 + r * d_h, row, sizeof(float) * d_h);
        for (int gi = 0; gi < d_h / group; ++gi)
            st |= quantize_group(row + gi * group, group, codes + gi * group,
                                 v_scales + r * (d_h / group) + gi);
        for (int j = 0; j < d_h / 2; ++j)
            v_codes[r * (d_h / 2) + j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));
    }
    return st;
}

/* ---- the whole transform + quantisation ------------------------------------ */

/*
 * q [T][Hq][d_h], k [T][Hkv][d_h]: bf16 bits.  pos [T].  cos_t/sin_t [max_pos][d_h/2],
 * or, with STYLE_SPLIT_TABLE in style, the split tables of orc_rope_table_split (positions
 * still range over [0, max_pos)).
 * phi [d_h/2] (used by the pairwise modes).  Outputs: q_out bf16 [T][Hq][d_h],
 * k_codes [T][Hkv][d_h/2], k_scales fp16 [T][Hkv][d_h/group]; optional fp32 copies
 * of the transformed rows k_f32 [T][Hkv][d_h] and q_f32 [T][Hq][d_h] (NULL to skip).
 * Returns 0, or -1 on a bad argument.
 */
int orc_transform_quantize(const uint16_t *q, const uint16_t *k, const int32_t *pos, int64_t T,
                           int Hq, int Hkv, int d_h, int style, const float *cos_t,
                           const float *sin_t, int max_pos, const float *phi, int mode, int b,
                           int group, uint16_t *q_out, uint8_t *k_codes, uint16_t *k_scales,
                           float *k_f32, float *q_f32, int *status)
{
    int P = d_h / 2;
    if (d_h < 2 || (d_h & 1) || d_h > 1024 || group < 2 || d_h % group || max_pos < 1)
        return -1;
    if (mode == MODE_BLOCK_HADAMARD && (b < 2 || b > d_h || (b & (b - 1)) || d_h % b))
        return -1;
    if ((mode == MODE_HADAMARD || mode == MODE_PAIRWISE_HADAMARD) && (d_h & (d_h - 1)))
        return -1;
    int split = (style & STYLE_SPLIT_TABLE) != 0;
    style &= ~STYLE_SPLIT_TABLE;
    float cphi[512], sphi[512], crope[512], srope[512], row[1024];
    int8_t codes[1024];
    if (mode == MODE_PAIRWISE || mode == MODE_PAIRWISE_HADAMARD) {
        if (!phi) return -1;
        for (int j = 0; j < P; ++j) {
            cphi[j] = (float)cos((double)phi[j]);
            sphi[j] = (float)sin((double)phi[j]);
        }
    }
    int st = 0;
    for (int64_t t = 0; t < T; ++t) {
        int m = pos[t];
        if (m < 0 || m >= max_pos) { st |= ST_POS_RANGE; m = m < 0 ? 0 : max_pos - 1; }
        const float *ct = cos_t + (int64_t)m * P, *stb = sin_t + (int64_t)m * P;
        if (split) {
            /* the high row's rotation turned by the low row's, with the pair-rotation
             * steps: c = fma(c_h, c_l, -(s_h*s_l)), s = fma(c_h, s_l, s_h*c_l) */
            const float *cl = cos_t + (int64_t)(m % 64) * P, *sl = sin_t + (int64_t)(m % 64) * P;
            const float *ch = cos_t + (int64_t)(64 + m / 64) * P;
            const float *sh = sin_t + (int64_t)(64 + m / 64) * P;
            split_table_entry(P, ch, sh, cl, sl, crope, srope);
            ct = crope;
            stb = srope;
        }
        for (int h = 0; h < Hq; ++h) {
            const uint16_t *src = q + (t * Hq + h) * d_h;
            for (int i = 0; i < d_h; ++i) row[i] = orc_bf16_to_f32(src[i]);
            transform_row(row, d_h, style, ct, stb, cphi, sphi, mode, b);
            uint16_t *dst = q_out + (t * Hq + h) * d_h;
            for (int i = 0; i < d_h; ++i) dst[i] = orc_f32_to_bf16(row[i]);
            if (q_f32) memcpy(q_f32 + (t * Hq + h) * d_h, row, sizeof(float) * d_h);
        }
        for (int h = 0; h < Hkv; ++h) {
            int64_t r = t * Hkv + h;
            const uint16_t *src = k + r * d_h;
            for (int i = 0; i < d_h; ++i) row[i] = orc_bf16_to_f32(src[i]);
            transform_row(row, d_h, style, ct, stb, cphi, sphi, mode, b);
            if (k_f32) memcpy(k_f32 + r * d_h, row, sizeof(float) * d_h);
            for (int gi = 0; gi < d_h / group; ++gi)
                st |= quantize_group(row + gi * group, group, codes + gi * group,
                                     k_scales + r * (d_h / group) + gi);
            for (int j = 0; j < P; ++j)
                k_codes[r * P + j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));
        }
    }
    if (status) *status |= st;
    return 0;
}
