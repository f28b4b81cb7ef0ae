/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the normalise-then-rotate path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or constant with the CUDA library and never calls it.
 *
 * Every function is the plain definition, written as loops in the order the
 * pages state the steps, with fp64 arithmetic except where the pages fix a
 * precision:
 *   - the rotation angle is the fp32 product fp32(pos) * inv_freq
 *     (vLLM mrope_vit_setup page, _vit_mrope_setup_kernel: positions are
 *     cast to fp32 and multiplied by the fp32 inverse frequency);
 *   - the residual stream is rounded to bf16 before it is normalised
 *     (vllm.cpp #185 "decode RmsNorm ran on ONE workgroup", the
 *     vt_round_through paragraph: the summed residual carries bf16 rounding);
 *   - optionally, the normalised value is rounded to bf16 before rotation
 *     (vllm-omni #7600, review of the interleaved tile: a bf16-rounded
 *     normalised value, an fp32 rotation and one final rounding), or rounded
 *     at the two points of the eager RMSNorm (vLLM #26234, rms_norm_kernel:
 *     the normalised value cast to bf16, then a bf16 product with the
 *     weight).
 * Outputs are returned unrounded (fp64), except bf16 streams that are
 * themselves the result (the residual) and fp32 planes.
 *
 * Parity pins live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ---------------------------------------------------------------- bf16 -- */

static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 (ties to even), returned as its bits.
 * bf16 = 1 sign bit, 8 exponent bits, 7 stored mantissa bits: 8 significant
 * bits for normals, a fixed quantum of 2^-133 below 2^-126. */
uint16_t oracle_bf16_round(double v)
{
    if (isnan(v))
        return 0x7fc0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return (uint16_t)(sign | 0x7f80);
    int ex;
    frexp(a, &ex);                 /* a = f * 2^ex with f in [0.5, 1) */
    int quantum = ex - 8;          /* weight of the last of 8 significant bits */
    if (quantum < -133)
        quantum = -133;
    double r = nearbyint(ldexp(a, -quantum));   /* ties to even (default mode) */
    double q = ldexp(r, quantum);
    if (q > 3.3895313892515355e38) /* above the largest finite bf16 */
        return (uint16_t)(sign | 0x7f80);
    float f = (float)q;            /* exact: at most 9 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7fff));
}

static double bf16_rounded_value(double v) { return bf16_value(oracle_bf16_round(v)); }

/* ------------------------------------------------------- section rules -- */
/* Axis codes: 0 = t, 1 = h, 2 = w, 3 = e (fourth position row). */

enum { SEC_NONE = 0, SEC_CONTIGUOUS = 1, SEC_INTERLEAVED = 2,
       SEC_INTERLEAVED_QUOTA = 3, SEC_IMROPE = 4 };

/* Contiguous sections: the first s0 pairs take t, the next s1 take h, the
 * next s2 take w (vLLM mrope_vit_setup page: the t, h and w planes hold
 * columns [0,half_t), [half_t, half_t+half_h), [half_t+half_h, half_rot)). */
static int axis_contiguous(const int32_t *s, int64_t j)
{
    if (j < s[0])
        return 0;
    if (j < (int64_t)s[0] + s[1])
        return 1;
    return 2;
}

static int64_t min3(int64_t a, int64_t b, int64_t c)
{
    int64_t m = a < b ? a : b;
    return m < c ? m : c;
}

/* Interleaved, tail contiguous: pair j takes axis j mod 3 while
 * j < 3 * min(s0, s1, s2); past that it takes the axis of its contiguous
 * section (the workload statement of the interleaved mRoPE configuration). */
static int axis_interleaved(const int32_t *s, int64_t j)
{
    int64_t m = min3(s[0], s[1], s[2]);
    if (j < 3 * m)
        return (int)(j % 3);
    return axis_contiguous(s, j);
}

/* Interleaved, tail by remaining quota: the same t,h,w cycle for the first
 * 3 * min pairs; each later pair goes to the first axis (t, then h, then w)
 * that has not yet received its section's count of pairs. */
static int axis_interleaved_quota(const int32_t *s, int64_t j)
{
    int64_t m = min3(s[0], s[1], s[2]);
    if (j < 3 * m)
        return (int)(j % 3);
    int64_t k = j - 3 * m;
    for (int a = 0; a < 3; ++a) {
        int64_t left = (int64_t)s[a] - m;
        if (k < left)
            return a;
        k -= left;
    }
    return 2;
}

/* Sector rule of the interleaved multi-section rotation with a fourth
 * section (llama.cpp fork PR #286, "The change", and the review that checks
 * it against ggml_mrope_cache_init): the sector is the pair index modulo the
 * sum of the four sections; sector mod 3 == 1 selects h while the sector is
 * below 3*s1, mod 3 == 2 selects w below 3*s2, mod 3 == 0 selects t below
 * 3*s0, and every other sector takes the fourth ("e") row. */
static int axis_imrope(const int32_t *s, int64_t j)
{
    int64_t total = (int64_t)s[0] + s[1] + s[2] + s[3];
    int64_t sector = j % total;
    int64_t r = sector % 3;
    if (r == 1 && sector < 3 * (int64_t)s[1])
        return 1;
    if (r == 2 && sector < 3 * (int64_t)s[2])
        return 2;
    if (r == 0 && sector < 3 * (int64_t)s[0])
        return 0;
    return 3;
}

int oracle_section_axis(int mode, const int32_t *sections, int64_t j)
{
    switch (mode) {
    case SEC_NONE: return 0;
    case SEC_CONTIGUOUS: return axis_contiguous(sections, j);
    case SEC_INTERLEAVED: return axis_interleaved(sections, j);
    case SEC_INTERLEAVED_QUOTA: return axis_interleaved_quota(sections, j);
    case SEC_IMROPE: return axis_imrope(sections, j);
    default: return -1;
    }
}

void oracle_section_map(int mode, const int32_t *sections, int64_t P, int8_t *axis_out)
{
    for (int64_t j = 0; j < P; ++j)
        axis_out[j] = (int8_t)oracle_section_axis(mode, sections, j);
}

/* --------------------------------------------------------------- angles -- */

typedef struct {
    int32_t kind;              /* 0: positions + inv_freq, 1: cos/sin table(s) */
    int32_t section_mode;
    int32_t sections[4];
    const int32_t *positions;  /* [rows, pos_row_stride] */
    int64_t pos_row_stride;    /* tokens per position row (whole buffer) */
    const float *inv_freq;     /* [P] */
    const float *cos_tab;      /* [planes, n_rows, ld] */
    const float *sin_tab;
    int64_t plane_stride;      /* elements between planes */
    int64_t ld;                /* elements between table rows */
    int64_t token_offset;      /* added to the launch-local token index */
} oracle_angle;

/* cos/sin of pair j for launch-local token n. */
static void angle_of(const oracle_angle *A, int64_t n, int64_t j, double *c, double *s)
{
    int64_t tok = A->token_offset + n;
    int axis = oracle_section_axis(A->section_mode, A->sections, j);
    if (A->kind == 0) {
        int32_t pos = A->positions[(int64_t)axis * A->pos_row_stride + tok];
        float theta = (float)((float)pos * A->inv_freq[j]);   /* fp32 product */
        *c = cos((double)theta);
        *s = sin((double)theta);
    } else {
        int64_t at = (int64_t)axis * A->plane_stride + tok * A->ld + j;
        *c = (double)A->cos_tab[at];
        *s = (double)A->sin_tab[at];
    }
}

/* ----------------------------------------------------- per-row helpers -- */

/* Rounding points of the normalised value (see oracle_qk_norm_rope). */
enum { ROUND_NONE = 0, ROUND_NORMALIZED = 1, ROUND_EAGER = 2 };

/* Distance, in bf16 quanta, below which a value counts as sitting on a
 * rounding midpoint: a single-precision evaluation of the same value (the
 * GPU's fp32 sum of squares and rsqrt differ from fp64 by about 1e-6
 * relative, a few 1e-4 quanta) may round it to the other neighbour. */
#define TIE_TOL 1e-3

/* 1 if v lies within TIE_TOL quanta of a bf16 rounding midpoint. */
static int near_bf16_tie(double v)
{
    double a = fabs(v);
    if (a == 0.0 || isinf(a) || isnan(a))
        return 0;
    int ex;
    frexp(a, &ex);
    int quantum = ex - 8;
    if (quantum < -133)
        quantum = -133;
    double u = ldexp(a, -quantum);   /* a in quanta */
    double f = u - floor(u);
    return fabs(f - 0.5) < TIE_TOL;
}

/* y = x / sqrt(mean(x^2) + eps) * gamma  (RMSNorm over the head dim), with the
 * rounding points of round_mode:
 *   ROUND_NONE        y unrounded;
 *   ROUND_NORMALIZED  y = bf16(x r gamma);
 *   ROUND_EAGER       y = bf16(bf16(x r) * gamma): the eager RMSNorm casts the
 *                     normalised value to the activation type, then multiplies
 *                     it by the bf16 weight with a bf16 result (vLLM #26234,
 *                     the rms_norm_kernel line the review quotes).
 * tie[d] (nullable) = 1 where the value rounded first sat on a midpoint. */
static void rms_norm_head(const uint16_t *x, const uint16_t *gamma, int64_t D, double eps,
                          int round_mode, double *y, uint8_t *tie)
{
    double ss = 0.0;
    for (int64_t d = 0; d < D; ++d) {
        double v = bf16_value(x[d]);
        ss += v * v;
    }
    double inv_rms = 1.0 / sqrt(ss / (double)D + eps);
    for (int64_t d = 0; d < D; ++d) {
        double xr = bf16_value(x[d]) * inv_rms;
        double g = bf16_value(gamma[d]);
        if (round_mode == ROUND_EAGER) {
            if (tie)
                tie[d] = (uint8_t)near_bf16_tie(xr);
            y[d] = bf16_rounded_value(bf16_rounded_value(xr) * g);
        } else if (round_mode == ROUND_NORMALIZED) {
            if (tie)
                tie[d] = (uint8_t)near_bf16_tie(xr * g);
            y[d] = bf16_rounded_value(xr * g);
        } else {
            if (tie)
                tie[d] = 0;
            y[d] = xr * g;
        }
    }
}

/* Rotate the first rot dims in pairs: NeoX pairs (j, j + rot/2), GPT-J pairs
 * (2j, 2j+1); a' = a cos - b sin, b' = b cos + a sin.  Dims >= rot pass. */
static void rotate_head(double *y, int64_t rot, int pairing, const oracle_angle *A,
                        int64_t n)
{
    int64_t P = rot / 2;
    for (int64_t j = 0; j < P; ++j) {
        int64_t ia = pairing == 0 ? j : 2 * j;
        int64_t ib = pairing == 0 ? j + P : 2 * j + 1;
        double c, s;
        angle_of(A, n, j, &c, &s);
        double a = y[ia], b = y[ib];
        y[ia] = a * c - b * s;
        y[ib] = b * c + a * s;
    }
}

/* ------------------------------------------------ QK norm + cat + rope -- */
/*
 * Streams are dense [T_s, H, D] bf16 (bits).  The joint output is the
 * concatenation over streams in order (text first), [sum T_s, H, D], fp64.
 * do_norm = 0 skips the RMSNorm (plain rotation of the input values).
 * round_mode (with do_norm): the rounding points of the normalised value, as
 * rms_norm_head states them; the rotation itself is exact (fp64) and the
 * output unrounded.
 * tie_q / tie_k (nullable, [sum T_s, H, D]): 1 where an output element
 * depends on a normalised value that sat on a bf16 rounding midpoint (the
 * element itself, or its rotation partner).
 */
int oracle_qk_norm_rope(int n_streams, const int64_t *T_s,
                        const uint16_t *const *q_s, const uint16_t *const *k_s,
                        const uint16_t *const *gq_s, const uint16_t *const *gk_s,
                        int64_t Hq, int64_t Hk, int64_t D, int64_t rot, int pairing,
                        double eps, int do_norm, int round_mode,
                        const oracle_angle *A, double *q_out, double *k_out,
                        uint8_t *tie_q, uint8_t *tie_k)
{
    if (D <= 0 || rot < 0 || rot > D || (rot & 1) || D > 4096)
        return -1;
    if (round_mode < ROUND_NONE || round_mode > ROUND_EAGER)
        return -1;
    double y[4096];
    uint8_t tie[4096];
    int64_t n = 0;                  /* joint token index */
    for (int s = 0; s < n_streams; ++s) {
        for (int64_t t = 0; t < T_s[s]; ++t, ++n) {
            for (int which = 0; which < 2; ++which) {
                int64_t H = which == 0 ? Hq : Hk;
                const uint16_t *src = which == 0 ? q_s[s] : k_s[s];
                const uint16_t *gam = which == 0 ? gq_s[s] : gk_s[s];
                double *dst = which == 0 ? q_out : k_out;
                uint8_t *tdst = which == 0 ? tie_q : tie_k;
                for (int64_t h = 0; h < H; ++h) {
                    const uint16_t *x = src + (t * H + h) * D;
                    if (do_norm) {
                        rms_norm_head(x, gam, D, eps, round_mode, y, tie);
                    } else {
                        for (int64_t d = 0; d < D; ++d) {
                            y[d] = bf16_value(x[d]);
                            tie[d] = 0;
                        }
                    }
                    rotate_head(y, rot, pairing, A, n);
                    memcpy(dst + (n * H + h) * D, y, (size_t)D * sizeof(double));
                    if (tdst) {
                        uint8_t *to = tdst + (n * H + h) * D;
                        memcpy(to, tie, (size_t)D);
                        for (int64_t j = 0; j < rot / 2; ++j) {
                            int64_t ia = pairing == 0 ? j : 2 * j;
                            int64_t ib = pairing == 0 ? j + rot / 2 : 2 * j + 1;
                            uint8_t any = (uint8_t)(tie[ia] | tie[ib]);
                            to[ia] = any;
                            to[ib] = any;
                        }
                    }
                }
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------ ViT setup -- */
/*
 * Positions of every token of every grid, enumerated by nested loops in the
 * token order of the ViT after spatial merging (vLLM mrope_vit_setup page,
 * _vit_mrope_setup_kernel docstring and comments): frame t, then merge-block
 * row bh, merge-block column bw, then the m x m patch inside the block
 * (row mh, column mw).  h = bh*m + mh, w = bw*m + mw.
 * Returns the token count, or -1 if a grid's h or w is not a multiple of m.
 */
int64_t oracle_vit_positions(const int32_t *grids, int64_t G, int32_t m, int32_t *pos,
                             int64_t N)
{
    int64_t n = 0;
    for (int64_t g = 0; g < G; ++g) {
        int32_t T = grids[3 * g], Hh = grids[3 * g + 1], W = grids[3 * g + 2];
        if (m <= 0 || Hh % m || W % m)
            return -1;
        for (int32_t t = 0; t < T; ++t)
            for (int32_t bh = 0; bh < Hh / m; ++bh)
                for (int32_t bw = 0; bw < W / m; ++bw)
                    for (int32_t mh = 0; mh < m; ++mh)
                        for (int32_t mw = 0; mw < m; ++mw) {
                            if (pos && n < N) {
                                pos[n] = t;
                                pos[N + n] = bh * m + mh;
                                pos[2 * N + n] = bw * m + mw;
                            }
                            ++n;
                        }
    }
    return n;
}

/*
 * The (3, N, P) cos/sin planes, P = nt + nh + nw.  Plane a holds, in its own
 * section columns only, cos/sin(fp32(pos_a) * inv_a[col - offset_a]); the
 * other columns are not written (same page: "Only each axis's mrope section
 * columns are written").  written[] (may be NULL) marks the written cells.
 */
void oracle_vit_planes(const int32_t *pos, int64_t N,
                       const float *inv_t, int64_t nt, const float *inv_h, int64_t nh,
                       const float *inv_w, int64_t nw,
                       float *cos_out, float *sin_out, uint8_t *written)
{
    int64_t P = nt + nh + nw;
    const float *inv[3] = {inv_t, inv_h, inv_w};
    int64_t off[3] = {0, nt, nt + nh};
    int64_t len[3] = {nt, nh, nw};
    for (int a = 0; a < 3; ++a)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t c = off[a]; c < off[a] + len[a]; ++c) {
                float theta = (float)((float)pos[a * N + n] * inv[a][c - off[a]]);
                int64_t at = ((int64_t)a * N + n) * P + c;
                cos_out[at] = (float)cos((double)theta);
                sin_out[at] = (float)sin((double)theta);
                if (written)
                    written[at] = 1;
            }
}

/* ------------------------------------------------ RMSNorm with residual -- */
/*
 * s = bf16(x + residual) is the new residual (returned as bits);
 * out = s / sqrt(mean(s^2) + eps) * gamma, in fp64.
 */
void oracle_rms_norm_residual(const uint16_t *x, const uint16_t *res, const uint16_t *gamma,
                              int64_t R, int64_t hidden, double eps,
                              uint16_t *res_out, double *out)
{
    for (int64_t r = 0; r < R; ++r) {
        const uint16_t *xr = x + r * hidden;
        const uint16_t *rr = res + r * hidden;
        uint16_t *ro = res_out + r * hidden;
        double ss = 0.0;
        for (int64_t i = 0; i < hidden; ++i) {
            ro[i] = oracle_bf16_round(bf16_value(xr[i]) + bf16_value(rr[i]));
            double s = bf16_value(ro[i]);
            ss += s * s;
        }
        double inv_rms = 1.0 / sqrt(ss / (double)hidden + eps);
        for (int64_t i = 0; i < hidden; ++i)
            out[r * hidden + i] = bf16_value(ro[i]) * inv_rms * bf16_value(gamma[i]);
    }
}

/* ------------------------------------------------------ FP8 E4M3 encoding -- */
/*
 * The static-FP8 output of rms_norm_fp8 (vLLM #26234 names the fused
 * rms_norm_static_fp8_quant_kernel; the format is the OCP FP8 E4M3 "FN" one
 * that kernel family writes): 1 sign bit, 4 exponent bits with bias 7, 3
 * mantissa bits; exponent field 0 holds the subnormals m * 2^-9; there are no
 * infinities and S.1111.111 is NaN, so the largest finite magnitude is
 * 1.75 * 2^8 = 448.  Values are rounded to the nearest representable value,
 * ties to the even mantissa, and magnitudes above 448 saturate to 448.
 */
uint8_t oracle_fp8_e4m3(double v)
{
    if (isnan(v))
        return 0x7F;
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    unsigned code;
    if (a < ldexp(1.0, -6)) {
        /* subnormal grid: steps of 2^-9; a rounding up to 8 steps is the
         * smallest normal, whose code is 8 as well */
        code = (unsigned)nearbyint(a * 512.0);
    } else {
        int e;
        frexp(a, &e);          /* a = f * 2^e, f in [0.5, 1) */
        e -= 1;                /* a = g * 2^e, g in [1, 2) */
        double q = nearbyint(ldexp(a, 3 - e));   /* g * 8 rounded: 8 .. 16 */
        if (q >= 16.0) {
            q = 8.0;
            e += 1;
        }
        if (e + 7 > 15)
            return sign | 0x7E;
        code = ((unsigned)(e + 7) << 3) | ((unsigned)q - 8u);
    }
    if (code > 0x7E)
        code = 0x7E;
    return sign | (uint8_t)code;
}

void oracle_fp8_e4m3_array(const double *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_fp8_e4m3(v[i]);
}

/*
 * rms_norm_fp8: with a residual (res != NULL) s = bf16(x + residual) becomes
 * the new residual; without one s = x.  y = s / sqrt(mean(s^2) + eps) * gamma
 * in fp64; y_scaled = y / scale; codes = E4M3(y_scaled).
 */
void oracle_rms_norm_fp8(const uint16_t *x, const uint16_t *res, const uint16_t *gamma,
                         int64_t R, int64_t hidden, double eps, double scale,
                         uint16_t *res_out, double *y_scaled, uint8_t *codes)
{
    for (int64_t r = 0; r < R; ++r) {
        const uint16_t *xr = x + r * hidden;
        double ss = 0.0;
        for (int64_t i = 0; i < hidden; ++i) {
            double s;
            if (res) {
                res_out[r * hidden + i] =
                    oracle_bf16_round(bf16_value(xr[i]) + bf16_value(res[r * hidden + i]));
                s = bf16_value(res_out[r * hidden + i]);
            } else {
                s = bf16_value(xr[i]);
            }
            ss += s * s;
        }
        double inv_rms = 1.0 / sqrt(ss / (double)hidden + eps);
        for (int64_t i = 0; i < hidden; ++i) {
            double s = res ? bf16_value(res_out[r * hidden + i]) : bf16_value(xr[i]);
            double y = s * inv_rms * bf16_value(gamma[i]);
            y_scaled[r * hidden + i] = y / scale;
            codes[r * hidden + i] = oracle_fp8_e4m3(y / scale);
        }
    }
}
