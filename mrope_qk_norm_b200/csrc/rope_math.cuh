// rope_math.cuh -- the per-row arithmetic shared by every lane-group rope
// kernel (item and streaming): unpacking a lane's 16-byte vectors of a head
// row into packed fp32x2 couples, the row's sum of squares, normalisation and
// rotation, and packing back to bf16.  Keeping one copy of it is what makes
// the kernels bit-identical to one another.
//
// Couples.  A lane holds NQ "quads" of a head row, each quad two rotation
// pairs: A = the first members of the two pairs, B = the second members, as
// float2 so Blackwell's FFMA2 / FMUL2 work on both pairs at once.  NeoX
// (PAIRED layout): a lane's slot 0 is vector u of the first rotary half and
// slot 1 vector u + rot/16 of the second, so element i of slot 0 pairs with
// element i of slot 1; the slots past them (NT tail vectors) are normalised
// only.  GPT-J (VECTOR layout): pairs (2j, 2j+1) sit in one 32-bit word, two
// words make one quad.
//
// Rotation of a pair (a, b) by angle theta with c = cos, s = sin:
//   a' = a c - b s,   b' = b c + a s.
// With the per-head RMSNorm folded in (y = x r g, r = rsqrt(mean(x^2) + eps),
// g = gamma of the column) the rotated pair is
//   a' = r (a (g_a c) + b (-(g_b s))),   b' = r (b (g_b c) + a (g_a s)),
// so the four per-column products are formed once per work item and each
// row costs two FMUL2 + two FFMA2 + two FMUL2 per quad.
#pragma once

#include "qkr_internal.cuh"

namespace qkr {
namespace {

enum Layout { PAIRED = 0, VECTOR = 1, EXCHANGE = 2, PAIRX = 3 };

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }

__device__ __forceinline__ uint32_t word(const uint4 &v, int i)
{
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}
__device__ __forceinline__ void set_word(uint4 &v, int i, uint32_t w)
{
    if (i == 0) v.x = w;
    else if (i == 1) v.y = w;
    else if (i == 2) v.z = w;
    else v.w = w;
}

__device__ __forceinline__ float2 round2_bf16(float2 a)
{
    const uint32_t w = pack2(a.x, a.y);
    return f2(bf_lo(w), bf_hi(w));
}

// Quads per lane and tail vectors per lane of a layout with NS slots.
template <int LAYOUT, int NS>
struct RowShape {
    static constexpr int NQ = LAYOUT == PAIRED ? 4 : 2 * NS;
    static constexpr int NT = LAYOUT == PAIRED ? NS - 2 : 0;
    static constexpr int NTA = NT > 0 ? NT : 1;  // array extent
};

// Unpacks a lane's vectors of one row (or of the gamma row) into couples.
template <int LAYOUT, int NS>
__device__ __forceinline__ void unpack_row(const uint4 (&v)[NS],
                                           float2 (&A)[RowShape<LAYOUT, NS>::NQ],
                                           float2 (&B)[RowShape<LAYOUT, NS>::NQ],
                                           float2 (&T)[RowShape<LAYOUT, NS>::NTA][4])
{
    constexpr int NQ = RowShape<LAYOUT, NS>::NQ;
    constexpr int NT = RowShape<LAYOUT, NS>::NT;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        if (LAYOUT == PAIRED) {
            const uint32_t wa = word(v[0], q), wb = word(v[1], q);
            A[q] = f2(bf_lo(wa), bf_hi(wa));
            B[q] = f2(bf_lo(wb), bf_hi(wb));
        } else {
            const uint32_t w0 = word(v[q >> 1], 2 * (q & 1));
            const uint32_t w1 = word(v[q >> 1], 2 * (q & 1) + 1);
            A[q] = f2(bf_lo(w0), bf_lo(w1));
            B[q] = f2(bf_hi(w0), bf_hi(w1));
        }
    }
#pragma unroll
    for (int k = 0; k < NT; ++k)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t w = word(v[2 + k], i);
            T[k][i] = f2(bf_lo(w), bf_hi(w));
        }
}

// This lane's part of the row's sum of squares (fixed order).
template <int LAYOUT, int NS>
__device__ __forceinline__ float row_sumsq(const float2 (&A)[RowShape<LAYOUT, NS>::NQ],
                                           const float2 (&B)[RowShape<LAYOUT, NS>::NQ],
                                           const float2 (&T)[RowShape<LAYOUT, NS>::NTA][4])
{
    constexpr int NQ = RowShape<LAYOUT, NS>::NQ;
    constexpr int NT = RowShape<LAYOUT, NS>::NT;
    float2 acc = f2(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        acc = __ffma2_rn(A[q], A[q], acc);
        acc = __ffma2_rn(B[q], B[q], acc);
    }
#pragma unroll
    for (int k = 0; k < NT; ++k)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            acc = __ffma2_rn(T[k][i], T[k][i], acc);
    return acc.x + acc.y;
}

// Per-work-item coefficients of the rotation (see the header comment).
// FOLD (norm with no intermediate rounding, kRoundNone): K0 = g_a c,
// K1 = -(g_b s), K2 = g_b c, K3 = g_a s.  Otherwise K0 = c, K1 = -s, K2 = c,
// K3 = s, and GA / GB keep the gammas for the explicit normalisation.
template <int NQ, bool FOLD>
struct RotCoef {
    float2 K0[NQ], K1[NQ], K2[NQ], K3[NQ];
};

template <int NQ, bool FOLD>
__device__ __forceinline__ void make_coef(RotCoef<NQ, FOLD> &k, const float2 (&C)[NQ],
                                          const float2 (&S)[NQ], const float2 (&GA)[NQ],
                                          const float2 (&GB)[NQ])
{
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        if (FOLD) {
            k.K0[q] = __fmul2_rn(GA[q], C[q]);
            const float2 bs = __fmul2_rn(GB[q], S[q]);
            k.K1[q] = f2(-bs.x, -bs.y);
            k.K2[q] = __fmul2_rn(GB[q], C[q]);
            k.K3[q] = __fmul2_rn(GA[q], S[q]);
        } else {
            k.K0[q] = C[q];
            k.K1[q] = f2(-S[q].x, -S[q].y);
            k.K2[q] = C[q];
            k.K3[q] = S[q];
        }
    }
}

// Rounding points of the normalised value (RMODE; RopeParams::round_norm):
//   kRoundNone       y = x r gamma stays fp32 (gamma folded into the rotation
//                    coefficients), the rotation is fused multiply-adds, and
//                    only the output is rounded;
//   kRoundNormalized y = bf16(x r gamma) before an fp32 rotation
//                    (QKR_FLAG_ROUND_NORMALIZED_BF16);
//   kRoundEager      y = bf16(bf16(x r) gamma) -- the eager RMSNorm casts the
//                    normalised value to bf16, then multiplies by the bf16
//                    weight -- and the rotation's products and sums are each
//                    rounded to fp32, with no contraction into fused
//                    multiply-adds (QKR_FLAG_EAGER_ROUNDING).
enum { kRoundNone = 0, kRoundNormalized = 1, kRoundEager = 2 };

// Normalise (NORM: by r and gamma) and rotate one row's couples in place.
template <int LAYOUT, int NS, bool NORM, int RMODE>
__device__ __forceinline__ void norm_rotate(
    float2 (&A)[RowShape<LAYOUT, NS>::NQ], float2 (&B)[RowShape<LAYOUT, NS>::NQ],
    float2 (&T)[RowShape<LAYOUT, NS>::NTA][4], float r,
    const RotCoef<RowShape<LAYOUT, NS>::NQ, NORM && RMODE == kRoundNone> &k,
    const float2 (&GA)[RowShape<LAYOUT, NS>::NQ], const float2 (&GB)[RowShape<LAYOUT, NS>::NQ],
    const float2 (&GT)[RowShape<LAYOUT, NS>::NTA][4])
{
    constexpr int NQ = RowShape<LAYOUT, NS>::NQ;
    constexpr int NT = RowShape<LAYOUT, NS>::NT;
    const float2 r2 = f2(r, r);
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        float2 a = A[q], b = B[q];
        if (NORM && RMODE == kRoundNormalized) {
            a = round2_bf16(__fmul2_rn(__fmul2_rn(a, r2), GA[q]));
            b = round2_bf16(__fmul2_rn(__fmul2_rn(b, r2), GB[q]));
        }
        if (NORM && RMODE == kRoundEager) {
            a = round2_bf16(__fmul2_rn(round2_bf16(__fmul2_rn(a, r2)), GA[q]));
            b = round2_bf16(__fmul2_rn(round2_bf16(__fmul2_rn(b, r2)), GB[q]));
        }
        float2 a2, b2;
        if (RMODE == kRoundEager) {
            // K1 = -s: a c + b (-s) is a c - b s with every step rounded
            a2 = __fadd2_rn(__fmul2_rn(a, k.K0[q]), __fmul2_rn(b, k.K1[q]));
            b2 = __fadd2_rn(__fmul2_rn(b, k.K2[q]), __fmul2_rn(a, k.K3[q]));
        } else {
            a2 = __ffma2_rn(b, k.K1[q], __fmul2_rn(a, k.K0[q]));
            b2 = __ffma2_rn(a, k.K3[q], __fmul2_rn(b, k.K2[q]));
        }
        if (NORM && RMODE == kRoundNone) {
            a2 = __fmul2_rn(a2, r2);
            b2 = __fmul2_rn(b2, r2);
        }
        A[q] = a2;
        B[q] = b2;
    }
    if (NORM) {
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                T[t][i] = RMODE == kRoundEager
                              ? round2_bf16(__fmul2_rn(round2_bf16(__fmul2_rn(T[t][i], r2)),
                                                       GT[t][i]))
                              : __fmul2_rn(__fmul2_rn(T[t][i], r2), GT[t][i]);
    }
}

// PAIRX layout: a lane holds one 16-byte vector of one rotary half (lane
// l < rot/16 the first half, the others the second) and takes its partner's
// vector from lane l ^ rot/16 by shuffle; with the two it forms the same
// couples as a PAIRED lane and computes only its own half: a' (first half)
// or b' (second), with the very operations norm_rotate uses for it, so the
// results are bit-identical to the PAIRED layout's.  Kc / Kp are the lane's
// coefficients (K0 / K1 for the first half, K2 / K3 for the second), Go / Gp
// its own and its partner's gammas.
template <bool NORM, int RMODE>
__device__ __forceinline__ void norm_rotate_half(const float2 (&A)[4], const float2 (&B)[4],
                                                 float r, bool first, const float2 (&Kc)[4],
                                                 const float2 (&Kp)[4], const float2 (&Go)[4],
                                                 const float2 (&Gp)[4], float2 (&O)[4])
{
    const float2 r2 = f2(r, r);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float2 own = first ? A[q] : B[q];
        float2 par = first ? B[q] : A[q];
        if (NORM && RMODE == kRoundNormalized) {
            own = round2_bf16(__fmul2_rn(__fmul2_rn(own, r2), Go[q]));
            par = round2_bf16(__fmul2_rn(__fmul2_rn(par, r2), Gp[q]));
        }
        if (NORM && RMODE == kRoundEager) {
            own = round2_bf16(__fmul2_rn(round2_bf16(__fmul2_rn(own, r2)), Go[q]));
            par = round2_bf16(__fmul2_rn(round2_bf16(__fmul2_rn(par, r2)), Gp[q]));
        }
        float2 o;
        if (RMODE == kRoundEager)
            o = __fadd2_rn(__fmul2_rn(own, Kc[q]), __fmul2_rn(par, Kp[q]));
        else
            o = __ffma2_rn(par, Kp[q], __fmul2_rn(own, Kc[q]));
        if (NORM && RMODE == kRoundNone)
            o = __fmul2_rn(o, r2);
        O[q] = o;
    }
}

// Packs a row's couples back into the lane's bf16 vectors (one rounding).
template <int LAYOUT, int NS>
__device__ __forceinline__ void pack_row(const float2 (&A)[RowShape<LAYOUT, NS>::NQ],
                                         const float2 (&B)[RowShape<LAYOUT, NS>::NQ],
                                         const float2 (&T)[RowShape<LAYOUT, NS>::NTA][4],
                                         uint4 (&out)[NS])
{
    constexpr int NQ = RowShape<LAYOUT, NS>::NQ;
    constexpr int NT = RowShape<LAYOUT, NS>::NT;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        if (LAYOUT == PAIRED) {
            set_word(out[0], q, pack2(A[q].x, A[q].y));
            set_word(out[1], q, pack2(B[q].x, B[q].y));
        } else {
            set_word(out[q >> 1], 2 * (q & 1), pack2(A[q].x, B[q].x));
            set_word(out[q >> 1], 2 * (q & 1) + 1, pack2(A[q].y, B[q].y));
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            set_word(out[2 + t], i, pack2(T[t][i].x, T[t][i].y));
}

}  // namespace
}  // namespace qkr
