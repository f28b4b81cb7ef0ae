// rope_rows.cu -- per-head RMSNorm + RoPE / mRoPE over (token, head) rows.
//
// One kernel family serves fused_qk_norm_rope (vllm-omni #7600: per-stream
// per-head RMSNorm of Q and K, text-first concatenation and RoPE in one
// launch) and mrope_apply (llama.cpp fork #286: each rotated pair reads the
// position row its section selects; a chunk reads the whole positions buffer
// from a token offset).
//
// B200 mapping.  The op moves ~4 bytes per element and does a handful of
// flops on it, so it is HBM-bound only if the instruction stream stays lean;
// the fast kernel is built for that:
//   * a CTA owns `tokens_per_cta` consecutive joint tokens and all of their Q
//     and K heads.  It first stages each token's (cos, sin) in shared memory
//     (sincosf from int32 positions, once per token and pair, or one read of
//     the fp32 table row) -- every head of the token reuses them;
//   * a work item is (token, Q or K, a block of U heads).  A group of LPR
//     lanes takes an item, loads the (cos, sin) of its pairs and the gamma of
//     its columns into registers once, and issues the 16-byte loads of all U
//     rows before any math (U * slots * 16 bytes in flight per lane);
//   * the math runs on Blackwell's packed fp32x2 instructions (FFMA2 / FMUL2)
//     with each float2 holding the first members of two pairs (A) or the
//     second members (B): rotation is A' = A C - B S, B' = B C + A S for
//     NeoX and GPT-J alike, so no lane ever needs another lane's data;
//   * NeoX with rot_dim % 16 == 0 (PAIRED layout): a lane loads vector u of
//     the first rotary half and vector u + rot/16 of the second half;
//     GPT-J (VECTOR layout): pairs (2j, 2j+1) sit in one 32-bit word, and two
//     words make one (A, B) float2 couple; pairs past rot_dim read (1, 0)
//     from the staged table, so they pass through exactly with no branch;
//   * the fp32 sum of squares is reduced with xor shuffles inside the group;
//     every loop trip count is uniform across a warp so the full-mask
//     shuffles are always complete.
// NeoX with rot_dim % 16 != 0 (EXCHANGE layout) is served by a plainer kernel
// that passes the normalised row through shared memory to reach partners.
// Addresses are 64-bit throughout (large storage offsets, vllm-omni #7600).

#include <climits>

#include "qkr_internal.cuh"

namespace qkr {
namespace {

constexpr int kThreads = 256;

enum Layout { PAIRED = 0, VECTOR = 1, EXCHANGE = 2 };

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

// Stage (cos, sin) of `ntok` tokens into shared memory, SoA, row stride cs_ld.
// Columns [P, pw) get the identity rotation (1, 0).
__device__ __forceinline__ void stage_angles(const RopeParams &p, int64_t tok0, int ntok,
                                             int cs_ld, float *cosv, float *sinv)
{
    const int pw = p.pw;
    for (int idx = threadIdx.x; idx < ntok * pw; idx += kThreads) {
        const int tt = idx / pw;
        const int j = idx - tt * pw;
        float c = 1.f, s = 0.f;
        if (j < p.P) {
            const int64_t n = p.token_offset + tok0 + tt;
            const int axis = section_axis(p.section_mode, p.sec, j);
            if (p.angle_kind == QKR_ANGLE_POSITIONS) {
                const int32_t pos = __ldg(p.pos + (int64_t)axis * p.pos_rs + n);
                const float theta = __fmul_rn((float)pos, __ldg(p.inv_freq + j));
                sincosf(theta, &s, &c);
            } else {
                const int64_t at = (int64_t)axis * p.plane_stride + n * p.ld + j;
                c = __ldg(p.cos + at);
                s = __ldg(p.sin + at);
            }
        }
        cosv[tt * cs_ld + j] = c;
        sinv[tt * cs_ld + j] = s;
    }
}

// ============================================================ fast kernel ==

template <int LAYOUT, int LPR, int NS, int U, bool NORM, bool ROUND>
__global__ void __launch_bounds__(kThreads)
rope_fast_kernel(const __grid_constant__ RopeParams p)
{
    // Quads (couples of pairs) per lane: PAIRED lo/hi vectors hold 4, each
    // VECTOR slot holds 2.  Pass-through slots (PAIRED tail) are scaled only.
    constexpr int NQ = LAYOUT == PAIRED ? 4 : 2 * NS;
    constexpr int NT = LAYOUT == PAIRED ? NS - 2 : 0;
    constexpr int G = kThreads / LPR;

    extern __shared__ float4 smem[];
    const int cs_ld = (p.pw + 3) & ~3;
    float *cosv = reinterpret_cast<float *>(smem);
    float *sinv = cosv + p.tokens_per_cta * cs_ld;

    const int64_t tok0 = (int64_t)blockIdx.x * p.tokens_per_cta;
    const int ntok = (int)min((int64_t)p.tokens_per_cta, p.T - tok0);
    stage_angles(p, tok0, ntok, cs_ld, cosv, sinv);
    __syncthreads();

    const int lane = threadIdx.x % LPR;
    const int grp = threadIdx.x / LPR;
    const int D = p.D;
    const int nvec = D >> 3;
    const int npv = p.rot >> 4;
    // vector index of each slot (-1: none)
    int vidx[NS];
#pragma unroll
    for (int k = 0; k < NS; ++k) {
        int v;
        if (LAYOUT == PAIRED)
            v = k == 0 ? (lane < npv ? lane : -1)
              : k == 1 ? (lane < npv ? lane + npv : -1)
                       : 2 * npv + lane + LPR * (k - 2);
        else
            v = lane + LPR * k;
        vidx[k] = (v >= 0 && v < nvec) ? v : -1;
    }
    // first pair index of each quad
    int qpair[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q)
        qpair[q] = LAYOUT == PAIRED ? 8 * lane + 2 * q : 4 * (lane + LPR * (q >> 1)) + 2 * (q & 1);

    const int nbq = (p.Hq + U - 1) / U;
    const int gpt = nbq + (p.Hk + U - 1) / U;
    const int items = ntok * gpt;

    for (int it0 = 0; it0 < items; it0 += G) {  // uniform trip count across the CTA
        const int item = it0 + grp;
        const bool live = item < items;
        const int it = live ? item : 0;
        const int tt = it / gpt;
        const int b = it - tt * gpt;
        const bool isk = b >= nbq;
        const int h0 = (isk ? b - nbq : b) * U;
        const int nh = min(U, (isk ? p.Hk : p.Hq) - h0);
        const int64_t n = tok0 + tt;
        const bool s1 = n >= p.split;
        const int64_t t = s1 ? n - p.split : n;
        const RopeStreamDev &S0 = p.st[0];
        const RopeStreamDev &S1 = p.st[1];
        const __nv_bfloat16 *base = isk ? (s1 ? S1.k : S0.k) : (s1 ? S1.q : S0.q);
        const int64_t ts = isk ? (s1 ? S1.k_ts : S0.k_ts) : (s1 ? S1.q_ts : S0.q_ts);
        const int64_t hs = isk ? (s1 ? S1.k_hs : S0.k_hs) : (s1 ? S1.q_hs : S0.q_hs);
        const __nv_bfloat16 *src = base + t * ts + (int64_t)h0 * hs;
        __nv_bfloat16 *dst = (isk ? p.k_out : p.q_out) + n * (isk ? p.ko_ts : p.qo_ts) +
                             (int64_t)h0 * D;

        uint4 raw[U][NS];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int k = 0; k < NS; ++k)
                raw[u][k] = (live && u < nh && vidx[k] >= 0)
                                ? ld_stream(src + u * hs + 8 * vidx[k])
                                : make_uint4(0, 0, 0, 0);

        // (cos, sin) of this lane's pairs for the item's token
        float2 C[NQ], Sn[NQ];
        {
            const float *cr = cosv + tt * cs_ld;
            const float *sr = sinv + tt * cs_ld;
            const bool have = LAYOUT == PAIRED ? vidx[0] >= 0 : true;
#pragma unroll
            for (int q = 0; q < NQ; q += 2) {
                const bool ok = have && (LAYOUT == PAIRED || vidx[q >> 1] >= 0);
                const float4 c4 = ok ? *reinterpret_cast<const float4 *>(cr + qpair[q])
                                     : make_float4(1.f, 1.f, 1.f, 1.f);
                const float4 s4 = ok ? *reinterpret_cast<const float4 *>(sr + qpair[q])
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                C[q] = f2(c4.x, c4.y);
                C[q + 1] = f2(c4.z, c4.w);
                Sn[q] = f2(s4.x, s4.y);
                Sn[q + 1] = f2(s4.z, s4.w);
            }
        }
        // gamma of this lane's columns, in the same (A, B) arrangement
        float2 GA[NQ], GB[NQ], GT[NT > 0 ? NT : 1][4];
        if (NORM) {
            const __nv_bfloat16 *gam = isk ? (s1 ? S1.gk : S0.gk) : (s1 ? S1.gq : S0.gq);
            uint4 gv[NS];
#pragma unroll
            for (int k = 0; k < NS; ++k)
                gv[k] = vidx[k] >= 0 ? ld_reuse(gam + 8 * vidx[k]) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                if (LAYOUT == PAIRED) {
                    const uint32_t wa = word(gv[0], q), wb = word(gv[1], q);
                    GA[q] = f2(bf_lo(wa), bf_hi(wa));
                    GB[q] = f2(bf_lo(wb), bf_hi(wb));
                } else {
                    const uint32_t w0 = word(gv[q >> 1], 2 * (q & 1));
                    const uint32_t w1 = word(gv[q >> 1], 2 * (q & 1) + 1);
                    GA[q] = f2(bf_lo(w0), bf_lo(w1));
                    GB[q] = f2(bf_hi(w0), bf_hi(w1));
                }
            }
#pragma unroll
            for (int k = 0; k < NT; ++k)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t w = word(gv[2 + k], i);
                    GT[k][i] = f2(bf_lo(w), bf_hi(w));
                }
        }

#pragma unroll
        for (int u = 0; u < U; ++u) {
            float2 A[NQ], B[NQ], TL[NT > 0 ? NT : 1][4];
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                if (LAYOUT == PAIRED) {
                    const uint32_t wa = word(raw[u][0], q), wb = word(raw[u][1], q);
                    A[q] = f2(bf_lo(wa), bf_hi(wa));
                    B[q] = f2(bf_lo(wb), bf_hi(wb));
                } else {
                    const uint32_t w0 = word(raw[u][q >> 1], 2 * (q & 1));
                    const uint32_t w1 = word(raw[u][q >> 1], 2 * (q & 1) + 1);
                    A[q] = f2(bf_lo(w0), bf_lo(w1));
                    B[q] = f2(bf_hi(w0), bf_hi(w1));
                }
            }
#pragma unroll
            for (int k = 0; k < NT; ++k)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t w = word(raw[u][2 + k], i);
                    TL[k][i] = f2(bf_lo(w), bf_hi(w));
                }

            if (NORM) {
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
                        acc = __ffma2_rn(TL[k][i], TL[k][i], acc);
                float ss = acc.x + acc.y;
#pragma unroll
                for (int off = LPR / 2; off > 0; off >>= 1)
                    ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float r = rsqrtf(fmaf(ss, p.inv_D, p.eps));
                const float2 r2 = f2(r, r);
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                    A[q] = __fmul2_rn(__fmul2_rn(A[q], r2), GA[q]);
                    B[q] = __fmul2_rn(__fmul2_rn(B[q], r2), GB[q]);
                    if (ROUND) {
                        A[q] = round2_bf16(A[q]);
                        B[q] = round2_bf16(B[q]);
                    }
                }
#pragma unroll
                for (int k = 0; k < NT; ++k)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        TL[k][i] = __fmul2_rn(__fmul2_rn(TL[k][i], r2), GT[k][i]);
            }

            // rotate: A' = A C - B S, B' = B C + A S (packed over two pairs)
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const float2 bs = __fmul2_rn(B[q], Sn[q]);
                const float2 bc = __fmul2_rn(B[q], C[q]);
                const float2 a2 = __ffma2_rn(A[q], C[q], f2(-bs.x, -bs.y));
                const float2 b2 = __ffma2_rn(A[q], Sn[q], bc);
                A[q] = a2;
                B[q] = b2;
            }

            uint4 outv[NS];
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                if (LAYOUT == PAIRED) {
                    set_word(outv[0], q, pack2(A[q].x, A[q].y));
                    set_word(outv[1], q, pack2(B[q].x, B[q].y));
                } else {
                    set_word(outv[q >> 1], 2 * (q & 1), pack2(A[q].x, B[q].x));
                    set_word(outv[q >> 1], 2 * (q & 1) + 1, pack2(A[q].y, B[q].y));
                }
            }
#pragma unroll
            for (int k = 0; k < NT; ++k)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    set_word(outv[2 + k], i, pack2(TL[k][i].x, TL[k][i].y));

            if (live && u < nh) {
#pragma unroll
                for (int k = 0; k < NS; ++k)
                    if (vidx[k] >= 0)
                        st_stream(dst + (int64_t)u * D + 8 * vidx[k], outv[k]);
            }
        }
    }
}

// ======================================================== exchange kernel ==
// NeoX with rot_dim % 16 != 0: a row's pair partners can sit anywhere in the
// row, so the normalised row passes through a per-group shared buffer.

template <int LPR, int NS>
__global__ void __launch_bounds__(kThreads)
rope_exchange_kernel(const __grid_constant__ RopeParams p)
{
    constexpr int G = kThreads / LPR;
    extern __shared__ float4 smem[];
    const int cs_ld = (p.pw + 3) & ~3;
    float *cosv = reinterpret_cast<float *>(smem);
    float *sinv = cosv + p.tokens_per_cta * cs_ld;

    const int64_t tok0 = (int64_t)blockIdx.x * p.tokens_per_cta;
    const int ntok = (int)min((int64_t)p.tokens_per_cta, p.T - tok0);
    stage_angles(p, tok0, ntok, cs_ld, cosv, sinv);
    __syncthreads();

    const int lane = threadIdx.x % LPR;
    const int grp = threadIdx.x / LPR;
    const int D = p.D;
    const int nvec = D >> 3;
    const int rows = ntok * p.rows_per_token;
    float *xbuf = sinv + p.tokens_per_cta * cs_ld + grp * D;
    const int half = p.rot >> 1;

    int vidx[NS];
#pragma unroll
    for (int k = 0; k < NS; ++k) {
        const int v = lane + LPR * k;
        vidx[k] = v < nvec ? v : -1;
    }

    for (int r0 = 0; r0 < rows; r0 += G) {  // uniform trip count
        const int r = r0 + grp;
        const bool live = r < rows;
        const int rr = live ? r : 0;
        const int tt = rr / p.rows_per_token;
        const int h = rr - tt * p.rows_per_token;
        const int64_t n = tok0 + tt;
        const bool s1 = n >= p.split;
        const int64_t t = s1 ? n - p.split : n;
        const bool isk = h >= p.Hq;
        const int hh = isk ? h - p.Hq : h;
        const RopeStreamDev &S = s1 ? p.st[1] : p.st[0];
        const __nv_bfloat16 *src = (isk ? S.k : S.q) + t * (isk ? S.k_ts : S.q_ts) +
                                   (int64_t)hh * (isk ? S.k_hs : S.q_hs);
        const __nv_bfloat16 *gam = isk ? S.gk : S.gq;
        __nv_bfloat16 *dst = (isk ? p.k_out : p.q_out) + n * (isk ? p.ko_ts : p.qo_ts) +
                             (int64_t)hh * D;

        float x[NS][8];
#pragma unroll
        for (int k = 0; k < NS; ++k)
            unpack8((live && vidx[k] >= 0) ? ld_stream(src + 8 * vidx[k]) : make_uint4(0, 0, 0, 0),
                    x[k]);
        if (p.norm) {
            float ss = 0.f;
#pragma unroll
            for (int k = 0; k < NS; ++k)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    ss = fmaf(x[k][e], x[k][e], ss);
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1)
                ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float inv_rms = rsqrtf(fmaf(ss, p.inv_D, p.eps));
#pragma unroll
            for (int k = 0; k < NS; ++k) {
                if (vidx[k] < 0)
                    continue;
                float g[8];
                unpack8(ld_reuse(gam + 8 * vidx[k]), g);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    x[k][e] = (x[k][e] * inv_rms) * g[e];
                    if (p.round_norm)
                        x[k][e] = round_bf16(x[k][e]);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < NS; ++k)
            if (vidx[k] >= 0)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    xbuf[8 * vidx[k] + e] = x[k][e];
        __syncwarp();
        const float *cr = cosv + tt * cs_ld;
        const float *sr = sinv + tt * cs_ld;
#pragma unroll
        for (int k = 0; k < NS; ++k) {
            if (vidx[k] < 0)
                continue;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int el = 8 * vidx[k] + e;
                if (el < p.rot) {
                    const bool lo = el < half;
                    const int j = lo ? el : el - half;
                    const float other = xbuf[lo ? el + half : el - half];
                    x[k][e] = lo ? x[k][e] * cr[j] - other * sr[j]
                                 : x[k][e] * cr[j] + other * sr[j];
                }
            }
        }
        __syncwarp();
        if (live) {
#pragma unroll
            for (int k = 0; k < NS; ++k)
                if (vidx[k] >= 0)
                    st_stream(dst + 8 * vidx[k], pack8(x[k]));
        }
    }
}

// ================================================================== host ==

using KernelFn = void (*)(RopeParams);

template <int LAYOUT, int LPR, int NS, int U>
KernelFn pick_flags(bool norm, bool round)
{
    if (!norm)
        return rope_fast_kernel<LAYOUT, LPR, NS, U, false, false>;
    return round ? rope_fast_kernel<LAYOUT, LPR, NS, U, true, true>
                 : rope_fast_kernel<LAYOUT, LPR, NS, U, true, false>;
}

template <int LAYOUT, int LPR, int NS>
KernelFn pick_u(int u, bool norm, bool round)
{
    switch (u) {
    case 1: return pick_flags<LAYOUT, LPR, NS, 1>(norm, round);
    case 2: return pick_flags<LAYOUT, LPR, NS, 2>(norm, round);
    case 3: return pick_flags<LAYOUT, LPR, NS, 3>(norm, round);
    case 4: return pick_flags<LAYOUT, LPR, NS, 4>(norm, round);
    default: return nullptr;
    }
}

template <int LAYOUT, int LPR>
KernelFn pick_ns(int ns, int u, bool norm, bool round)
{
    if constexpr (LAYOUT == PAIRED) {
        // slots 0/1: the two rotary halves of the lane's pairs; 2, 3: pass-through tail
        switch (ns) {
        case 2: return pick_u<LAYOUT, LPR, 2>(u, norm, round);
        case 3: return pick_u<LAYOUT, LPR, 3>(u, norm, round);
        case 4: return pick_u<LAYOUT, LPR, 4>(u, norm, round);
        default: return nullptr;
        }
    } else if constexpr (LAYOUT == VECTOR) {
        switch (ns) {
        case 1: return pick_u<LAYOUT, LPR, 1>(u, norm, round);
        case 2: return pick_u<LAYOUT, LPR, 2>(u, norm, round);
        default: return nullptr;
        }
    } else {
        switch (ns) {
        case 1: return rope_exchange_kernel<LPR, 1>;
        case 2: return rope_exchange_kernel<LPR, 2>;
        default: return nullptr;
        }
    }
}

template <int LAYOUT>
KernelFn pick(int lpr, int ns, int u, bool norm, bool round)
{
    switch (lpr) {
    case 1: return pick_ns<LAYOUT, 1>(ns, u, norm, round);
    case 2: return pick_ns<LAYOUT, 2>(ns, u, norm, round);
    case 4: return pick_ns<LAYOUT, 4>(ns, u, norm, round);
    case 8: return pick_ns<LAYOUT, 8>(ns, u, norm, round);
    case 16: return pick_ns<LAYOUT, 16>(ns, u, norm, round);
    default: return nullptr;
    }
}

int g_force_pipe = 0;  // 0 automatic, 1 register kernel, 2 pipelined kernel
int g_force_u = 0;     // tuning override of heads per item (0: automatic)
int g_force_tt = 0;    // tuning override of tokens per CTA (0: automatic)

int pow2_ceil(int v)
{
    int p = 1;
    while (p < v)
        p <<= 1;
    return p;
}

}  // namespace

void set_rope_shape_override(int pipeline, int heads_per_item, int tokens_per_cta)
{
    g_force_pipe = pipeline;
    g_force_u = heads_per_item;
    g_force_tt = tokens_per_cta;
}

cudaError_t launch_rope_rows(const RopeParams &p_in, int pairing, cudaStream_t stream,
                             LaunchRecord *rec)
{
    RopeParams p = p_in;
    const int nvec = p.D / 8;
    int layout, lpr, ns;
    if (p.rot > 0 && pairing == QKR_PAIRING_NEOX && p.rot % 16 == 0 &&
        (nvec - p.rot / 8) <= 2 * pow2_ceil(p.rot / 16)) {
        layout = PAIRED;
        const int npv = p.rot / 16;
        lpr = pow2_ceil(npv);
        ns = 2 + (nvec - 2 * npv + lpr - 1) / lpr;
    } else {
        layout = (p.rot > 0 && pairing == QKR_PAIRING_NEOX) ? EXCHANGE : VECTOR;
        lpr = pow2_ceil((nvec + 1) / 2);
        if (lpr > 16)
            lpr = 16;
        ns = (nvec + lpr - 1) / lpr;
    }
    // The bulk-copy pipelined kernel (rope_tma.cu) is selected explicitly: at
    // these sizes a plain register kernel is within ~10% of a device-to-device
    // copy of the same bytes and the pipelined kernel is slower.
    if (layout != EXCHANGE && g_force_pipe == 2)
        return launch_rope_tma(p, layout == PAIRED, lpr, ns, g_force_tt, stream, rec);
    // staged (cos, sin) columns: GPT-J stages every pair of the head so pairs
    // past rot_dim rotate by the identity
    p.pw = layout == VECTOR ? p.D / 2 : p.P;
    const int cs_ld = (p.pw + 3) & ~3;
    const int groups = kThreads / lpr;

    // Heads per work item (U) and tokens per CTA.  A sweep on B200 over
    // U in 1..4 and tokens per CTA in {1, 2, 4, 8, 16} (joint 512+4096 x 24
    // heads, both pairings; mRoPE 8192 x (16+8) heads) put U = 2 with 4
    // tokens per CTA within 3% of the best shape in every case: two rows of
    // loads in flight per lane at 80 registers (three CTAs per SM), and grids
    // of ~1-2k CTAs that keep the last wave short.  Head-stationary mappings,
    // deeper per-lane prefetch and a bulk-copy pipeline measured no faster:
    // in steady state even a device-to-device copy of these ~100 MB runs at
    // ~5.5 TB/s, and this kernel is within ~10% of it.
    const int max_tt_smem = cs_ld > 0 ? 16384 / (8 * cs_ld) : 64;
    int best_u = layout == EXCHANGE ? 1 : 2;
    int best_tt = 4 < max_tt_smem ? 4 : max_tt_smem;
    if (g_force_u > 0 && layout != EXCHANGE)
        best_u = g_force_u;
    if (g_force_tt > 0)
        best_tt = g_force_tt < max_tt_smem ? g_force_tt : max_tt_smem;
    if (best_tt > p.T)
        best_tt = (int)p.T;
    p.tokens_per_cta = best_tt;

    size_t smem = (size_t)best_tt * cs_ld * 2 * sizeof(float);
    if (layout == EXCHANGE)
        smem += (size_t)groups * p.D * sizeof(float);
    smem = (smem + 15) & ~(size_t)15;

    const bool norm = p.norm != 0, round = p.round_norm != 0;
    KernelFn fn = layout == PAIRED ? pick<PAIRED>(lpr, ns, best_u, norm, round)
                : layout == VECTOR ? pick<VECTOR>(lpr, ns, best_u, norm, round)
                                   : pick<EXCHANGE>(lpr, ns, 1, norm, round);
    if (!fn)
        return cudaErrorInvalidConfiguration;
    const int64_t grid = (p.T + best_tt - 1) / best_tt;
    if (grid > INT_MAX)
        return cudaErrorInvalidConfiguration;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    fn<<<(unsigned)grid, kThreads, smem, stream>>>(p);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess && rec) {
        *rec = LaunchRecord();
        rec->kernel = layout == PAIRED   ? QKR_KERNEL_ROPE_PAIRED
                    : layout == VECTOR   ? QKR_KERNEL_ROPE_VECTOR
                                         : QKR_KERNEL_ROPE_EXCHANGE;
        rec->lanes_per_row = lpr;
        rec->slots = ns;
        rec->tokens_per_cta = best_tt;
        rec->heads_per_item = layout == EXCHANGE ? 1 : best_u;
        rec->cluster = 1;
        rec->block = kThreads;
        rec->grid = grid;
        rec->launches = 1;
    }
    return err;
}

}  // namespace qkr
