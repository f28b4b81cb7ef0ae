// rope_fast.cuh -- the item-based per-head RMSNorm + RoPE / mRoPE kernel.
//
// One kernel template serves fused_qk_norm_rope (vllm-omni #7600: per-stream
// per-head RMSNorm of Q and K, text-first concatenation and RoPE in one
// launch) and mrope_apply (llama.cpp fork #286: the section a pair falls in
// picks the position row its angle comes from; a launch over part of the
// tokens indexes the full-length position rows from its first token).  Its
// instantiations are split over several translation units (rope_fast_*.cu) so
// they compile in parallel; each unit exports one picker.
//
// B200 mapping.  The op moves ~4 bytes per element and does a handful of
// flops on it, so it is HBM-bound only if the instruction stream stays lean:
//   * a CTA owns a balanced range of consecutive joint tokens and all of
//     their Q and K heads; the grid is sized to the device (for the
//     direct-angle kernels, one or two waves of resident CTAs whose token
//     count gives every lane group the same number of work items), so every
//     SM gets the same share of rows and no pass is left part empty;
//   * a work item is (token, Q or K, a block of U heads).  A group of LPR
//     lanes takes an item, loads the (cos, sin) of its pairs and the gamma of
//     its columns into registers once, and issues the 16-byte loads of all U
//     rows before any math (U * slots * 16 bytes in flight per lane);
//   * staged angles: each token's (cos, sin) is computed once (sincosf of
//     the fp32 position x inv_freq product) or read once from the table into
//     shared memory, and every head of the token reuses it.  Direct angles
//     (an fp32 table whose rows allow 16-byte reads of four pairs): every
//     item reads its token's row straight from the table (L1/L2 serve the
//     other heads), so the kernel has no staging prologue and no block
//     barrier, and a CTA's table and row loads are in flight together;
//   * the math runs on Blackwell's packed fp32x2 instructions (FFMA2 / FMUL2)
//     with each float2 holding the first members of two pairs (A) or the
//     second members (B): rotation is A' = A C - B S, B' = B C + A S for
//     NeoX and GPT-J alike, so no lane ever needs another lane's data;
//   * NeoX with rot_dim % 16 == 0 (PAIRED layout): a lane loads vector u of
//     the first rotary half and vector u + rot/16 of the second half;
//     GPT-J (VECTOR layout): pairs (2j, 2j+1) sit in one 32-bit word, and two
//     words make one (A, B) float2 couple; pairs past rot_dim take (1, 0), so
//     they pass through exactly with no branch;
//   * NeoX rows of head_dim 64 rotated whole, with staged angles (PAIRX
//     layout): a lane loads one vector of one rotary half and takes its
//     partner's vector from lane l ^ rot/16 by shuffle, then runs the PAIRED
//     arithmetic for its own half only, bit-identical to the PAIRED layout;
//   * the fp32 sum of squares is reduced with xor shuffles inside the group;
//     every loop trip count is uniform across a warp so the full-mask
//     shuffles are always complete.
// Addresses are 64-bit throughout (large storage offsets, vllm-omni #7600).
#pragma once

#include "rope_math.cuh"

namespace qkr {

using KernelFn = void (*)(RopeParams);

// Pickers exported by the instantiation units: layout and angle path (staged
// or direct) fixed by the unit; lanes per row, slots, heads per item and the
// norm flags chosen at run time.
KernelFn pick_fast_paired_staged(int lpr, int ns, int u, bool norm, int rmode);
KernelFn pick_fast_paired_direct(int lpr, int ns, int u, bool norm, int rmode);
KernelFn pick_fast_vector_staged(int lpr, int ns, int u, bool norm, int rmode);
KernelFn pick_fast_vector_direct(int lpr, int ns, int u, bool norm, int rmode);
KernelFn pick_fast_pairx_staged(int lpr, int ns, int u, bool norm, int rmode);

namespace {

constexpr int kThreads = 256;

// The CTA's range of joint tokens: CTA c owns tok_base tokens, plus one when
// c < tok_rem (tok_base = T / grid, tok_rem = T % grid, set by the launcher),
// so the ranges are balanced and contiguous.  T < 2^31 (checked by the
// launcher), so 32-bit arithmetic is exact -- the 64-bit division a
// c * T / grid split needs costs every thread ~100 instructions.
__device__ __forceinline__ int64_t cta_first_token(const RopeParams &p)
{
    const int c = (int)blockIdx.x;
    return (int64_t)(c * p.tok_base + min(c, p.tok_rem));
}
__device__ __forceinline__ int cta_tokens(const RopeParams &p)
{
    return p.tok_base + ((int)blockIdx.x < p.tok_rem ? 1 : 0);
}

// Stage (cos, sin) of `ntok` tokens into shared memory, SoA, row stride cs_ld.
// Columns [P, pw) get the identity rotation (1, 0).  Thread i takes cells
// i, i + kThreads, ... of the ntok x pw tile; its (token, column) advances by
// a fixed step instead of a division per cell.
__device__ __forceinline__ void stage_angles(const RopeParams &p, int64_t tok0, int ntok,
                                             int cs_ld, float *cosv, float *sinv)
{
    const int pw = p.pw;
    if (pw <= 0)
        return;
    const int dt = kThreads / pw, dj = kThreads - (kThreads / pw) * pw;
    int tt = (int)threadIdx.x / pw;
    int j = (int)threadIdx.x - tt * pw;
    while (tt < ntok) {
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
        tt += dt;
        j += dj;
        if (j >= pw) {
            j -= pw;
            ++tt;
        }
    }
}

// (cos, sin) of the four pairs j0 .. j0+3 (j0 % 4 == 0) of token n straight
// from the fp32 table, one 16-byte load each.  The launcher takes this path
// only when it is exact: 16-byte aligned rows (tab_vec4), P % 4 == 0 and
// section boundaries on multiples of 4 under a contiguous (or no) section
// map, so four pairs never straddle P or a plane change.  Pairs past P take
// the identity (1, 0).
__device__ __forceinline__ void table_quad(const RopeParams &p, int64_t n, int j0, float4 &c4,
                                           float4 &s4)
{
    if (j0 < p.P) {
        const int axis = section_axis(p.section_mode, p.sec, j0);
        const int64_t at = (int64_t)axis * p.plane_stride + (p.token_offset + n) * p.ld + j0;
        c4 = __ldg(reinterpret_cast<const float4 *>(p.cos + at));
        s4 = __ldg(reinterpret_cast<const float4 *>(p.sin + at));
    } else {
        c4 = make_float4(1.f, 1.f, 1.f, 1.f);
        s4 = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// One work item: U consecutive heads of one token's Q or K.
struct Item {
    const __nv_bfloat16 *src;  // first head's row
    __nv_bfloat16 *dst;        // first head's output row
    int64_t hs;                // source head stride
    int tt;                    // token within the CTA's tile
    int nh;                    // heads in this item (0: no work)
    bool isk;
    bool s1;                   // second stream
};

// n / d and n % d for 0 <= n <= 256 and d >= 1, with recip = floor(2^16 / d)
// from the host: (n * recip) >> 16 is the quotient or one short of it (the
// error of recip is under n / 2^16 < 1), and one correction step fixes it.
__device__ __forceinline__ void divmod_small(int n, int d, int recip, int &q, int &r)
{
    q = (n * recip) >> 16;
    r = n - q * d;
    if (r >= d) {
        r -= d;
        ++q;
    }
}

// Position of a lane group in the CTA's item sequence (item = tt * gpt + b),
// advanced by G items per pass without an integer division.
struct ItemCursor {
    int tt;  // token within the CTA's range
    int b;   // item within the token, [0, gpt)
    __device__ __forceinline__ void start(int item, int gpt, int recip)
    {
        divmod_small(item, gpt, recip, tt, b);
    }
    // dq = G / gpt, dr = G % gpt
    __device__ __forceinline__ void advance(int dq, int dr, int gpt)
    {
        tt += dq;
        b += dr;
        if (b >= gpt) {
            b -= gpt;
            ++tt;
        }
    }
};

template <int U>
__device__ __forceinline__ Item decode_item(const RopeParams &p, int64_t tok0,
                                            const ItemCursor &c, int ntok, int nbq)
{
    Item r;
    const bool live = c.tt < ntok;
    r.tt = live ? c.tt : 0;
    const int b = live ? c.b : 0;
    r.isk = b >= nbq;
    const int h0 = (r.isk ? b - nbq : b) * U;
    r.nh = live ? min(U, (r.isk ? p.Hk : p.Hq) - h0) : 0;
    const int64_t n = tok0 + r.tt;
    r.s1 = n >= p.split;
    const int64_t t = r.s1 ? n - p.split : n;
    const RopeStreamDev &S = r.s1 ? p.st[1] : p.st[0];
    const __nv_bfloat16 *base = r.isk ? S.k : S.q;
    const int64_t ts = r.isk ? S.k_ts : S.q_ts;
    r.hs = r.isk ? S.k_hs : S.q_hs;
    r.src = base + t * ts + (int64_t)h0 * r.hs;
    // K scatter (rope_set_rows): row n of K goes to output row k_rows[n]; a row
    // outside the output is not written and raises bit 4 of the status word
    int64_t orow = n;
    if (r.isk && p.k_rows && live) {
        orow = __ldg(reinterpret_cast<const long long *>(p.k_rows) + n);
        if (orow < 0 || orow >= p.k_out_rows) {
            atomicOr(p.status, 4u);
            r.nh = 0;
            orow = 0;
        }
    }
    r.dst = (r.isk ? p.k_out : p.q_out) + orow * (r.isk ? p.ko_ts : p.qo_ts) +
            (int64_t)h0 * p.D;
    return r;
}

// The 16-byte loads of an item's U rows (zero for absent heads and slots).
template <int U, int NS>
__device__ __forceinline__ void load_item_rows(const Item &m, const int (&vidx)[NS],
                                               uint4 (&raw)[U][NS])
{
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
        for (int k = 0; k < NS; ++k)
            raw[u][k] = (u < m.nh && vidx[k] >= 0) ? ld_stream(m.src + u * m.hs + 8 * vidx[k])
                                                   : make_uint4(0, 0, 0, 0);
}

// Joint Q/K/V: before its Q/K items a CTA copies the V rows of its tokens into
// v_out unchanged, VR rows per group at a time, with the lanes' own vector
// slots (which cover the whole head dim in both layouts).  No math and no
// shuffles, and its registers are free again before the Q/K loop, so that
// loop keeps its occupancy.  The table-path kernels keep four rows in flight:
// joint Q/K/V 512+4096 tokens x 24 heads 29.47 -> 28.26 us (GPT-J, 3 V rows
// per group: one round trip instead of two), 29.86 -> 29.53 us (NeoX).  The
// kernels with staged angles keep two: there the larger copy raised the
// register count of the small positions launches' kernel (56 -> 64) and made
// those launches 1-3% slower.
template <int NS, int LPR, int VR>
__device__ __forceinline__ void copy_v_rows(const RopeParams &p, int64_t tok0, int ntok,
                                            const int (&vidx)[NS])
{
    constexpr int G = kThreads / LPR;
    const int rows = ntok * p.Hv;
    for (int r0 = threadIdx.x / LPR; r0 < rows; r0 += VR * G) {
        uint4 raw[VR][NS];
        __nv_bfloat16 *dst[VR];
#pragma unroll
        for (int j = 0; j < VR; ++j) {
            const int r = r0 + j * G;
            const bool live = r < rows;
            const int tt = live ? r / p.Hv : 0;
            const int h = live ? r - tt * p.Hv : 0;
            const int64_t n = tok0 + tt;
            const bool s1 = n >= p.split;
            const int64_t t = s1 ? n - p.split : n;
            const RopeStreamDev &S = s1 ? p.st[1] : p.st[0];
            const __nv_bfloat16 *src = S.v + t * S.v_ts + (int64_t)h * S.v_hs;
            dst[j] = live ? p.v_out + n * p.vo_ts + (int64_t)h * p.D : nullptr;
#pragma unroll
            for (int k = 0; k < NS; ++k)
                raw[j][k] = (live && vidx[k] >= 0) ? ld_stream(src + 8 * vidx[k])
                                                   : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < VR; ++j)
#pragma unroll
            for (int k = 0; k < NS; ++k)
                if (dst[j] && vidx[k] >= 0)
                    st_stream(dst[j] + 8 * vidx[k], raw[j][k]);
    }
}

template <int LAYOUT, int LPR, int NS, int U, bool NORM, int RMODE, bool DIRECT>
__device__ __forceinline__ void rope_fast_body(const RopeParams &p)
{
    pdl_enter(p.independent);
    // Quads (couples of pairs) per lane: PAIRED lo/hi vectors hold 4, each
    // VECTOR slot holds 2.  Pass-through slots (PAIRED tail) are scaled only.
    // A PAIRX lane rebuilds the two PAIRED slots of its pairs (its own vector
    // and its partner's) and runs the PAIRED arithmetic on them.
    constexpr int ML = LAYOUT == PAIRX ? PAIRED : LAYOUT;
    constexpr int MNS = LAYOUT == PAIRX ? 2 : NS;
    constexpr int NQ = RowShape<ML, MNS>::NQ;
    constexpr int NTA = RowShape<ML, MNS>::NTA;
    constexpr int G = kThreads / LPR;

    extern __shared__ float4 smem[];
    const int cs_ld = (p.pw + 3) & ~3;
    float *cosv = reinterpret_cast<float *>(smem);
    float *sinv = cosv + p.tokens_per_cta * cs_ld;

    // Balanced ranges of at most tokens_per_cta consecutive joint tokens.
    const int64_t tok0 = cta_first_token(p);
    const int ntok = cta_tokens(p);

    const int lane = threadIdx.x % LPR;
    const int grp = threadIdx.x / LPR;
    const int D = p.D;
    const int nvec = D >> 3;
    const int npv = p.rot >> 4;
    // PAIRX: the lane's pairs are those of vector hl of the first half, and
    // its own vector is in the first half when `first`
    const int hl = LAYOUT == PAIRX ? (lane & (npv - 1)) : lane;
    const bool first = lane < npv;
    // vector index of each slot (-1: none)
    int vidx[NS];
#pragma unroll
    for (int k = 0; k < NS; ++k) {
        int v;
        if (LAYOUT == PAIRX)
            v = lane;
        else if (LAYOUT == PAIRED)
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
        qpair[q] = LAYOUT == PAIRED || LAYOUT == PAIRX ? 8 * hl + 2 * q
                                                        : 4 * (lane + LPR * (q >> 1)) + 2 * (q & 1);

    const int nbq = (p.Hq + U - 1) / U;
    const int gpt = nbq + (p.Hk + U - 1) / U;
    const int items = ntok * gpt;

    ItemCursor cur;
    cur.start(grp, gpt, p.gpt_recip);
    int dq, dr;
    divmod_small(G, gpt, p.gpt_recip, dq, dr);
    // Staged GPT-J rows: the first item's rows are in flight while the angles
    // are staged, so a CTA pays one memory round trip before its first
    // rotation, not two (1024 .. 2048 tokens x 4+4 or 16+16 heads, positions:
    // 3-19% faster).  NeoX rows keep the loads after the barrier: holding the
    // rows across the staging took the paired kernel from 80 to 100 registers
    // and ran 2-4% slower below 1024 tokens.
    constexpr bool kEarlyRows = !DIRECT && LAYOUT == VECTOR;
    Item m;
    uint4 raw[U][NS];
    if (kEarlyRows) {
        m = decode_item<U>(p, tok0, cur, ntok, nbq);
        load_item_rows<U, NS>(m, vidx, raw);
    }
    if (!DIRECT) {
        stage_angles(p, tok0, ntok, cs_ld, cosv, sinv);
        __syncthreads();
    }

    // joint Q/K/V: the CTA's V rows first (plain copies), then its Q/K items
    if (p.Hv > 0)
        copy_v_rows<NS, LPR, DIRECT ? 4 : 2>(p, tok0, ntok, vidx);

    for (int it0 = 0; it0 < items; it0 += G, cur.advance(dq, dr, gpt)) {  // uniform trips
        if (!kEarlyRows || it0 > 0) {
            m = decode_item<U>(p, tok0, cur, ntok, nbq);
            load_item_rows<U, NS>(m, vidx, raw);
        }

        // (cos, sin) of this lane's pairs for the item's token
        float2 C[NQ], Sn[NQ];
        {
            const bool have = LAYOUT == PAIRED ? vidx[0] >= 0 : true;
#pragma unroll
            for (int q = 0; q < NQ; q += 2) {
                const bool ok = m.nh > 0 && have &&
                                (LAYOUT == PAIRED || LAYOUT == PAIRX || vidx[q >> 1] >= 0);
                float4 c4 = make_float4(1.f, 1.f, 1.f, 1.f);
                float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (ok) {
                    if (DIRECT) {
                        table_quad(p, tok0 + m.tt, qpair[q], c4, s4);
                    } else {
                        c4 = *reinterpret_cast<const float4 *>(cosv + m.tt * cs_ld + qpair[q]);
                        s4 = *reinterpret_cast<const float4 *>(sinv + m.tt * cs_ld + qpair[q]);
                    }
                }
                C[q] = f2(c4.x, c4.y);
                C[q + 1] = f2(c4.z, c4.w);
                Sn[q] = f2(s4.x, s4.y);
                Sn[q + 1] = f2(s4.z, s4.w);
            }
        }
        // gamma of this lane's columns, in the same (A, B) arrangement
        float2 GA[NQ], GB[NQ], GT[NTA][4];
        if (NORM) {
            const RopeStreamDev &S = m.s1 ? p.st[1] : p.st[0];
            const __nv_bfloat16 *gam = m.isk ? S.gk : S.gq;
            if constexpr (LAYOUT == PAIRX) {
                const uint4 gv[2] = {ld_reuse(gam + 8 * hl), ld_reuse(gam + 8 * (hl + npv))};
                unpack_row<PAIRED, 2>(gv, GA, GB, GT);
            } else {
                uint4 gv[NS];
#pragma unroll
                for (int k = 0; k < NS; ++k)
                    gv[k] = vidx[k] >= 0 ? ld_reuse(gam + 8 * vidx[k]) : make_uint4(0, 0, 0, 0);
                unpack_row<LAYOUT, NS>(gv, GA, GB, GT);
            }
        }
        RotCoef<NQ, NORM && RMODE == kRoundNone> kc;
        make_coef(kc, C, Sn, GA, GB);

        if constexpr (LAYOUT == PAIRX) {
            // this lane's half: coefficients and gammas of its own and its
            // partner's members
            float2 Kc[NQ], Kp[NQ], Go[NQ], Gp[NQ];
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                Kc[q] = first ? kc.K0[q] : kc.K2[q];
                Kp[q] = first ? kc.K1[q] : kc.K3[q];
                Go[q] = first ? GA[q] : GB[q];
                Gp[q] = first ? GB[q] : GA[q];
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint4 own = raw[u][0];
                uint4 par;
                par.x = __shfl_xor_sync(0xffffffffu, own.x, npv);
                par.y = __shfl_xor_sync(0xffffffffu, own.y, npv);
                par.z = __shfl_xor_sync(0xffffffffu, own.z, npv);
                par.w = __shfl_xor_sync(0xffffffffu, own.w, npv);
                const uint4 pv[2] = {first ? own : par, first ? par : own};
                float2 A[NQ], B[NQ], TL[NTA][4];
                unpack_row<PAIRED, 2>(pv, A, B, TL);
                float r = 1.f;
                if (NORM) {
                    // the PAIRED lane's sum over both members, reduced over
                    // the rot/16 lanes of this half: the PAIRED order
                    float ss = row_sumsq<PAIRED, 2>(A, B, TL);
#pragma unroll
                    for (int off = LPR / 4; off > 0; off >>= 1)
                        ss += __shfl_xor_sync(0xffffffffu, ss, off);
                    r = rsqrtf(fmaf(ss, p.inv_D, p.eps));
                }
                float2 O[NQ];
                norm_rotate_half<NORM, RMODE>(A, B, r, first, Kc, Kp, Go, Gp, O);
                uint4 outv;
#pragma unroll
                for (int q = 0; q < NQ; ++q)
                    set_word(outv, q, pack2(O[q].x, O[q].y));
                if (u < m.nh)
                    st_stream(m.dst + (int64_t)u * D + 8 * lane, outv);
            }
        } else {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float2 A[NQ], B[NQ], TL[NTA][4];
            unpack_row<LAYOUT, NS>(raw[u], A, B, TL);
            float r = 1.f;
            if (NORM) {
                float ss = row_sumsq<LAYOUT, NS>(A, B, TL);
#pragma unroll
                for (int off = LPR / 2; off > 0; off >>= 1)
                    ss += __shfl_xor_sync(0xffffffffu, ss, off);
                r = rsqrtf(fmaf(ss, p.inv_D, p.eps));
            }
            norm_rotate<LAYOUT, NS, NORM, RMODE>(A, B, TL, r, kc, GA, GB, GT);
            uint4 outv[NS];
            pack_row<LAYOUT, NS>(A, B, TL, outv);
            if (u < m.nh) {
#pragma unroll
                for (int k = 0; k < NS; ++k)
                    if (vidx[k] >= 0)
                        st_stream(m.dst + (int64_t)u * D + 8 * vidx[k], outv[k]);
            }
        }
        }
    }
    pdl_exit(p.independent);
}

// The item kernel under three register policies, picked by shape, because
// the allocation decides how many CTAs share an SM and the compiler's own
// choice moves with small code changes:
//   * rope_fast_kernel_narrow, one 16-byte vector per lane (GPT-J rows of
//     up to 128 elements) without the norm, with the normalised-value
//     rounding, or at 6 heads per item: at least 4 CTAs per SM (64
//     registers, no spill; 5 for items of at most 2 heads or without the
//     norm).  Left to itself the compiler gave these 58-77 registers (76
//     at 6 heads with the norm: 3 CTAs per SM).  Items of at most 2 heads
//     with the norm stay with the compiler: bounded to 5 CTAs they ran 5%
//     slower (GPT-J, positions, 1024 tokens);
//   * rope_fast_kernel_wide, NeoX rows of three or more slots (ViT apply at
//     D=80, 4 heads per item, ~126 registers): at least 2 CTAs per SM.  A
//     139-register build of that shape ran at one CTA per SM, 28% slower;
//   * rope_fast_kernel, the rest: the compiler's own allocation.  On the
//     GPT-J headline shape (4 heads per item) that is 64 registers, 4 CTAs
//     per SM; a declared minimum of 4 CTAs gave 64 registers too but ran
//     0.7% slower, and a minimum of 2 let it take 88 (2 CTAs per SM).
template <int LAYOUT, int LPR, int NS, int U, bool NORM, int RMODE, bool DIRECT>
__global__ void __launch_bounds__(kThreads) rope_fast_kernel(const __grid_constant__ RopeParams p)
{
    rope_fast_body<LAYOUT, LPR, NS, U, NORM, RMODE, DIRECT>(p);
}
template <int LAYOUT, int LPR, int NS, int U, bool NORM, int RMODE, bool DIRECT>
__global__ void __launch_bounds__(kThreads, 2)
rope_fast_kernel_wide(const __grid_constant__ RopeParams p)
{
    rope_fast_body<LAYOUT, LPR, NS, U, NORM, RMODE, DIRECT>(p);
}

template <int LAYOUT, int LPR, int NS, int U, bool NORM, int RMODE, bool DIRECT>
__global__ void __launch_bounds__(kThreads, NORM && U > 2 ? 4 : 5)
rope_fast_kernel_narrow(const __grid_constant__ RopeParams p)
{
    rope_fast_body<LAYOUT, LPR, NS, U, NORM, RMODE, DIRECT>(p);
}

template <int LAYOUT, int LPR, int NS, int U, bool NORM, int RMODE, bool DIRECT>
constexpr KernelFn item_kernel()
{
    if constexpr (LAYOUT == PAIRED && NS >= 3)
        return rope_fast_kernel_wide<LAYOUT, LPR, NS, U, NORM, RMODE, DIRECT>;
    else if constexpr (LAYOUT == VECTOR && NS == 1 &&
                       (!NORM || RMODE == kRoundNormalized || U == 6))
        return rope_fast_kernel_narrow<LAYOUT, LPR, NS, U, NORM, RMODE, DIRECT>;
    else
        return rope_fast_kernel<LAYOUT, LPR, NS, U, NORM, RMODE, DIRECT>;
}

// ------------------------------------------------------------- pickers --

template <int LAYOUT, bool DIRECT, int LPR, int NS, int U>
KernelFn pick_flags(bool norm, int rmode)
{
    if (!norm)
        return item_kernel<LAYOUT, LPR, NS, U, false, kRoundNone, DIRECT>();
    switch (rmode) {
    case kRoundNone: return item_kernel<LAYOUT, LPR, NS, U, true, kRoundNone, DIRECT>();
    case kRoundNormalized: return item_kernel<LAYOUT, LPR, NS, U, true, kRoundNormalized, DIRECT>();
    case kRoundEager: return item_kernel<LAYOUT, LPR, NS, U, true, kRoundEager, DIRECT>();
    default: return nullptr;
    }
}

template <int LAYOUT, bool DIRECT, int LPR, int NS>
KernelFn pick_u(int u, bool norm, int rmode)
{
    switch (u) {
    case 1: return pick_flags<LAYOUT, DIRECT, LPR, NS, 1>(norm, rmode);
    case 2: return pick_flags<LAYOUT, DIRECT, LPR, NS, 2>(norm, rmode);
    case 3: return pick_flags<LAYOUT, DIRECT, LPR, NS, 3>(norm, rmode);
    case 4: return pick_flags<LAYOUT, DIRECT, LPR, NS, 4>(norm, rmode);
    case 6:
        // one-vector GPT-J rows of 128 elements with table angles read per item
        if constexpr (LAYOUT == VECTOR && DIRECT && LPR == 16 && NS == 1)
            return pick_flags<LAYOUT, DIRECT, LPR, NS, 6>(norm, rmode);
        else
            return nullptr;
    default: return nullptr;
    }
}

template <int LAYOUT, bool DIRECT, int LPR>
KernelFn pick_ns(int ns, int u, bool norm, int rmode)
{
    if constexpr (LAYOUT == PAIRX) {
        // head_dim 64 rotated whole: one vector per lane, 8 lanes per row
        if constexpr (LPR == 8 && !DIRECT)
            return ns == 1 ? pick_u<LAYOUT, DIRECT, LPR, 1>(u, norm, rmode) : nullptr;
        else
            return nullptr;
    } else if constexpr (LAYOUT == PAIRED) {
        // slots 0/1: the two rotary halves of the lane's pairs; 2, 3: pass-through tail
        switch (ns) {
        case 2: return pick_u<LAYOUT, DIRECT, LPR, 2>(u, norm, rmode);
        case 3: return pick_u<LAYOUT, DIRECT, LPR, 3>(u, norm, rmode);
        case 4: return pick_u<LAYOUT, DIRECT, LPR, 4>(u, norm, rmode);
        default: return nullptr;
        }
    } else {
        switch (ns) {
        case 1: return pick_u<LAYOUT, DIRECT, LPR, 1>(u, norm, rmode);
        case 2: return pick_u<LAYOUT, DIRECT, LPR, 2>(u, norm, rmode);
        default: return nullptr;
        }
    }
}

template <int LAYOUT, bool DIRECT>
KernelFn pick_fast(int lpr, int ns, int u, bool norm, int rmode)
{
    switch (lpr) {
    case 1: return pick_ns<LAYOUT, DIRECT, 1>(ns, u, norm, rmode);
    case 2: return pick_ns<LAYOUT, DIRECT, 2>(ns, u, norm, rmode);
    case 4: return pick_ns<LAYOUT, DIRECT, 4>(ns, u, norm, rmode);
    case 8: return pick_ns<LAYOUT, DIRECT, 8>(ns, u, norm, rmode);
    case 16: return pick_ns<LAYOUT, DIRECT, 16>(ns, u, norm, rmode);
    default: return nullptr;
    }
}

}  // namespace
}  // namespace qkr
