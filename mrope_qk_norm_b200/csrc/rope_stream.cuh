// rope_stream.cuh -- the streaming variant of the item-based rope kernel.
//
// Same arithmetic as rope_fast.cuh (per-head RMSNorm of Q and K, text-first
// concatenation, RoPE / mRoPE with packed fp32x2 math, one final rounding),
// with the row traffic decoupled from the register file:
//   * CTAs each owning a balanced range of a few joint tokens (4-8);
//   * every thread streams its own 16-byte row vectors into a shared-memory
//     ring S passes ahead with cp.async (LDGSTS, L2-only), so about
//     (S-1) x U x slots x 16 bytes per thread are in flight while it computes
//     the current pass -- in the plain item kernel the loads of one pass only
//     go out after the previous pass's math, and registers cap the depth;
//   * a thread reads back only vectors it copied itself, so a pass needs no
//     block barrier, only cp.async.wait_group on the thread's own groups;
//   * the (cos, sin) of all of the CTA's tokens are staged once in shared
//     memory at the start (sincosf of the fp32 position x inv_freq product,
//     or the fp32 table), while the first passes' rows are already in
//     flight.
// Invalid vectors (past the head dim, past the item's heads, a dead item) are
// zero-filled by the copy itself (source size 0), which keeps the sum of
// squares exact.
#pragma once

#include "rope_fast.cuh"

namespace qkr {

// Exported by rope_stream_paired.cu / rope_stream_vector.cu.
KernelFn pick_stream_paired(int lpr, int ns, int u, bool norm);
KernelFn pick_stream_vector(int lpr, int ns, int u, bool norm);

namespace {

// 16-byte copy global -> shared (shared-window address), zero-filled when
// !valid (source size 0), so sums of squares over dead vectors stay exact.
__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void *gmem_src, bool valid)
{
    const int src_size = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_dst),
                 "l"(gmem_src), "r"(src_size)
                 : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t smem_src)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_src)
                 : "memory");
    return v;
}
__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
// Wait until at most `pending` of this thread's most recent groups are in
// flight (the ring depth is a launch parameter; the instruction takes an
// immediate).  This waits on the thread's own copies, which always complete.
__device__ __forceinline__ void cp_async_wait(int pending)
{
    switch (pending) {
    case 0: asm volatile("cp.async.wait_group 0;\n" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;\n" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;\n" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 3;\n" ::: "memory"); break;
    }
}

// Shared-memory ring geometry: stage s, vector k = u * NS + slot, thread t
// at ((s * U * NS + k) * kThreads + t) * 16 bytes -- a warp's accesses to one
// vector index are 512 consecutive bytes (conflict-free 128-bit access).  A
// thread keeps the shared-window address of its stage-0 vector 0; a stage
// adds a compile-time stride, a vector a compile-time offset.
template <int U, int NS>
struct Ring {
    static constexpr uint32_t kVecStride = kThreads * 16;
    static constexpr uint32_t kStageStride = U * NS * kVecStride;
};

// Normalise, rotate and store the U rows of one work item from ring stage st.
template <int LAYOUT, int LPR, int NS, int U, bool NORM, int RMODE>
__device__ __forceinline__ void stream_rows(
    const RopeParams &p, const Item &m, uint32_t stage_addr, const int (&vidx)[NS],
    const float2 (&C)[RowShape<LAYOUT, NS>::NQ], const float2 (&Sn)[RowShape<LAYOUT, NS>::NQ],
    const float2 (&GA)[RowShape<LAYOUT, NS>::NQ], const float2 (&GB)[RowShape<LAYOUT, NS>::NQ],
    const float2 (&GT)[RowShape<LAYOUT, NS>::NTA][4])
{
    constexpr int NQ = RowShape<LAYOUT, NS>::NQ;
    constexpr int NTA = RowShape<LAYOUT, NS>::NTA;
    RotCoef<NQ, NORM && RMODE == kRoundNone> kc;
    make_coef(kc, C, Sn, GA, GB);
#pragma unroll
    for (int u = 0; u < U; ++u) {
        uint4 raw[NS];
#pragma unroll
        for (int k = 0; k < NS; ++k)
            raw[k] = lds128(stage_addr + (u * NS + k) * Ring<U, NS>::kVecStride);
        float2 A[NQ], B[NQ], TL[NTA][4];
        unpack_row<LAYOUT, NS>(raw, A, B, TL);
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
                    st_stream(m.dst + (int64_t)u * p.D + 8 * vidx[k], outv[k]);
        }
    }
}

template <int LAYOUT, int LPR, int NS, int U, bool NORM>
__global__ void __launch_bounds__(kThreads)
rope_stream_kernel(const __grid_constant__ RopeParams p)
{
    pdl_enter(p.independent);
    constexpr int NQ = RowShape<LAYOUT, NS>::NQ;
    constexpr int NTA = RowShape<LAYOUT, NS>::NTA;
    constexpr int G = kThreads / LPR;
    const int S = p.stages;
    const int rmode = p.round_norm;  // uniform: the paths below are warp-uniform

    extern __shared__ float4 smem[];
    uint4 *ring = reinterpret_cast<uint4 *>(smem);
    const int cs_ld = (p.pw + 3) & ~3;
    float *cosv = reinterpret_cast<float *>(ring + (size_t)S * U * NS * kThreads);
    float *sinv = cosv + p.tokens_per_cta * cs_ld;

    const int64_t tok0 = cta_first_token(p);
    const int ntok = cta_tokens(p);

    const int lane = threadIdx.x % LPR;
    const int grp = threadIdx.x / LPR;
    const int D = p.D;
    const int nvec = D >> 3;
    const int npv = p.rot >> 4;
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
    int qpair[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q)
        qpair[q] = LAYOUT == PAIRED ? 8 * lane + 2 * q : 4 * (lane + LPR * (q >> 1)) + 2 * (q & 1);

    const int nbq = (p.Hq + U - 1) / U;
    const int gpt = nbq + (p.Hk + U - 1) / U;
    const int items = ntok * gpt;
    const int passes = (items + G - 1) / G;  // uniform across the CTA

    // Copy this thread's vectors of pass `pass` into ring stage `pass % S`
    // (one commit group per pass, empty past the last pass).  Passes are
    // issued in order, so the stage is a counter that wraps at S.
    int dq, dr;
    divmod_small(G, gpt, p.gpt_recip, dq, dr);
    ItemCursor icur, ccur;  // the pass being copied in, the pass being computed
    icur.start(grp, gpt, p.gpt_recip);
    ccur = icur;
    const uint32_t ring_base = (uint32_t)__cvta_generic_to_shared(ring) + threadIdx.x * 16;
    int ist = 0, cst = 0;   // ring stage being issued into, being computed from
    // With a two-pass ring the item a pass computes is the one the previous
    // issue decoded: carry it instead of decoding it again.
    Item carried;
    auto issue = [&](int pass) {
        if (pass < passes) {
            const Item m = decode_item<U>(p, tok0, icur, ntok, nbq);
            carried = m;
            icur.advance(dq, dr, gpt);
            const uint32_t sa = ring_base + ist * Ring<U, NS>::kStageStride;
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int k = 0; k < NS; ++k) {
                    const bool ok = u < m.nh && vidx[k] >= 0;
                    const __nv_bfloat16 *src = ok ? m.src + u * m.hs + 8 * vidx[k] : m.src;
                    cp_async16(sa + (u * NS + k) * Ring<U, NS>::kVecStride, src, ok);
                }
        }
        ist = ist + 1 == S ? 0 : ist + 1;
        cp_async_commit();
    };

    for (int s = 0; s < S - 1; ++s)
        issue(s);
    stage_angles(p, tok0, ntok, cs_ld, cosv, sinv);
    __syncthreads();

    for (int pass = 0; pass < passes; ++pass) {
        Item m;
        if (S == 2) {
            m = carried;
        } else {
            m = decode_item<U>(p, tok0, ccur, ntok, nbq);
            ccur.advance(dq, dr, gpt);
        }
        issue(pass + S - 1);
        cp_async_wait(S - 1);
        const uint32_t stage_addr = ring_base + cst * Ring<U, NS>::kStageStride;
        cst = cst + 1 == S ? 0 : cst + 1;

        float2 C[NQ], Sn[NQ];
        {
            const float *cr = cosv + m.tt * cs_ld;
            const float *sr = sinv + m.tt * cs_ld;
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
        float2 GA[NQ], GB[NQ], GT[NTA][4];
        if (NORM) {
            const RopeStreamDev &Sd = m.s1 ? p.st[1] : p.st[0];
            const __nv_bfloat16 *gam = m.isk ? Sd.gk : Sd.gq;
            uint4 gv[NS];
#pragma unroll
            for (int k = 0; k < NS; ++k)
                gv[k] = vidx[k] >= 0 ? ld_reuse(gam + 8 * vidx[k]) : make_uint4(0, 0, 0, 0);
            unpack_row<LAYOUT, NS>(gv, GA, GB, GT);
        }

        if (rmode == kRoundEager)
            stream_rows<LAYOUT, LPR, NS, U, NORM, kRoundEager>(p, m, stage_addr, vidx, C, Sn, GA, GB,
                                                               GT);
        else if (rmode == kRoundNormalized)
            stream_rows<LAYOUT, LPR, NS, U, NORM, kRoundNormalized>(p, m, stage_addr, vidx, C, Sn,
                                                                    GA, GB, GT);
        else
            stream_rows<LAYOUT, LPR, NS, U, NORM, kRoundNone>(p, m, stage_addr, vidx, C, Sn, GA, GB,
                                                              GT);
    }
    cp_async_wait(0);  // nothing is left in flight (the trailing groups are empty)
    if (p.Hv > 0)
        copy_v_rows<NS, LPR, 2>(p, tok0, ntok, vidx);
    pdl_exit(p.independent);
}

template <int LAYOUT, int LPR, int NS, int U>
KernelFn pick_stream_norm(bool norm)
{
    return norm ? rope_stream_kernel<LAYOUT, LPR, NS, U, true>
                : rope_stream_kernel<LAYOUT, LPR, NS, U, false>;
}

template <int LAYOUT, int LPR, int NS>
KernelFn pick_stream_u(int u, bool norm)
{
    switch (u) {
    case 1: return pick_stream_norm<LAYOUT, LPR, NS, 1>(norm);
    case 2: return pick_stream_norm<LAYOUT, LPR, NS, 2>(norm);
    case 4: return pick_stream_norm<LAYOUT, LPR, NS, 4>(norm);
    default: return nullptr;
    }
}

template <int LAYOUT, int LPR>
KernelFn pick_stream_ns(int ns, int u, bool norm)
{
    if constexpr (LAYOUT == PAIRED) {
        switch (ns) {
        case 2: return pick_stream_u<LAYOUT, LPR, 2>(u, norm);
        case 3: return pick_stream_u<LAYOUT, LPR, 3>(u, norm);
        case 4: return pick_stream_u<LAYOUT, LPR, 4>(u, norm);
        default: return nullptr;
        }
    } else {
        switch (ns) {
        case 1: return pick_stream_u<LAYOUT, LPR, 1>(u, norm);
        case 2: return pick_stream_u<LAYOUT, LPR, 2>(u, norm);
        default: return nullptr;
        }
    }
}

template <int LAYOUT>
KernelFn pick_stream(int lpr, int ns, int u, bool norm)
{
    switch (lpr) {
    case 1: return pick_stream_ns<LAYOUT, 1>(ns, u, norm);
    case 2: return pick_stream_ns<LAYOUT, 2>(ns, u, norm);
    case 4: return pick_stream_ns<LAYOUT, 4>(ns, u, norm);
    case 8: return pick_stream_ns<LAYOUT, 8>(ns, u, norm);
    case 16: return pick_stream_ns<LAYOUT, 16>(ns, u, norm);
    default: return nullptr;
    }
}

}  // namespace
}  // namespace qkr
