// rope_rows.cu -- per-head RMSNorm + RoPE / mRoPE over (token, head) rows.
//
// One kernel serves fused_qk_norm_rope (vllm-omni #7600: per-stream per-head
// RMSNorm of Q and K, text-first concatenation and RoPE in one launch) and
// mrope_apply (llama.cpp fork #286: each rotated pair reads the position row
// its section selects; a chunk reads the whole positions buffer from a token
// offset).
//
// B200 mapping.  The op is HBM-bound (a few flops per byte), so the kernel
// is built around 16-byte coalesced streaming loads/stores and enough bytes
// in flight per SM:
//   * a CTA owns `tokens_per_cta` consecutive joint tokens and all of their
//     Q and K heads; it first writes the tokens' (cos, sin) for every pair
//     into shared memory (computed once per token with sincosf from int32
//     positions, or read once from fp32 tables) and every head row of those
//     tokens reuses them;
//   * a head row is owned by a group of LPR lanes (LPR a power of two); each
//     lane holds NS 16-byte vectors of the row in registers, the fp32 sum of
//     squares is reduced with xor shuffles inside the group;
//   * each group issues the loads of U rows before any math, so U*NS*16
//     bytes per lane are in flight;
//   * NeoX with rot_dim % 16 == 0 uses the PAIRED layout: a lane loads vector
//     u of the first half AND vector u + rot/16 of the second half, so both
//     members of each of its 8 pairs are in its own registers;
//   * GPT-J pairs (2j, 2j+1) never leave a 16-byte vector (VECTOR layout);
//   * NeoX with rot_dim % 16 != 0 (EXCHANGE layout) passes the normalised
//     row through a per-group shared-memory buffer to reach partners.
// Addresses are 64-bit throughout (large storage offsets, vllm-omni #7600).

#include <climits>

#include "qkr_internal.cuh"

namespace qkr {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsInFlight = 2;  // U: rows per group whose loads are issued together

enum Layout { PAIRED = 0, VECTOR = 1, EXCHANGE = 2 };

// Vector index (in units of 8 elements) held by `lane` in `slot`, or -1.
template <int LAYOUT, int LPR>
__device__ __forceinline__ int vec_index(int slot, int lane, int nvec, int npv)
{
    if (LAYOUT == PAIRED) {
        if (slot == 0)
            return lane < npv ? lane : -1;
        if (slot == 1)
            return lane < npv ? lane + npv : -1;
        const int v = 2 * npv + lane + LPR * (slot - 2);
        return v < nvec ? v : -1;
    }
    const int v = lane + LPR * slot;
    return v < nvec ? v : -1;
}

template <int LAYOUT, int LPR, int NS>
__global__ void __launch_bounds__(kThreads)
rope_rows_kernel(const __grid_constant__ RopeParams p)
{
    extern __shared__ float4 smem[];
    float2 *cs = reinterpret_cast<float2 *>(smem);  // [tokens_per_cta][cs_ld] (cos, sin)

    const int64_t tok0 = (int64_t)blockIdx.x * p.tokens_per_cta;
    const int ntok = (int)min((int64_t)p.tokens_per_cta, p.T - tok0);
    const int P = p.P;
    const int cs_ld = (P + 7) & ~7;  // padded so 16-byte shared loads stay aligned

    // ---- angles of this CTA's tokens, once per token ----------------------
    for (int idx = threadIdx.x; idx < ntok * P; idx += kThreads) {
        const int tt = idx / P;
        const int j = idx - tt * P;
        const int64_t n = p.token_offset + tok0 + tt;
        const int axis = section_axis(p.section_mode, p.sec, j);
        float c, s;
        if (p.angle_kind == QKR_ANGLE_POSITIONS) {
            const int32_t pos = __ldg(p.pos + (int64_t)axis * p.pos_rs + n);
            const float theta = __fmul_rn((float)pos, __ldg(p.inv_freq + j));
            sincosf(theta, &s, &c);
        } else {
            const int64_t at = (int64_t)axis * p.plane_stride + n * p.ld + j;
            c = __ldg(p.cos + at);
            s = __ldg(p.sin + at);
        }
        cs[tt * cs_ld + j] = make_float2(c, s);
    }
    __syncthreads();

    // ---- head rows ----------------------------------------------------------
    constexpr int G = kThreads / LPR;  // row groups per CTA
    constexpr int U = kRowsInFlight;
    const int lane = threadIdx.x % LPR;
    const int grp = threadIdx.x / LPR;
    const int D = p.D;
    const int nvec = D >> 3;
    const int npv = p.rot >> 4;  // PAIRED: vectors per half of the rotary dims
    const int rows = ntok * p.rows_per_token;
    float *xbuf = reinterpret_cast<float *>(cs + p.tokens_per_cta * cs_ld) + grp * D;  // EXCHANGE

    int vidx[NS];
#pragma unroll
    for (int k = 0; k < NS; ++k)
        vidx[k] = vec_index<LAYOUT, LPR>(k, lane, nvec, npv);

    for (int base = 0; base < rows; base += G * U) {
        uint4 raw[U][NS];
        __nv_bfloat16 *dst[U];
        const __nv_bfloat16 *gam[U];
        int trow[U];
        bool live[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = base + grp + u * G;
            live[u] = r < rows;
            const int rr = live[u] ? r : 0;
            const int tt = rr / p.rows_per_token;
            const int h = rr - tt * p.rows_per_token;
            const int64_t n = tok0 + tt;
            const bool s1 = n >= p.split;
            const int64_t t = s1 ? n - p.split : n;
            const bool isk = h >= p.Hq;
            const int hh = isk ? h - p.Hq : h;
            const __nv_bfloat16 *src;
            if (isk) {
                src = (s1 ? p.st[1].k : p.st[0].k) + t * (s1 ? p.st[1].k_ts : p.st[0].k_ts) +
                      (int64_t)hh * (s1 ? p.st[1].k_hs : p.st[0].k_hs);
                gam[u] = s1 ? p.st[1].gk : p.st[0].gk;
                dst[u] = p.k_out + n * p.ko_ts + (int64_t)hh * D;
            } else {
                src = (s1 ? p.st[1].q : p.st[0].q) + t * (s1 ? p.st[1].q_ts : p.st[0].q_ts) +
                      (int64_t)hh * (s1 ? p.st[1].q_hs : p.st[0].q_hs);
                gam[u] = s1 ? p.st[1].gq : p.st[0].gq;
                dst[u] = p.q_out + n * p.qo_ts + (int64_t)hh * D;
            }
            trow[u] = tt;
#pragma unroll
            for (int k = 0; k < NS; ++k)
                raw[u][k] = (live[u] && vidx[k] >= 0) ? ld_stream(src + 8 * vidx[k])
                                                      : make_uint4(0, 0, 0, 0);
        }

#pragma unroll
        for (int u = 0; u < U; ++u) {
            float x[NS][8];
#pragma unroll
            for (int k = 0; k < NS; ++k)
                unpack8(raw[u][k], x[k]);

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
                    unpack8(ld_reuse(gam[u] + 8 * vidx[k]), g);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        x[k][e] = (x[k][e] * inv_rms) * g[e];
                        if (p.round_norm)
                            x[k][e] = round_bf16(x[k][e]);
                    }
                }
            }

            const float2 *csr = cs + trow[u] * cs_ld;
            if (LAYOUT == PAIRED) {
                if (vidx[0] >= 0) {
                    const float4 *c4 = reinterpret_cast<const float4 *>(csr + 8 * lane);
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float4 w = c4[e2];  // (cos, sin) of pairs 2*e2 and 2*e2+1
                        const float cv[2] = {w.x, w.z}, sv[2] = {w.y, w.w};
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            const int e = 2 * e2 + h2;
                            const float a = x[0][e], b = x[1][e];
                            x[0][e] = a * cv[h2] - b * sv[h2];
                            x[1][e] = b * cv[h2] + a * sv[h2];
                        }
                    }
                }
            } else if (LAYOUT == VECTOR) {
#pragma unroll
                for (int k = 0; k < NS; ++k) {
                    const int v = vidx[k];
                    if (v < 0 || 8 * v >= p.rot)
                        continue;
                    const float4 *c4 = reinterpret_cast<const float4 *>(csr + 4 * v);
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const float4 w = c4[e2];  // pairs 4v + 2*e2, 4v + 2*e2 + 1
                        const float cv[2] = {w.x, w.z}, sv[2] = {w.y, w.w};
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            const int e = 4 * e2 + 2 * h2;
                            if (8 * v + e < p.rot) {
                                const float a = x[k][e], b = x[k][e + 1];
                                x[k][e] = a * cv[h2] - b * sv[h2];
                                x[k][e + 1] = b * cv[h2] + a * sv[h2];
                            }
                        }
                    }
                }
            } else {  // EXCHANGE: NeoX partners through shared memory
#pragma unroll
                for (int k = 0; k < NS; ++k)
                    if (vidx[k] >= 0)
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            xbuf[8 * vidx[k] + e] = x[k][e];
                __syncwarp();
                const int half = p.rot >> 1;
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
                            const float2 w = csr[j];
                            x[k][e] = lo ? x[k][e] * w.x - other * w.y
                                         : x[k][e] * w.x + other * w.y;
                        }
                    }
                }
                __syncwarp();
            }

            if (live[u]) {
#pragma unroll
                for (int k = 0; k < NS; ++k)
                    if (vidx[k] >= 0)
                        st_stream(dst[u] + 8 * vidx[k], pack8(x[k]));
            }
        }
    }
}

using KernelFn = void (*)(RopeParams);

template <int LAYOUT, int LPR>
KernelFn pick_ns(int ns)
{
    if constexpr (LAYOUT == PAIRED) {
        // slots 0/1: the two halves of the lane's pairs; 2, 3: pass-through tail
        switch (ns) {
        case 2: return rope_rows_kernel<LAYOUT, LPR, 2>;
        case 3: return rope_rows_kernel<LAYOUT, LPR, 3>;
        case 4: return rope_rows_kernel<LAYOUT, LPR, 4>;
        default: return nullptr;
        }
    } else {
        switch (ns) {
        case 1: return rope_rows_kernel<LAYOUT, LPR, 1>;
        case 2: return rope_rows_kernel<LAYOUT, LPR, 2>;
        default: return nullptr;
        }
    }
}

template <int LAYOUT>
KernelFn pick(int lpr, int ns)
{
    switch (lpr) {
    case 1: return pick_ns<LAYOUT, 1>(ns);
    case 2: return pick_ns<LAYOUT, 2>(ns);
    case 4: return pick_ns<LAYOUT, 4>(ns);
    case 8: return pick_ns<LAYOUT, 8>(ns);
    case 16: return pick_ns<LAYOUT, 16>(ns);
    default: return nullptr;
    }
}

int pow2_ceil(int v)
{
    int p = 1;
    while (p < v)
        p <<= 1;
    return p;
}

}  // namespace

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
        const int ntail = nvec - 2 * npv;
        ns = 2 + (ntail + lpr - 1) / lpr;
    } else {
        layout = (p.rot > 0 && pairing == QKR_PAIRING_NEOX) ? EXCHANGE : VECTOR;
        lpr = pow2_ceil((nvec + 1) / 2);
        if (lpr > 16)
            lpr = 16;
        ns = (nvec + lpr - 1) / lpr;
    }
    const int groups = kThreads / lpr;
    const int rows_per_pass = groups * kRowsInFlight;

    // Tokens per CTA: the count (up to 16) whose rows fill whole passes best,
    // bounded so the (cos, sin) tile stays small.
    const int rpt = p.rows_per_token;
    const int cs_ld = (p.P + 7) & ~7;
    const int max_tt_smem = cs_ld > 0 ? 24576 / (8 * cs_ld) : 64;
    int best_tt = 1;
    double best_util = -1.0;
    for (int tt = 1; tt <= 16 && tt <= max_tt_smem; ++tt) {
        const long rows = (long)tt * rpt;
        const long passes = (rows + rows_per_pass - 1) / rows_per_pass;
        const double util = (double)rows / (double)(passes * rows_per_pass);
        if (util > best_util + 0.01) {
            best_util = util;
            best_tt = tt;
        }
    }
    if (best_tt > p.T)
        best_tt = (int)p.T;
    p.tokens_per_cta = best_tt;

    size_t smem = (size_t)best_tt * cs_ld * sizeof(float2);
    if (layout == EXCHANGE)
        smem += (size_t)groups * p.D * sizeof(float);
    smem = (smem + 15) & ~(size_t)15;

    KernelFn fn = layout == PAIRED ? pick<PAIRED>(lpr, ns)
                : layout == VECTOR ? pick<VECTOR>(lpr, ns)
                                   : pick<EXCHANGE>(lpr, ns);
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
        rec->kernel = layout == PAIRED   ? QKR_KERNEL_ROPE_PAIRED
                    : layout == VECTOR   ? QKR_KERNEL_ROPE_VECTOR
                                         : QKR_KERNEL_ROPE_EXCHANGE;
        rec->lanes_per_row = lpr;
        rec->slots = ns;
        rec->tokens_per_cta = best_tt;
        rec->cluster = 1;
        rec->block = kThreads;
        rec->grid = grid;
        rec->launches = 1;
    }
    return err;
}

}  // namespace qkr
