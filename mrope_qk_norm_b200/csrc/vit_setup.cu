// vit_setup.cu -- ViT mRoPE cos/sin plane setup (vLLM mrope_vit_setup page:
// VitMropeSetup and _vit_mrope_setup_kernel) plus the two debug kernels that
// expose the section rule and the grid-to-position mapping to the tests.
//
// B200 mapping.  The setup writes 2 * 4 bytes per (token, section column),
// computing one sincosf per cell; at these sizes (8 MB for 16k tokens) it is
// bound by latency (launch, the metadata loads, sincosf's dependent chain),
// not by bytes or issue.  So every warp works on its own, with no block
// barrier, and keeps many independent chains in flight: a warp owns 8
// consecutive tokens; lanes 0..7 derive one token's (t, h, w) each (the grid
// found by shuffles over a register copy of the grid boundaries when there
// are at most 32 grids) while the lane's inv_freq loads are in flight, the
// positions are broadcast by shuffle, and each lane owns two columns of
// every 64 (axis, section offset and inv_freq fixed for the pass), all eight
// tokens unrolled, so a warp's stores to a token row are contiguous.  CTAs of
// 8 warps (255 for 16268 tokens): on B200 that measured 4.43 us against
// 4.47 at 16 warps, 4.91 at 4, and 5.0-6.9 us with 4 or 16 tokens per warp.
#include <climits>

#include "qkr_internal.cuh"

namespace qkr {
namespace {

constexpr int kThreads = 256;     // debug kernels
constexpr int kVitWarps = 8;      // warps per setup CTA
constexpr int kVitTokPerWarp = 8; // tokens one warp writes
constexpr int kVitThreads = 32 * kVitWarps;
constexpr int kTokens = kVitWarps * kVitTokPerWarp;  // tokens per setup CTA

// a / d for a, d < 2^20 (d >= 1): a single-precision quotient estimate (the
// approximate divide is within 2 ulp, so the estimate is within 1 of a / d)
// truncated, then made exact by one integer correction step on the
// remainder.  Several times shorter in latency than the 32-bit integer
// division routine, and the positions sit on the setup's critical path.
__device__ __forceinline__ uint32_t udiv_small(uint32_t a, uint32_t d)
{
    uint32_t q = (uint32_t)__fdividef((float)a, (float)d);
    const int r = (int)(a - q * d);
    q = r < 0 ? q - 1 : (r >= (int)d ? q + 1 : q);
    return q;
}

// (t, h, w) of the token at `local` index inside a grid of [., h, w] with
// merge size m.  Inside a frame of h*w tokens, tokens come in m x m merge
// blocks in row-major block order, each block's patches in row-major order.
__device__ __forceinline__ void grid_position(int64_t local, int h, int w, int m, int &tp,
                                              int &hp, int &wp)
{
    const int64_t frame = max((int64_t)h * w, (int64_t)1);
    if (local >= 0 && local < (1 << 20) && frame < (1 << 20) && m > 0 && m < 1024) {
        // the usual case: every quotient by the short division above
        const uint32_t l32 = (uint32_t)local, f32 = (uint32_t)frame, mm = (uint32_t)(m * m);
        const uint32_t t32 = udiv_small(l32, f32);
        const uint32_t in_frame = l32 - t32 * f32;
        const uint32_t block = udiv_small(in_frame, mm);
        const uint32_t patch = in_frame - block * mm;
        const uint32_t bpr = (uint32_t)max(w / m, 1);
        const uint32_t brow = udiv_small(block, bpr);
        const uint32_t bcol = block - brow * bpr;
        const uint32_t prow = udiv_small(patch, (uint32_t)m);
        tp = (int)t32;
        hp = (int)(brow * (uint32_t)m + prow);
        wp = (int)(bcol * (uint32_t)m + (patch - prow * (uint32_t)m));
        return;
    }
    if (frame <= 0xffffffffLL && local >= 0 && local <= 0xffffffffLL && m > 0) {
        // 32-bit unsigned arithmetic (a 64-bit division is several times longer)
        const uint32_t l32 = (uint32_t)local, f32 = (uint32_t)frame, mm = (uint32_t)(m * m);
        const uint32_t t32 = l32 / f32;
        const uint32_t in_frame = l32 - t32 * f32;
        const uint32_t block = in_frame / mm;
        const uint32_t patch = in_frame - block * mm;
        const uint32_t bpr = (uint32_t)max(w / m, 1);
        const uint32_t brow = block / bpr;
        const uint32_t bcol = block - brow * bpr;
        tp = (int)t32;
        hp = (int)(brow * (uint32_t)m + patch / (uint32_t)m);
        wp = (int)(bcol * (uint32_t)m + patch % (uint32_t)m);
        return;
    }
    tp = (int)(local / frame);
    const int64_t in_frame = local - (int64_t)tp * frame;
    const int mm = m * m;
    const int64_t block = in_frame / mm;        // merge-block index in the frame
    const int patch = (int)(in_frame - block * mm);
    const int64_t blocks_per_row = max(w / m, 1);
    const int64_t brow = block / blocks_per_row;
    const int64_t bcol = block - brow * blocks_per_row;
    hp = (int)(brow * m + patch / m);
    wp = (int)(bcol * m + patch % m);
}

// (t, h, w) of token n: the grid is the g with cu[g] <= n < cu[g+1] (binary
// search over the nondecreasing boundaries; empty grids are never selected).
__device__ __forceinline__ void token_position(const int32_t *cu, const int32_t *grids, int G,
                                               int64_t n, int m, int &tp, int &hp, int &wp)
{
    int lo = 0, hi = G;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if ((int64_t)__ldg(cu + mid + 1) <= n)
            lo = mid + 1;
        else
            hi = mid;
    }
    const int g = lo < G ? lo : G - 1;
    grid_position(n - (int64_t)__ldg(cu + g), __ldg(grids + 3 * g + 1), __ldg(grids + 3 * g + 2),
                  m, tp, hp, wp);
}

// CS: columns per lane per pass of 32 * CS columns -- 2, or 1 when a row has
// at most 32 columns (two per lane would leave the second half dead).
template <int CS>
__global__ void __launch_bounds__(kVitThreads)
vit_setup_kernel(const __grid_constant__ VitParams p)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t n0 = ((int64_t)blockIdx.x * kVitWarps + warp) * kVitTokPerWarp;
    constexpr int cstep = 32 * CS;  // columns per pass
    if (n0 >= p.N)
        return;  // warp-uniform
    const int ntok = (int)min((int64_t)kVitTokPerWarp, p.N - n0);

    // This lane's columns of the first pass (all of them when P <= cstep):
    // their axis and inv_freq do not depend on the tokens, so the inv_freq
    // loads go out now, beside the grid metadata loads below, instead of
    // after the positions are known.
    const int P = p.P;
    const int end_t = p.half[0], end_h = p.half[0] + p.half[1];
    float f01[CS];
#pragma unroll
    for (int i = 0; i < CS; ++i) {
        const int col = 32 * i + lane;
        const int axis = col < end_t ? 0 : (col < end_h ? 1 : 2);
        const int off = axis == 0 ? 0 : (axis == 1 ? end_t : end_h);
        f01[i] = col < P ? __ldg(p.inv[axis] + (col - off)) : 0.f;
    }

    // Lane j < ntok derives the position of token n0 + j (other lanes repeat
    // the last token, so every lane runs the same code).
    const int64_t n = n0 + min(lane, ntok - 1);
    int tp, hp, wp;
    if (p.G <= 32) {
        // lane l holds grid l's boundaries and sizes: one load each, and the
        // grid of a token is the number of grids that end at or before it --
        // one ballot per token of the warp (the tokens are consecutive)
        const bool have = lane < p.G;
        const int32_t end_l = have ? __ldg(p.cu + lane + 1) : 0;
        const int32_t start_l = have ? __ldg(p.cu + lane) : 0;
        const int32_t h_l = have ? __ldg(p.grids + 3 * lane + 1) : 1;
        const int32_t w_l = have ? __ldg(p.grids + 3 * lane + 2) : 1;
        const int myj = min(lane, ntok - 1);
        int g = 0;
#pragma unroll
        for (int j = 0; j < kVitTokPerWarp; ++j) {
            const unsigned ends = __ballot_sync(0xffffffffu, have && (int64_t)end_l <= n0 + j);
            if (myj == j)
                g = __popc(ends);
        }
        g = min(g, p.G - 1);
        const int32_t start = __shfl_sync(0xffffffffu, start_l, g);
        const int32_t h = __shfl_sync(0xffffffffu, h_l, g);
        const int32_t w = __shfl_sync(0xffffffffu, w_l, g);
        grid_position(n - (int64_t)start, h, w, p.m, tp, hp, wp);
    } else {
        token_position(p.cu, p.grids, p.G, n, p.m, tp, hp, wp);
    }

    // Merge size 2 with h and w even (every grid then starts on a multiple
    // of 4 tokens): the warp's 8 tokens are two whole 2x2 merge blocks, token
    // 4b + 2i + k at (t_b, h_b + i, w_b + k) from its block's first patch.  A
    // column then takes at most 4 distinct angles over the 8 tokens (t: one
    // per block, h: h_b + {0, 1}, w: w_b + {0, 1}), so each lane computes 4
    // sincosf per column instead of 8 and picks per token.  The same
    // expression on the same position, so the values are identical.  The
    // warp checks the pattern on its own positions and otherwise takes the
    // general loop below.
    const int bt0 = __shfl_sync(0xffffffffu, tp, 0), bt1 = __shfl_sync(0xffffffffu, tp, 4);
    const int bh0 = __shfl_sync(0xffffffffu, hp, 0), bh1 = __shfl_sync(0xffffffffu, hp, 4);
    const int bw0 = __shfl_sync(0xffffffffu, wp, 0), bw1 = __shfl_sync(0xffffffffu, wp, 4);
    bool blocks = false;
    if (p.m == 2 && ntok == kVitTokPerWarp) {  // warp-uniform
        const int b = (lane >> 2) & 1;
        const bool ok = lane >= kVitTokPerWarp ||
                        (tp == (b ? bt1 : bt0) && hp == (b ? bh1 : bh0) + ((lane >> 1) & 1) &&
                         wp == (b ? bw1 : bw0) + (lane & 1));
        blocks = __all_sync(0xffffffffu, ok);
    }
    if (blocks) {
        for (int c0 = 0; c0 < P; c0 += cstep) {  // uniform trip count
            int axis[CS];
            bool live[CS];
            float *cdst[CS], *sdst[CS];
            float cv[CS][4], sv[CS][4];  // slot s = 2b + d: block b, offset d on h / w
#pragma unroll
            for (int i = 0; i < CS; ++i) {
                const int col = c0 + 32 * i + lane;
                live[i] = col < P;
                axis[i] = col < end_t ? 0 : (col < end_h ? 1 : 2);
                const int off = axis[i] == 0 ? 0 : (axis[i] == 1 ? end_t : end_h);
                const float f =
                    c0 == 0 ? f01[i] : (live[i] ? __ldg(p.inv[axis[i]] + (col - off)) : 0.f);
                cdst[i] = p.cos_out + ((int64_t)axis[i] * p.N + n0) * P + col;
                sdst[i] = p.sin_out + ((int64_t)axis[i] * p.N + n0) * P + col;
#pragma unroll
                for (int sl = 0; sl < 4; ++sl) {
                    const int d = sl & 1;
                    const int pos = axis[i] == 0   ? (sl < 2 ? bt0 : bt1)
                                    : axis[i] == 1 ? (sl < 2 ? bh0 : bh1) + d
                                                   : (sl < 2 ? bw0 : bw1) + d;
                    sincosf(__fmul_rn((float)pos, f), &sv[i][sl], &cv[i][sl]);
                }
            }
#pragma unroll
            for (int j = 0; j < kVitTokPerWarp; ++j) {
                const int st = 2 * (j >> 2), sh = st + ((j >> 1) & 1), sw = st + (j & 1);
#pragma unroll
                for (int i = 0; i < CS; ++i) {
                    // st, sh, sw are constants once unrolled: register picks
                    const float c = axis[i] == 0 ? cv[i][st] : (axis[i] == 1 ? cv[i][sh] : cv[i][sw]);
                    const float sn = axis[i] == 0 ? sv[i][st] : (axis[i] == 1 ? sv[i][sh] : sv[i][sw]);
                    if (live[i]) {
                        __stcs(cdst[i] + (int64_t)j * P, c);
                        __stcs(sdst[i] + (int64_t)j * P, sn);
                    }
                }
            }
        }
        return;
    }

    // General case.  CS columns per lane per pass, every token of the warp
    // unrolled: CS x kVitTokPerWarp independent sincosf per lane in flight,
    // since the kernel is bound by their dependent latency, not by bytes or
    // issue.
    for (int c0 = 0; c0 < P; c0 += cstep) {  // uniform trip count
        int axis[CS];
        bool live[CS];
        float f[CS];
        float *cdst[CS], *sdst[CS];
#pragma unroll
        for (int i = 0; i < CS; ++i) {
            const int col = c0 + 32 * i + lane;
            live[i] = col < P;
            axis[i] = col < end_t ? 0 : (col < end_h ? 1 : 2);
            const int off = axis[i] == 0 ? 0 : (axis[i] == 1 ? end_t : end_h);
            f[i] = c0 == 0 ? f01[i] : (live[i] ? __ldg(p.inv[axis[i]] + (col - off)) : 0.f);
            cdst[i] = p.cos_out + ((int64_t)axis[i] * p.N + n0) * P + col;
            sdst[i] = p.sin_out + ((int64_t)axis[i] * p.N + n0) * P + col;
        }
#pragma unroll
        for (int j = 0; j < kVitTokPerWarp; ++j) {
            if (j < ntok) {  // warp-uniform
                const int pt = __shfl_sync(0xffffffffu, tp, j);
                const int ph = __shfl_sync(0xffffffffu, hp, j);
                const int pw = __shfl_sync(0xffffffffu, wp, j);
#pragma unroll
                for (int i = 0; i < CS; ++i) {
                    const int pos = axis[i] == 0 ? pt : (axis[i] == 1 ? ph : pw);
                    const float theta = __fmul_rn((float)pos, f[i]);
                    float sv, cv;
                    sincosf(theta, &sv, &cv);
                    if (live[i]) {
                        __stcs(cdst[i] + (int64_t)j * P, cv);
                        __stcs(sdst[i] + (int64_t)j * P, sv);
                    }
                }
            }
        }
    }
}

__global__ void vit_positions_kernel(const __grid_constant__ VitParams p, int32_t *out)
{
    pdl_wait();
    pdl_trigger();
    const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= p.N)
        return;
    int tp, hp, wp;
    token_position(p.cu, p.grids, p.G, n, p.m, tp, hp, wp);
    out[n] = tp;
    out[p.N + n] = hp;
    out[2 * p.N + n] = wp;
}

struct SectionArgs {
    int mode;
    int sec[4];
    int P;
};

__global__ void section_map_kernel(const __grid_constant__ SectionArgs a, int8_t *out)
{
    pdl_wait();
    pdl_trigger();
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j < a.P)
        out[j] = (int8_t)section_axis(a.mode, a.sec, j);
}

}  // namespace

cudaError_t launch_vit_setup(const VitParams &p_in, cudaStream_t stream, LaunchRecord *rec)
{
    // Two columns per lane; one when a row has at most 32.  Splitting a
    // block of 8 tokens' 64 columns over two warps (twice the resident warps)
    // measured 4.17 us against 3.97 us: each warp then derives the positions.
    const VitParams &p = p_in;
    const int tokens = kTokens;
    const int64_t grid = (p.N + tokens - 1) / tokens;
    if (grid > INT_MAX)
        return cudaErrorInvalidConfiguration;
    cudaError_t err = p.P > 32 ? launch(vit_setup_kernel<2>, dim3((unsigned)grid),
                                        dim3(kVitThreads), 0, stream, 1, p)
                               : launch(vit_setup_kernel<1>, dim3((unsigned)grid),
                                        dim3(kVitThreads), 0, stream, 1, p);
    if (err == cudaSuccess && rec) {
        *rec = LaunchRecord();
        rec->kernel = QKR_KERNEL_VIT_SETUP;
        rec->tokens_per_cta = tokens;
        rec->block = kVitThreads;
        rec->grid = grid;
        rec->launches = 1;
    }
    return err;
}

cudaError_t launch_vit_positions(const VitParams &p, int32_t *pos_out, cudaStream_t stream,
                                 LaunchRecord *rec)
{
    const int64_t grid = (p.N + kThreads - 1) / kThreads;
    if (grid > INT_MAX)
        return cudaErrorInvalidConfiguration;
    cudaError_t err = launch(vit_positions_kernel, dim3((unsigned)grid), dim3(kThreads), 0,
                             stream, 1, p, pos_out);
    if (err == cudaSuccess && rec) {
        *rec = LaunchRecord();
        rec->kernel = QKR_KERNEL_VIT_POSITIONS;
        rec->block = kThreads;
        rec->grid = grid;
        rec->launches = 1;
    }
    return err;
}

cudaError_t launch_section_map(int mode, const int (&sec)[4], int P, int8_t *out,
                               cudaStream_t stream, LaunchRecord *rec)
{
    SectionArgs a;
    a.mode = mode;
    for (int i = 0; i < 4; ++i)
        a.sec[i] = sec[i];
    a.P = P;
    const int grid = (P + 127) / 128;
    cudaError_t err = launch(section_map_kernel, dim3(grid), dim3(128), 0, stream, 1, a, out);
    if (err == cudaSuccess && rec) {
        *rec = LaunchRecord();
        rec->kernel = QKR_KERNEL_SECTION_MAP;
        rec->block = 128;
        rec->grid = grid;
        rec->launches = 1;
    }
    return err;
}

}  // namespace qkr
