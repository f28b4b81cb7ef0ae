// vit_setup.cu -- ViT mRoPE cos/sin plane setup (vLLM mrope_vit_setup page:
// VitMropeSetup and _vit_mrope_setup_kernel) plus the two debug kernels that
// expose the section rule and the grid-to-position mapping to the tests.
//
// B200 mapping.  The setup writes 2 * 4 bytes per (token, section column),
// computing one sincosf per cell; it is latency- and launch-bound at these
// sizes (8 MB for 16k tokens).  A CTA covers kTokens tokens.  It first stages
// the grid metadata (cu_seqlens, grids) and inv_freq in shared memory with
// independent loads -- one memory round trip instead of the binary search's
// chain of dependent loads -- then one thread per token derives (t, h, w)
// into shared memory, and each thread keeps one column (axis, offset and
// inv_freq fixed in registers) while walking the tokens, consecutive threads
// on consecutive columns so each warp's stores are contiguous.

#include <climits>

#include "qkr_internal.cuh"

namespace qkr {
namespace {

constexpr int kThreads = 256;
constexpr int kTokens = 32;
constexpr int kSmemGrids = 512;  // grids whose metadata a CTA stages in shared memory
constexpr int kMaxVitPairs = 512;  // per-axis inv_freq lengths staged in shared memory

// (t, h, w) of token n (cu / grids in shared or global memory).  The grid is
// the g with cu[g] <= n < cu[g+1]
// (binary search over the nondecreasing boundaries; empty grids are never
// selected).  Inside a frame of h*w tokens, tokens come in m x m merge blocks
// in row-major block order, each block's patches in row-major order.
__device__ __forceinline__ void token_position(const int32_t *cu, const int32_t *grids, int G,
                                               int64_t n, int m, int &tp, int &hp, int &wp)
{
    int lo = 0, hi = G;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if ((int64_t)cu[mid + 1] <= n)
            lo = mid + 1;
        else
            hi = mid;
    }
    const int g = lo < G ? lo : G - 1;
    const int64_t local = n - (int64_t)cu[g];
    const int h = grids[3 * g + 1];
    const int w = grids[3 * g + 2];
    const int64_t frame = max((int64_t)h * w, (int64_t)1);
    if (frame <= 0xffffffffLL && local >= 0 && local <= 0xffffffffLL && m > 0) {
        // the usual case, in 32-bit unsigned arithmetic (a 64-bit division is
        // several times longer, and this chain is the CTA's critical path)
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

__global__ void __launch_bounds__(kThreads) vit_setup_kernel(const __grid_constant__ VitParams p)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int spos[3][kTokens];
    __shared__ int32_t scu[kSmemGrids + 1];
    __shared__ int32_t sgrid[3 * kSmemGrids];
    __shared__ float sinv[3][kMaxVitPairs];
    // Stage the grid metadata and inv_freq with independent loads (one DRAM
    // round trip) instead of the binary search's chain of dependent loads.
    const bool staged = p.G <= kSmemGrids;
    if (staged) {
        for (int i = threadIdx.x; i <= p.G; i += kThreads)
            scu[i] = __ldg(p.cu + i);
        for (int i = threadIdx.x; i < 3 * p.G; i += kThreads)
            sgrid[i] = __ldg(p.grids + i);
    }
    const bool inv_staged =
        p.half[0] <= kMaxVitPairs && p.half[1] <= kMaxVitPairs && p.half[2] <= kMaxVitPairs;
    if (inv_staged)
        for (int a = 0; a < 3; ++a)
            for (int i = threadIdx.x; i < p.half[a]; i += kThreads)
                sinv[a][i] = __ldg(p.inv[a] + i);
    __syncthreads();

    const int64_t n0 = (int64_t)blockIdx.x * kTokens;
    const int ntok = (int)min((int64_t)kTokens, p.N - n0);
    if (threadIdx.x < ntok) {
        int tp, hp, wp;
        token_position(staged ? scu : p.cu, staged ? sgrid : p.grids, p.G, n0 + threadIdx.x,
                       p.m, tp, hp, wp);
        spos[0][threadIdx.x] = tp;
        spos[1][threadIdx.x] = hp;
        spos[2][threadIdx.x] = wp;
    }
    __syncthreads();

    const int P = p.P;
    const int end_t = p.half[0], end_h = p.half[0] + p.half[1];
    if (P <= kThreads) {
        // A thread owns one column for the whole pass: its axis, section
        // offset and inv_freq are fixed, and it walks the CTA's tokens with
        // a stride of kThreads / P (consecutive threads on consecutive
        // columns of one token row, so each warp's stores are contiguous).
        const int tpp = kThreads / P;
        const int col = threadIdx.x % P;
        const int tsub = threadIdx.x / P;
        if (tsub < tpp) {
            const int axis = col < end_t ? 0 : (col < end_h ? 1 : 2);
            const int off = axis == 0 ? 0 : (axis == 1 ? end_t : end_h);
            const float f = inv_staged ? sinv[axis][col - off] : __ldg(p.inv[axis] + (col - off));
            const int64_t base = ((int64_t)axis * p.N + n0) * P + col;
#pragma unroll 4
            for (int tt = tsub; tt < ntok; tt += tpp) {
                const float theta = __fmul_rn((float)spos[axis][tt], f);
                float s, c;
                sincosf(theta, &s, &c);
                __stcs(p.cos_out + base + (int64_t)tt * P, c);
                __stcs(p.sin_out + base + (int64_t)tt * P, s);
            }
        }
    } else {
        for (int idx = threadIdx.x; idx < ntok * P; idx += kThreads) {
            const int tt = idx / P;
            const int col = idx - tt * P;
            const int axis = col < end_t ? 0 : (col < end_h ? 1 : 2);
            const int off = axis == 0 ? 0 : (axis == 1 ? end_t : end_h);
            const float f = inv_staged ? sinv[axis][col - off] : __ldg(p.inv[axis] + (col - off));
            const float theta = __fmul_rn((float)spos[axis][tt], f);
            float s, c;
            sincosf(theta, &s, &c);
            const int64_t at = ((int64_t)axis * p.N + n0 + tt) * P + col;
            __stcs(p.cos_out + at, c);
            __stcs(p.sin_out + at, s);
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

cudaError_t launch_vit_setup(const VitParams &p, cudaStream_t stream, LaunchRecord *rec)
{
    const int64_t grid = (p.N + kTokens - 1) / kTokens;
    if (grid > INT_MAX)
        return cudaErrorInvalidConfiguration;
    cudaError_t err = launch(vit_setup_kernel, dim3((unsigned)grid), dim3(kThreads), 0, stream,
                             1, p);
    if (err == cudaSuccess && rec) {
        *rec = LaunchRecord();
        rec->kernel = QKR_KERNEL_VIT_SETUP;
        rec->tokens_per_cta = kTokens;
        rec->block = kThreads;
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
