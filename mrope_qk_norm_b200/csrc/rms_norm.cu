// rms_norm.cu -- hidden-size RMSNorm with fused residual add.
//
// s = bf16(x + residual) is written back to residual; out = s * rsqrt(mean(s^2)
// + eps) * gamma with an fp32 sum of squares of the bf16-rounded s (vllm.cpp
// #185: the residual stream carries bf16 rounding; vLLM #26234: vectorised
// reads of the row for the variance).
//
// B200 mapping.  Each thread keeps VPT 16-byte vectors of the row in
// registers, so the row crosses HBM exactly once (read x and residual, write
// residual and out).  The occupancy problem of vllm.cpp #185 (one workgroup
// per row leaves the GPU idle when a decode step has one row) is solved with
// a thread-block cluster: when rows are few (up to 32), each row is split
// across a cluster of 4 or 8 CTAs, every CTA reduces its slice,
// the partial sums are exchanged through distributed shared memory (read by
// every CTA in rank order, so all CTAs get the same bit-identical total), and
// each CTA normalises its slice.  No global scratch, no atomics, no spin-wait
// on a flag: the cluster barrier's co-residency is guaranteed by the hardware.

#include <cooperative_groups.h>
#include <cuda_fp8.h>

#include <atomic>
#include <climits>

#include "qkr_internal.cuh"

namespace cg = cooperative_groups;

namespace qkr {
namespace {

constexpr int kMaxThreads = 1024;

// Sum over the block, identical in every thread; fixed order.
__device__ __forceinline__ float block_sum(float v, float *red)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, off);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = (blockDim.x + 31) >> 5;
    if (lane == 0)
        red[warp] = v;
    __syncthreads();
    float t = 0.f;
    for (int w = 0; w < nwarps; ++w)
        t += red[w];
    return t;
}

// One vector per thread (decode rows and rows up to 8192 wide): gamma is
// loaded with x and the residual, so the row's last memory round trip is not
// taken after the block reduction.  Wider per-thread slices load it after the
// reduction: 4 more registers per vector would cut the large-row kernels'
// resident CTAs.
template <int VPT>
constexpr bool kEarlyGamma = VPT == 1;

// Loads the slice [v0, v1) of a row (vector units), forms s = bf16(x + res),
// writes it back to residual and returns the fp32 sum of s^2 of this thread
// (and, with kEarlyGamma, the slice's gamma vectors in gv).  Without a
// residual (p.res == NULL, FP8 variant) s = x.
template <int VPT>
__device__ __forceinline__ float load_sum(const RmsParams &p, int64_t row, int v0, int v1,
                                          float (&s)[VPT][8], bool (&live)[VPT],
                                          uint4 (&gv)[VPT])
{
    const __nv_bfloat16 *xr = p.x + row * p.xs;
    const bool has_res = p.res != nullptr;
    __nv_bfloat16 *rr = has_res ? p.res + row * p.rs : nullptr;
    uint4 xv[VPT], rv[VPT];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int v = v0 + threadIdx.x + k * blockDim.x;
        live[k] = v < v1;
        xv[k] = live[k] ? ld_stream(xr + 8 * v) : make_uint4(0, 0, 0, 0);
        rv[k] = live[k] && has_res ? ld_stream(rr + 8 * v) : make_uint4(0, 0, 0, 0);
        if (kEarlyGamma<VPT>)
            gv[k] = live[k] ? ld_reuse(p.gamma + 8 * v) : make_uint4(0, 0, 0, 0);
    }
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        float a[8], b[8];
        unpack8(xv[k], a);
        unpack8(rv[k], b);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            s[k][e] = a[e] + b[e];
        const uint4 packed = pack8(s[k]);
        unpack8(packed, s[k]);  // the residual stream is bf16: normalise the rounded sum
#pragma unroll
        for (int e = 0; e < 8; ++e)
            ss = fmaf(s[k][e], s[k][e], ss);
        if (live[k] && has_res)
            st_stream(rr + 8 * (v0 + threadIdx.x + k * blockDim.x), packed);
    }
    return ss;
}

// out = s * inv_rms * gamma: bf16, or (FP8) the E4M3 code of out / scale,
// computed as out * fp32(1 / scale) (one multiply per element instead of a
// division), rounded to nearest even and saturated to +-448
// (cvt.rn.satfinite.e4m3x2.f32).
template <int VPT, bool FP8>
__device__ __forceinline__ void scale_store(const RmsParams &p, int64_t row, int v0,
                                            float inv_rms, float (&s)[VPT][8],
                                            const bool (&live)[VPT], const uint4 (&gv)[VPT],
                                            float scale)
{
    float inv_scale = 1.f;  // y / scale is taken as y * fp32(1 / scale)
    if (FP8)
        inv_scale = __frcp_rn(kEarlyGamma<VPT> ? scale : __ldg(p.scale));
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        if (!live[k])
            continue;
        const int v = v0 + threadIdx.x + k * blockDim.x;
        float g[8];
        unpack8(kEarlyGamma<VPT> ? gv[k] : ld_reuse(p.gamma + 8 * v), g);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            s[k][e] = (s[k][e] * inv_rms) * g[e];
        if (FP8) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 q = make_float2(s[k][2 * i] * inv_scale,
                                             s[k][2 * i + 1] * inv_scale);
                w[i] = (uint32_t)__nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
            }
            const uint2 codes = make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
            __stcs(reinterpret_cast<uint2 *>(p.out8 + row * p.os + 8 * v), codes);
        } else {
            st_stream(p.out + row * p.os + 8 * v, pack8(s[k]));
        }
    }
}

// One CTA per row.
template <int VPT, bool FP8>
__global__ void __launch_bounds__(kMaxThreads) rms_rows_kernel(const __grid_constant__ RmsParams p)
{
    pdl_wait();
    pdl_trigger();
    __shared__ float red[32];
    const int64_t row = blockIdx.x;
    const float scale = FP8 && kEarlyGamma<VPT> ? __ldg(p.scale) : 1.f;
    float s[VPT][8];
    bool live[VPT];
    uint4 gv[VPT];
    const float ss = load_sum<VPT>(p, row, 0, p.hidden >> 3, s, live, gv);
    const float total = block_sum(ss, red);
    const float inv_rms = rsqrtf(fmaf(total, p.inv_hidden, p.eps));
    scale_store<VPT, FP8>(p, row, 0, inv_rms, s, live, gv, scale);
}

// One cluster per row; CTA `rank` owns vectors [rank*per, (rank+1)*per).
template <int VPT, bool FP8>
__global__ void __launch_bounds__(kMaxThreads)
rms_cluster_kernel(const __grid_constant__ RmsParams p)
{
    pdl_wait();
    pdl_trigger();
    __shared__ float red[32];
    __shared__ float partial;
    cg::cluster_group cluster = cg::this_cluster();
    const int cs = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int64_t row = blockIdx.x / cs;
    const int nvec = p.hidden >> 3;
    const int per = (nvec + cs - 1) / cs;
    const int v0 = rank * per;
    const int v1 = min(v0 + per, nvec);

    const float scale = FP8 && kEarlyGamma<VPT> ? __ldg(p.scale) : 1.f;
    float s[VPT][8];
    bool live[VPT];
    uint4 gv[VPT];
    const float ss = load_sum<VPT>(p, row, v0, v1, s, live, gv);
    const float mine = block_sum(ss, red);
    if (threadIdx.x == 0)
        partial = mine;
    cluster.sync();  // every CTA's partial is visible cluster-wide
    float total = 0.f;
    for (int r = 0; r < cs; ++r)
        total += *cluster.map_shared_rank(&partial, r);
    cluster.barrier_arrive();  // done reading the other CTAs' shared memory
    const float inv_rms = rsqrtf(fmaf(total, p.inv_hidden, p.eps));
    scale_store<VPT, FP8>(p, row, v0, inv_rms, s, live, gv, scale);
    cluster.barrier_wait();    // no CTA leaves while its partial may still be read
}

using Fn = void (*)(RmsParams);

template <bool FP8>
Fn rows_fn(int vpt)
{
    switch (vpt) {
    case 1: return rms_rows_kernel<1, FP8>;
    case 2: return rms_rows_kernel<2, FP8>;
    case 4: return rms_rows_kernel<4, FP8>;
    case 8: return rms_rows_kernel<8, FP8>;
    default: return nullptr;
    }
}

template <bool FP8>
Fn cluster_fn(int vpt)
{
    switch (vpt) {
    case 1: return rms_cluster_kernel<1, FP8>;
    case 2: return rms_cluster_kernel<2, FP8>;
    case 4: return rms_cluster_kernel<4, FP8>;
    case 8: return rms_cluster_kernel<8, FP8>;
    default: return nullptr;
    }
}

std::atomic<int> g_force_cluster{0};  // tuning override of CTAs per row (0: automatic)
std::atomic<int> g_force_threads{0};  // tuning override of threads per CTA (0: automatic)

// Smallest power-of-two vectors-per-thread keeping the block at or under
// `target` threads (and never above 1024).
void shape(int vectors, int target, int &vpt, int &threads)
{
    vpt = 1;
    while (vpt < 8 && (vectors + vpt - 1) / vpt > target)
        vpt <<= 1;
    threads = (vectors + vpt - 1) / vpt;
    threads = ((threads + 31) / 32) * 32;
    if (threads > kMaxThreads)
        threads = kMaxThreads;
}

}  // namespace

void set_rms_cluster_override(int cluster, int threads)
{
    g_force_cluster = cluster;
    g_force_threads = threads;
}

cudaError_t launch_rms_norm_residual(const RmsParams &p, cudaStream_t stream, LaunchRecord *rec)
{
    const bool fp8 = p.out8 != nullptr;
    const int nvec = p.hidden >> 3;
    // CTAs per row and threads per CTA, from sweeps on B200 (R = 1 .. 4096,
    // hidden 2048 .. 65536, graph-replayed back-to-back launches):
    //   * one CTA per row whenever a row fits one CTA (hidden <= 8192): every
    //     vector of the row in flight at once beats a cluster split, whose
    //     launch and DSMEM exchange cost ~0.9 us (R = 1 x 2048: 1.28 us
    //     against 2.13 us split over 8 CTAs; R = 1 x 5120: 1.66 against 2.21);
    //   * wider rows at decode sizes split over a cluster: 8 CTAs up to 16
    //     rows, 4 up to 32 (R = 1 x 65536: 3.3 us against 11.3 us in one CTA);
    //   * width: one vector per thread for up to 128 rows (up to 1024
    //     threads), two per thread beyond (R = 1024 x 8192: 12.0 us at 512
    //     threads against 12.4 at 256 and 13.7 at 1024).
    // A cluster slice keeps at least 32 vectors per CTA.
    int cs = 1;
    if (nvec > 1024 && p.R <= 32)
        cs = p.R <= 16 ? 8 : 4;
    while (cs > 1 && nvec / cs < 32)
        cs >>= 1;
    if (g_force_cluster > 0 && nvec / g_force_cluster >= 1)
        cs = g_force_cluster;
    int vpt, threads;
    const int per = (nvec + cs - 1) / cs;
    int target = cs == 8 ? 512 : (p.R <= 128 ? 1024 : (per + 1) / 2);
    if (target > kMaxThreads)
        target = kMaxThreads;  // wider rows take more vectors per thread
    if (target < 32)
        target = 32;
    if (g_force_threads > 0)
        target = g_force_threads;
    shape(per, target, vpt, threads);
    if ((int64_t)threads * vpt < per)
        return cudaErrorInvalidConfiguration;
    const int64_t grid = p.R * cs;
    if (grid > INT_MAX)
        return cudaErrorInvalidConfiguration;

    cudaError_t err;
    if (cs == 1) {
        err = launch(fp8 ? rows_fn<true>(vpt) : rows_fn<false>(vpt), dim3((unsigned)grid),
                     dim3(threads), 0, stream, 1, p);
    } else {
        Fn fn = fp8 ? cluster_fn<true>(vpt) : cluster_fn<false>(vpt);
        if (cs > 8) {
            err = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (err != cudaSuccess)
                return err;
        }
        err = launch(fn, dim3((unsigned)grid), dim3(threads), 0, stream, cs, p);
    }
    if (err == cudaSuccess && rec) {
        *rec = LaunchRecord();
        rec->kernel = cs == 1 ? QKR_KERNEL_RMS_ROWS : QKR_KERNEL_RMS_CLUSTER;
        rec->slots = vpt;
        rec->cluster = cs;
        rec->block = threads;
        rec->grid = grid;
        rec->launches = 1;
    }
    return err;
}

}  // namespace qkr
