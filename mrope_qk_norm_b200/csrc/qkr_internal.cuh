// qkr_internal.cuh -- device helpers and launch descriptors shared by the
// CUDA translation units of the library (not part of the public ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/qkr.h"

namespace qkr {

// ---------------------------------------------------------------- bf16 x8 --
// A 16-byte vector holds 8 consecutive bf16 elements; element 2i sits in the
// low half of word i.

__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8])
{
    return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]),
                      pack2(f[6], f[7]));
}

__device__ __forceinline__ float round_bf16(float x)
{
    return __bfloat162float(__float2bfloat16_rn(x));
}

// Streaming (evict-first) 16-byte global accesses for data touched once.
__device__ __forceinline__ uint4 ld_stream(const void *p)
{
    return __ldcs(reinterpret_cast<const uint4 *>(p));
}
__device__ __forceinline__ void st_stream(void *p, const uint4 &v)
{
    __stcs(reinterpret_cast<uint4 *>(p), v);
}
// Cached read-only 16-byte load for data every row reuses (gamma).
__device__ __forceinline__ uint4 ld_reuse(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// ------------------------------------------------ programmatic dependency --
// A kernel launched with programmatic stream serialisation may begin while
// the previous kernel of the stream is still draining (its CTAs get resident
// and wait), instead of after it has fully retired.  Every library kernel
// calls pdl_wait() before its first global-memory access: the wait returns
// once the previous grid has completed and its writes are visible, so the
// usual stream ordering holds for everything the kernel reads or writes.
// pdl_trigger() lets the next dependent launch begin scheduling.  Both are
// no-ops for a kernel launched without the attribute.  The wait is the
// hardware's grid-completion dependency (like a stream dependency), not a
// software spin on a flag.
__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// The rope kernels' entry and exit under QKR_FLAG_INDEPENDENT.  A call the
// caller declares independent of the previous kernel on the stream (it reads
// nothing that kernel writes, writes nothing it reads or writes) starts its
// work without the grid-dependency wait, so its CTAs stream their rows while
// the previous kernel's last CTAs drain, and takes the wait just before it
// exits instead: it cannot complete before the previous kernel has, so every
// kernel after it still sees the writes of both.  The previous kernel's CTAs
// have all started when this one launches (each triggers its dependents
// first thing), so a CTA waiting at the end never holds an SM that the
// previous kernel still needs.
__device__ __forceinline__ void pdl_enter(int independent)
{
    if (!independent)
        pdl_wait();
    pdl_trigger();
}
__device__ __forceinline__ void pdl_exit(int independent)
{
    if (independent)
        pdl_wait();
}

// Process-wide switch (qkr_launch_overlap); 1 = launch with the attribute.
int launch_overlap();
void set_launch_overlap(int enable);

// Launch `fn` on `stream` with the programmatic-serialisation attribute when
// the switch is on, plus an optional cluster dimension (cluster_x > 1).
template <typename... Params, typename... Args>
cudaError_t launch(void (*fn)(Params...), dim3 grid, dim3 block, size_t smem,
                   cudaStream_t stream, int cluster_x, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (launch_overlap()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, fn, std::forward<Args>(args)...);
}

// ------------------------------------------------------------ section rule --
// Axis (0 t, 1 h, 2 w, 3 e) of rotated pair j under a section mode; the
// rules are stated in include/qkr.h next to QKR_SECTIONS_*.
__device__ __forceinline__ int section_axis(int mode, const int (&sec)[4], int j)
{
    if (mode == QKR_SECTIONS_NONE)
        return 0;
    const int st = sec[0], sh = sec[1], sw = sec[2];
    if (mode == QKR_SECTIONS_IMROPE) {
        const int sector = j % (st + sh + sw + sec[3]);
        const int cls = sector % 3;                       // 0 t, 1 h, 2 w
        const int quota = cls == 0 ? st : (cls == 1 ? sh : sw);
        return sector < 3 * quota ? cls : 3;
    }
    const int m = min(st, min(sh, sw));
    if (mode != QKR_SECTIONS_CONTIGUOUS && j < 3 * m)
        return j % 3;
    if (mode == QKR_SECTIONS_INTERLEAVED_QUOTA) {
        int k = j - 3 * m;
        if (k < st - m)
            return 0;
        k -= st - m;
        return k < sh - m ? 1 : 2;
    }
    return j < st ? 0 : (j < st + sh ? 1 : 2);
}

// ---------------------------------------------------- rope row descriptors --

struct RopeStreamDev {
    const __nv_bfloat16 *q;   // already advanced by the storage offset
    const __nv_bfloat16 *k;
    const __nv_bfloat16 *v;   // joint Q/K/V only (copied unchanged)
    int64_t q_ts, q_hs, k_ts, k_hs, v_ts, v_hs;
    const __nv_bfloat16 *gq;
    const __nv_bfloat16 *gk;
};

struct RopeParams {
    RopeStreamDev st[2];
    int64_t split;            // joint row where stream 1 starts (INT64_MAX: one stream)
    __nv_bfloat16 *q_out;
    __nv_bfloat16 *k_out;
    __nv_bfloat16 *v_out;     // joint Q/K/V only
    int64_t qo_ts, ko_ts, vo_ts;
    int64_t T;                // joint tokens in this launch
    int Hq, Hk, D, rot, P;
    int Hv;                   // V heads copied into v_out (0: Q/K only)
    int rows_per_token;       // Hq + Hk + Hv
    int tokens_per_cta;
    int tok_base, tok_rem;    // balanced split over the grid: CTA c owns tok_base tokens,
                              // one more when c < tok_rem (T / grid, T % grid)
    int gpt_recip;            // 2^16 / (work items per token), for the item cursor
    int pw;                   // (cos, sin) columns staged per token: P, or D/2 for GPT-J
                              // (pairs in [P, D/2) get the identity (1, 0))
    float eps, inv_D;
    int norm, round_norm;
    int angle_kind, section_mode;
    int sec[4];
    const int32_t *pos;
    int64_t pos_rs;
    const float *inv_freq;
    const float *cos;
    const float *sin;
    int64_t ld, plane_stride;
    int tab_vec4;             // table bases 16-byte aligned, ld and plane_stride % 4 == 0
    const int64_t *k_rows;    // scatter: output row of each K token (NULL: row n)
    int64_t k_out_rows;       // scatter: rows of k_out
    unsigned *status;         // device status word (scatter: out-of-range rows)
    int stages;               // streaming kernel: depth of the cp.async row ring
    int independent;          // QKR_FLAG_INDEPENDENT: wait for the previous grid at the end
    int64_t token_offset;
};

struct LaunchRecord {
    int kernel = QKR_KERNEL_NONE;
    int lanes_per_row = 0, slots = 0, tokens_per_cta = 0, heads_per_item = 0, cluster = 1,
        block = 0, pipelined = 0, direct_angles = 0, stages = 0;
    int64_t grid = 0, launches = 0;
};

// Launch-shape override of the rope kernels (0: automatic); pipeline: 0 auto,
// 1 item kernel only, 3 streaming kernel only; stages: passes of the streaming
// kernel's row ring.
void set_rope_shape_override(int pipeline, int heads_per_item, int tokens_per_cta,
                             int stages);
// Lanes per head row of the GPT-J (VECTOR) layout, for tuning (0: automatic).
void set_rope_lanes_override(int lanes);

// Reads (and optionally clears, in one atomic step on the device) the device
// status word that kernels raise bits in (status.cu).  Synchronous.
cudaError_t read_device_status(unsigned *status, bool reset);
// Device address of that status word on the current device.
cudaError_t device_status_address(unsigned **addr);
// The launch-floor probe: an empty kernel with the library's launch attributes.
cudaError_t launch_null(int64_t grid, int block, cudaStream_t stream, LaunchRecord *rec);

// Each launcher enqueues exactly one kernel and returns the CUDA launch status.
cudaError_t launch_rope_rows(const RopeParams &p, int pairing, cudaStream_t stream,
                             LaunchRecord *rec);

struct VitParams {
    const float *inv[3];
    int half[3];
    int P;
    const int32_t *cu;
    const int32_t *grids;
    int G;
    int64_t N;
    int m;
    float *cos_out;
    float *sin_out;
};
cudaError_t launch_vit_setup(const VitParams &p, cudaStream_t stream, LaunchRecord *rec);
cudaError_t launch_vit_positions(const VitParams &p, int32_t *pos_out, cudaStream_t stream,
                                 LaunchRecord *rec);
cudaError_t launch_section_map(int mode, const int (&sec)[4], int P, int8_t *out,
                               cudaStream_t stream, LaunchRecord *rec);

struct RmsParams {
    const __nv_bfloat16 *x;
    __nv_bfloat16 *res;       // NULL (FP8 variant only): no residual add
    const __nv_bfloat16 *gamma;
    __nv_bfloat16 *out;       // bf16 output (rms_norm_residual)
    uint8_t *out8;            // FP8 E4M3 output (rms_norm_fp8)
    const float *scale;       // FP8: static per-tensor scale (device fp32 [1])
    int64_t R;
    int hidden;
    int64_t xs, rs, os;
    float eps, inv_hidden;
};
cudaError_t launch_rms_norm_residual(const RmsParams &p, cudaStream_t stream,
                                     LaunchRecord *rec);
// CTAs per row and threads per CTA of the RMSNorm kernels, for tuning (0: automatic).
void set_rms_cluster_override(int cluster, int threads);

}  // namespace qkr
