// rope_tma.cu -- bulk-copy pipelined per-head RMSNorm + RoPE (sm_100a).
//
// Same arithmetic as the item kernel (the shared row math of rope_math.cuh;
// fused_qk_norm_rope, vllm-omni #7600; mrope_apply, llama.cpp fork #286).  A memory-bound
// kernel must keep tens of KB per SM in flight; here those bytes wait in a
// shared-memory ring filled by the copy engine instead of in registers:
//
//   * persistent grid along tokens (as many CTAs per SM as fit), and
//     gridDim.y splits the head slots (Q heads, then K heads) when there are
//     more than one CTA's consumers can own;
//   * a tile is `tokens_per_tile` consecutive joint tokens; CTA x takes tiles
//     x, x + gridDim.x, ...;
//   * warp 0 is the producer.  For each tile it waits until a stage of the
//     ring is free, arrives on the stage's "full" mbarrier with the tile's
//     byte count and issues 1-D cp.async.bulk copies (global -> shared,
//     completion on that mbarrier) of the CTA's head rows of the tile's
//     tokens -- one copy per (token, Q or K) run when heads are dense, else
//     one per row.  It never waits on a load of its own;
//   * the other warps are consumers, one group of LPR lanes per head slot
//     (head-stationary): gamma stays in registers, and for each tile the
//     group reads its head's rows for the tile's tokens from shared memory,
//     takes each token's (cos, sin) from a shared table the consumers stage
//     up front (in chunks, between consumer-only named barriers), runs the
//     packed fp32x2 RMSNorm + rotation, writes 16-byte streaming stores and
//     releases the stage through its "empty" mbarrier;
//   * every wait is bounded by a clock budget.  On timeout the thread sets a
//     device error word and an abort flag; the producer waits (again bounded)
//     for the copies it issued, the consumers skip the remaining work while
//     keeping their barrier sequence, and all threads return.
// No TMA multicast is used: each CTA copies only what it consumes.

#include <climits>

#include "rope_math.cuh"

namespace qkr {

__device__ unsigned int g_device_error;  // QKR device status word (0: no error)

namespace {

constexpr int kMaxConsumerThreads = 384;
constexpr int kMaxThreads = 32 + kMaxConsumerThreads;
constexpr int kStages = 4;
constexpr long long kWaitBudgetCycles = 4000000000LL;  // ~2 s at 1.9 GHz

// ---------------------------------------------------------------- PTX -----

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Barrier among the consumer threads only (named barrier 1).
__device__ __forceinline__ void consumers_sync(int nthreads)
{
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Bounded wait on a phase of an mbarrier.  Returns false on timeout or when
// another thread of the CTA has aborted.
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort,
                                           unsigned code)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort)
            return false;
        if (clock64() - t0 > kWaitBudgetCycles) {
            atomicOr(&g_device_error, code);
            *abort = 1;
            return false;
        }
    }
    return true;
}

struct TileGeom {
    int64_t tok0;
    int ntok;
};

__device__ __forceinline__ TileGeom tile_geom(const RopeParams &p, int64_t tile)
{
    TileGeom g;
    g.tok0 = tile * p.tokens_per_cta;
    g.ntok = (int)min((int64_t)p.tokens_per_cta, p.T - g.tok0);
    return g;
}

// Launch-time constants of one pipelined launch.
struct TmaGeom {
    int64_t n_tiles;
    int stage_bytes;   // bytes of one ring stage (tokens_per_tile * hc rows)
    int chunk_tiles;   // tiles whose (cos, sin) are staged at once
    int hc;            // head slots owned by a CTA (consumer lane groups)
    int n_consumers;   // consumer threads (multiple of 32)
};

// ---------------------------------------------------------- the kernel ----

template <int LAYOUT, int LPR, int NS, bool NORM, bool ROUND>
__global__ void __launch_bounds__(kMaxThreads, 2)
rope_tma_kernel(const __grid_constant__ RopeParams p, const __grid_constant__ TmaGeom tg)
{
    pdl_wait();
    pdl_trigger();
    constexpr int NQ = RowShape<LAYOUT, NS>::NQ;
    constexpr int NTA = RowShape<LAYOUT, NS>::NTA;

    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty = full + kStages;
    volatile int *abort = reinterpret_cast<volatile int *>(empty + kStages);
    const int cs_ld = (p.pw + 3) & ~3;
    const int TT = p.tokens_per_cta;
    // (cos, sin) of a chunk of this CTA's tiles: [chunk tile][token][cs_ld]
    float *ang_cos = reinterpret_cast<float *>(smem + 128);
    float *ang_sin = ang_cos + (size_t)tg.chunk_tiles * TT * cs_ld;
    unsigned char *stages =
        smem + 128 + (((size_t)tg.chunk_tiles * TT * cs_ld * 8 + 127) & ~(size_t)127);

    const int warp = threadIdx.x >> 5;
    const int lane32 = threadIdx.x & 31;
    const int D = p.D;
    const int hc = tg.hc;
    const int slot0 = blockIdx.y * hc;                       // first head slot of this CTA
    const int nslots = min(hc, p.Hq + p.Hk - slot0);         // head slots this CTA owns
    const int nq = max(0, min(p.Hq - slot0, nslots));        // of them Q heads
    const int ncw = tg.n_consumers >> 5;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], ncw);
        }
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    const RopeStreamDev &S0 = p.st[0];
    const RopeStreamDev &S1 = p.st[1];
    const int64_t my_tiles =
        blockIdx.x < tg.n_tiles ? (tg.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (warp == 0) {
        // =============================== producer ===========================
        int issued[kStages] = {0, 0, 0, 0};
        bool ok = true;
        for (int64_t i = 0; i < my_tiles; ++i) {
            const int64_t tile = blockIdx.x + i * gridDim.x;
            const int slot = (int)(i % kStages);
            const int use = (int)(i / kStages);
            // the whole warp takes the same decision, so the __syncwarp below and
            // the drain see all 32 lanes
            const bool w_ok = use == 0 || wait_phase(&empty[slot], (use - 1) & 1, abort, 1u);
            if (!__all_sync(0xffffffffu, w_ok)) {
                ok = false;
                break;
            }
            __nv_bfloat16 *st =
                reinterpret_cast<__nv_bfloat16 *>(stages + (size_t)slot * tg.stage_bytes);
            const TileGeom g = tile_geom(p, tile);
            if (lane32 == 0)
                mbar_arrive_expect_tx(&full[slot], (uint32_t)g.ntok * nslots * D * 2);
            __syncwarp();
            // stage rows: [token][head slot of this CTA][D]
            for (int tt = 0; tt < g.ntok; ++tt) {
                const int64_t n = g.tok0 + tt;
                const bool s1 = n >= p.split;
                const int64_t t = s1 ? n - p.split : n;
                const RopeStreamDev &S = s1 ? S1 : S0;
#pragma unroll
                for (int kind = 0; kind < 2; ++kind) {
                    // this CTA's heads of this kind: slots [a, b) of the CTA
                    const int a = kind ? nq : 0;
                    const int b = kind ? nslots : nq;
                    if (a >= b)
                        continue;
                    const int h0 = kind ? slot0 + nq - p.Hq : slot0;  // first head index
                    const __nv_bfloat16 *base = kind ? S.k : S.q;
                    const int64_t ts = kind ? S.k_ts : S.q_ts;
                    const int64_t hs = kind ? S.k_hs : S.q_hs;
                    const __nv_bfloat16 *src = base + t * ts + (int64_t)h0 * hs;
                    __nv_bfloat16 *dst = st + ((size_t)tt * hc + a) * D;
                    if (hs == D) {
                        if (lane32 == ((tt * 2 + kind) & 31))
                            bulk_g2s(dst, src, (uint32_t)(b - a) * D * 2, &full[slot]);
                    } else {
                        for (int r = lane32; r < b - a; r += 32)
                            bulk_g2s(dst + (size_t)r * D, src + r * hs, (uint32_t)D * 2,
                                     &full[slot]);
                    }
                }
            }
            ++issued[slot];
        }
        if (!ok) {
            // drain: wait (bounded) for the copies this CTA issued, then leave
            for (int s = 0; s < kStages; ++s) {
                if (issued[s] == 0)
                    continue;
                const long long t0 = clock64();
                while (!mbar_try_wait(&full[s], (issued[s] - 1) & 1) &&
                       clock64() - t0 < kWaitBudgetCycles) {
                }
            }
        }
        return;
    }

    // ================================ consumers =============================
    const int ctid = threadIdx.x - 32;
    const int lane = ctid % LPR;
    const int grp = ctid / LPR;              // head slot within the CTA
    const bool have = grp < nslots;
    const bool isk = grp >= nq;
    const int h = isk ? slot0 + grp - p.Hq : slot0 + grp;
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
        vidx[k] = (have && v >= 0 && v < nvec) ? v : -1;
    }
    int qpair[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q)
        qpair[q] = LAYOUT == PAIRED ? 8 * lane + 2 * q : 4 * (lane + LPR * (q >> 1)) + 2 * (q & 1);
    __nv_bfloat16 *const obase = (isk ? p.k_out : p.q_out) + (int64_t)(have ? h : 0) * D;
    const int64_t ots = isk ? p.ko_ts : p.qo_ts;

    float2 GA[NQ], GB[NQ], GT[NTA][4];
    int gstream = -1;
    bool dead = false;  // a wait ran out: skip work but keep the barrier sequence

    for (int64_t i = 0; i < my_tiles; ++i) {
        const int64_t tile = blockIdx.x + i * gridDim.x;
        const int64_t ci = i % tg.chunk_tiles;  // position inside the angle chunk
        if (ci == 0) {
            // stage (cos, sin) of the chunk's tiles; identity past the rotated pairs
            consumers_sync(tg.n_consumers);  // everyone is done with the previous chunk
            const int64_t nct = min((int64_t)tg.chunk_tiles, my_tiles - i);
            const int per_tile = TT * p.pw;
            for (int64_t e = ctid; e < nct * per_tile; e += tg.n_consumers) {
                const int lt = (int)(e / per_tile);
                const int r = (int)(e - (int64_t)lt * per_tile);
                const int tt = r / p.pw;
                const int j = r - tt * p.pw;
                const TileGeom gg = tile_geom(p, tile + (int64_t)lt * gridDim.x);
                float c = 1.f, sn = 0.f;
                if (tt < gg.ntok && j < p.P) {
                    const int64_t n = p.token_offset + gg.tok0 + tt;
                    const int axis = section_axis(p.section_mode, p.sec, j);
                    if (p.angle_kind == QKR_ANGLE_POSITIONS) {
                        const int32_t pos = __ldg(p.pos + (int64_t)axis * p.pos_rs + n);
                        sincosf(__fmul_rn((float)pos, __ldg(p.inv_freq + j)), &sn, &c);
                    } else {
                        const int64_t at = (int64_t)axis * p.plane_stride + n * p.ld + j;
                        c = __ldg(p.cos + at);
                        sn = __ldg(p.sin + at);
                    }
                }
                const size_t row = (size_t)lt * TT + tt;
                ang_cos[row * cs_ld + j] = c;
                ang_sin[row * cs_ld + j] = sn;
            }
            consumers_sync(tg.n_consumers);
        }
        const int slot = (int)(i % kStages);
        const int use = (int)(i / kStages);
        // warp-uniform decision: the shuffles below need every lane of the warp
        const bool w_ok = !dead && wait_phase(&full[slot], use & 1, abort, 2u);
        dead = !__all_sync(0xffffffffu, w_ok);
        if (dead)
            continue;
        const __nv_bfloat16 *st =
            reinterpret_cast<const __nv_bfloat16 *>(stages + (size_t)slot * tg.stage_bytes);
        const float *cosv = ang_cos + (size_t)ci * TT * cs_ld;
        const float *sinv = ang_sin + (size_t)ci * TT * cs_ld;
        const TileGeom g = tile_geom(p, tile);

        for (int tt = 0; tt < g.ntok; ++tt) {  // one token per step (uniform trip count)
            uint4 raw[NS];
#pragma unroll
            for (int k = 0; k < NS; ++k)
                raw[k] = vidx[k] >= 0 ? *reinterpret_cast<const uint4 *>(
                                            st + ((size_t)tt * hc + grp) * D + 8 * vidx[k])
                                      : make_uint4(0, 0, 0, 0);
            {
                const int64_t n = g.tok0 + tt;
                const int s1 = n >= p.split;
                if (NORM && s1 != gstream) {  // first row, or the tile crossed into stream 1
                    gstream = s1;
                    const __nv_bfloat16 *gam = isk ? (s1 ? S1.gk : S0.gk) : (s1 ? S1.gq : S0.gq);
                    uint4 gv[NS];
#pragma unroll
                    for (int k = 0; k < NS; ++k)
                        gv[k] = vidx[k] >= 0 ? ld_reuse(gam + 8 * vidx[k]) : make_uint4(0, 0, 0, 0);
                    unpack_row<LAYOUT, NS>(gv, GA, GB, GT);
                }

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
                float2 C[NQ], Sn[NQ];
                const float *cr = cosv + tt * cs_ld;
                const float *sr = sinv + tt * cs_ld;
#pragma unroll
                for (int q = 0; q < NQ; q += 2) {
                    const bool okq = LAYOUT == PAIRED ? vidx[0] >= 0 : vidx[q >> 1] >= 0;
                    const float4 c4 = okq ? *reinterpret_cast<const float4 *>(cr + qpair[q])
                                          : make_float4(1.f, 1.f, 1.f, 1.f);
                    const float4 s4 = okq ? *reinterpret_cast<const float4 *>(sr + qpair[q])
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                    C[q] = f2(c4.x, c4.y);
                    C[q + 1] = f2(c4.z, c4.w);
                    Sn[q] = f2(s4.x, s4.y);
                    Sn[q + 1] = f2(s4.z, s4.w);
                }
                RotCoef<NQ, NORM && !ROUND> kc;
                make_coef(kc, C, Sn, GA, GB);
                norm_rotate<LAYOUT, NS, NORM, ROUND>(A, B, TL, r, kc, GA, GB, GT);
                uint4 outv[NS];
                pack_row<LAYOUT, NS>(A, B, TL, outv);
                __nv_bfloat16 *dst = obase + n * ots;
#pragma unroll
                for (int k = 0; k < NS; ++k)
                    if (vidx[k] >= 0)
                        st_stream(dst + 8 * vidx[k], outv[k]);
            }
        }
        __syncwarp();
        if (lane32 == 0)
            mbar_arrive(&empty[slot]);
    }
}

using KernelFn = void (*)(RopeParams, TmaGeom);

template <int LAYOUT, int LPR, int NS>
KernelFn pick_flags(bool norm, bool round)
{
    if (!norm)
        return rope_tma_kernel<LAYOUT, LPR, NS, false, false>;
    return round ? rope_tma_kernel<LAYOUT, LPR, NS, true, true>
                 : rope_tma_kernel<LAYOUT, LPR, NS, true, false>;
}

template <int LAYOUT, int LPR>
KernelFn pick_ns(int ns, bool norm, bool round)
{
    if constexpr (LAYOUT == PAIRED) {
        switch (ns) {
        case 2: return pick_flags<LAYOUT, LPR, 2>(norm, round);
        case 3: return pick_flags<LAYOUT, LPR, 3>(norm, round);
        case 4: return pick_flags<LAYOUT, LPR, 4>(norm, round);
        default: return nullptr;
        }
    } else {
        switch (ns) {
        case 1: return pick_flags<LAYOUT, LPR, 1>(norm, round);
        case 2: return pick_flags<LAYOUT, LPR, 2>(norm, round);
        default: return nullptr;
        }
    }
}

template <int LAYOUT>
KernelFn pick(int lpr, int ns, bool norm, bool round)
{
    switch (lpr) {
    case 1: return pick_ns<LAYOUT, 1>(ns, norm, round);
    case 2: return pick_ns<LAYOUT, 2>(ns, norm, round);
    case 4: return pick_ns<LAYOUT, 4>(ns, norm, round);
    case 8: return pick_ns<LAYOUT, 8>(ns, norm, round);
    case 16: return pick_ns<LAYOUT, 16>(ns, norm, round);
    default: return nullptr;
    }
}

int sm_count()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace

// Returns cudaErrorNotSupported when the call is outside what the pipelined
// kernel serves (joint V, scatter): it is reached only when a caller forces it
// through qkr_tune_rope, and such a call then fails with QKR_ERR_CUDA.
cudaError_t launch_rope_tma(const RopeParams &p_in, int layout_paired, int lpr, int ns,
                            int tokens_per_tile, cudaStream_t stream, LaunchRecord *rec)
{
    if (p_in.k_rows)
        return cudaErrorNotSupported;  // the scatter is served by the other kernels
    if (p_in.Hv > 0)
        return cudaErrorNotSupported;  // joint Q/K/V is served by the other kernels
    RopeParams p = p_in;
    const int layout = layout_paired ? PAIRED : VECTOR;
    p.pw = layout == VECTOR ? p.D / 2 : p.P;
    const int cs_ld = (p.pw + 3) & ~3;
    const int slots_total = p.Hq + p.Hk;

    // head slots per CTA: as many as the consumer threads allow
    const int max_hc = kMaxConsumerThreads / lpr;
    const int gy = (slots_total + max_hc - 1) / max_hc;
    const int hc = (slots_total + gy - 1) / gy;
    const int n_consumers = ((hc * lpr + 31) / 32) * 32;
    if (gy > 65535)
        return cudaErrorNotSupported;

    // tokens per tile: a stage of about 24 KB
    const int row_bytes = hc * p.D * 2;
    int tt = tokens_per_tile > 0 ? tokens_per_tile : (int)(24 * 1024 / row_bytes);
    if (tt < 1)
        tt = 1;
    if (tt > 16)
        tt = 16;
    if ((long)tt * row_bytes > 64 * 1024)
        return cudaErrorNotSupported;
    if (tt > p.T)
        tt = (int)p.T;
    p.tokens_per_cta = tt;
    const int stage_bytes = ((tt * row_bytes) + 127) & ~127;
    const int64_t n_tiles = (p.T + tt - 1) / tt;

    KernelFn fn = layout == PAIRED ? pick<PAIRED>(lpr, ns, p.norm != 0, p.round_norm != 0)
                                   : pick<VECTOR>(lpr, ns, p.norm != 0, p.round_norm != 0);
    if (!fn)
        return cudaErrorNotSupported;

    // angle staging: all of a CTA's tiles if they fit in 16 KB, else chunks;
    // CTAs per SM from the occupancy of this shared-memory footprint
    const int64_t bytes_per_tile = (int64_t)tt * cs_ld * 8;
    TmaGeom tg;
    tg.n_tiles = n_tiles;
    tg.stage_bytes = stage_bytes;
    tg.hc = hc;
    tg.n_consumers = n_consumers;
    int64_t grid_x = 0;
    size_t smem = 0;
    for (int pass = 0; pass < 2; ++pass) {
        const int64_t guess_ctas = grid_x > 0 ? grid_x : 2LL * sm_count();
        const int64_t tiles_per_cta = (n_tiles + guess_ctas - 1) / guess_ctas;
        int64_t chunk = 16 * 1024 / (bytes_per_tile > 0 ? bytes_per_tile : 1);
        if (chunk < 1)
            chunk = 1;
        if (chunk > tiles_per_cta)
            chunk = tiles_per_cta;
        tg.chunk_tiles = (int)chunk;
        smem = 128 + (((size_t)chunk * bytes_per_tile + 127) & ~(size_t)127) +
               (size_t)kStages * stage_bytes;
        if (smem > 200 * 1024)
            return cudaErrorNotSupported;
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess)
            return e;
        int resident = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, fn, 32 + n_consumers, smem) !=
                cudaSuccess ||
            resident < 1)
            resident = 1;
        grid_x = (int64_t)resident * sm_count() / gy;
        if (grid_x < 1)
            grid_x = 1;
        if (grid_x > n_tiles)
            grid_x = n_tiles;
    }
    cudaError_t e = launch(fn, dim3((unsigned)grid_x, (unsigned)gy), dim3(32 + n_consumers),
                           smem, stream, 1, p, tg);
    if (e == cudaSuccess && rec) {
        *rec = LaunchRecord();
        rec->kernel = layout == PAIRED ? QKR_KERNEL_ROPE_PAIRED : QKR_KERNEL_ROPE_VECTOR;
        rec->lanes_per_row = lpr;
        rec->slots = ns;
        rec->tokens_per_cta = tt;
        rec->heads_per_item = hc;
        rec->cluster = 1;
        rec->block = 32 + n_consumers;
        rec->grid = grid_x * gy;
        rec->launches = 1;
        rec->pipelined = 1;
    }
    return e;
}

cudaError_t device_status_address(unsigned **addr)
{
    void *a = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&a, g_device_error);
    *addr = static_cast<unsigned *>(a);
    return e;
}

cudaError_t read_device_status(unsigned *status, bool reset)
{
    cudaError_t e = cudaMemcpyFromSymbol(status, g_device_error, sizeof(unsigned));
    if (e == cudaSuccess && reset) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned));
    }
    return e;
}

}  // namespace qkr
