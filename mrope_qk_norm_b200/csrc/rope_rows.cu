// rope_rows.cu -- launcher of the per-head RMSNorm + RoPE / mRoPE kernels,
// and the exchange kernel.
//
// Layout choice: NeoX with rot_dim % 16 == 0 runs the item kernel's PAIRED
// layout, GPT-J its VECTOR layout (rope_fast.cuh).  NeoX with
// rot_dim % 16 != 0 (EXCHANGE layout) is served by a plainer kernel here that
// passes the normalised row through shared memory to reach partners.

#include <algorithm>
#include <atomic>
#include <climits>
#include <mutex>
#include <vector>

#include "rope_stream.cuh"

namespace qkr {
namespace {

// ======================================================== exchange kernel ==
// NeoX with rot_dim % 16 != 0: a row's pair partners can sit anywhere in the
// row, so the normalised row passes through a per-group shared buffer.

template <int LPR, int NS>
__global__ void __launch_bounds__(kThreads)
rope_exchange_kernel(const __grid_constant__ RopeParams p)
{
    pdl_enter(p.independent);
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
        // rows of a token: Hq Q heads, Hk K heads, then Hv V heads (copied)
        const bool isv = h >= p.Hq + p.Hk;
        const bool isk = !isv && h >= p.Hq;
        const int hh = isv ? h - p.Hq - p.Hk : isk ? h - p.Hq : h;
        const RopeStreamDev &S = s1 ? p.st[1] : p.st[0];
        const __nv_bfloat16 *src = (isv ? S.v : isk ? S.k : S.q) +
                                   t * (isv ? S.v_ts : isk ? S.k_ts : S.q_ts) +
                                   (int64_t)hh * (isv ? S.v_hs : isk ? S.k_hs : S.q_hs);
        const __nv_bfloat16 *gam = isk ? S.gk : S.gq;
        int64_t orow = n;
        bool write = live;
        if (isk && p.k_rows && live) {  // K scatter (rope_set_rows)
            orow = __ldg(reinterpret_cast<const long long *>(p.k_rows) + n);
            if (orow < 0 || orow >= p.k_out_rows) {
                atomicOr(p.status, 4u);
                write = false;
                orow = 0;
            }
        }
        __nv_bfloat16 *dst = (isv ? p.v_out : isk ? p.k_out : p.q_out) +
                             orow * (isv ? p.vo_ts : isk ? p.ko_ts : p.qo_ts) + (int64_t)hh * D;

        float x[NS][8];
        uint4 raw[NS];
#pragma unroll
        for (int k = 0; k < NS; ++k) {
            raw[k] = (live && vidx[k] >= 0) ? ld_stream(src + 8 * vidx[k]) : make_uint4(0, 0, 0, 0);
            unpack8(raw[k], x[k]);
        }
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
                    if (p.round_norm == kRoundEager)
                        x[k][e] = round_bf16(__fmul_rn(round_bf16(__fmul_rn(x[k][e], inv_rms)),
                                                       g[e]));
                    else
                        x[k][e] = (x[k][e] * inv_rms) * g[e];
                    if (p.round_norm == kRoundNormalized)
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
                    if (p.round_norm == kRoundEager)  // every product and sum rounded
                        x[k][e] = lo ? __fsub_rn(__fmul_rn(x[k][e], cr[j]), __fmul_rn(other, sr[j]))
                                     : __fadd_rn(__fmul_rn(x[k][e], cr[j]), __fmul_rn(other, sr[j]));
                    else
                        x[k][e] = lo ? x[k][e] * cr[j] - other * sr[j]
                                     : x[k][e] * cr[j] + other * sr[j];
                }
            }
        }
        __syncwarp();
        if (write) {
#pragma unroll
            for (int k = 0; k < NS; ++k)
                if (vidx[k] >= 0)
                    st_stream(dst + 8 * vidx[k], isv ? raw[k] : pack8(x[k]));
        }
    }
    pdl_exit(p.independent);
}

// ================================================================== host ==

KernelFn pick_exchange(int lpr, int ns)
{
#define QKR_EXCHANGE_CASE(L)                                   \
    case L:                                                    \
        return ns == 1 ? rope_exchange_kernel<L, 1>            \
             : ns == 2 ? rope_exchange_kernel<L, 2> : nullptr;
    switch (lpr) {
        QKR_EXCHANGE_CASE(1)
        QKR_EXCHANGE_CASE(2)
        QKR_EXCHANGE_CASE(4)
        QKR_EXCHANGE_CASE(8)
        QKR_EXCHANGE_CASE(16)
    default: return nullptr;
    }
#undef QKR_EXCHANGE_CASE
}

// Process-wide tuning overrides (atomics: a knob set from one thread while
// another launches is a race on the launch shape only, never on memory).
std::atomic<int> g_force_pipe{0};  // 0 automatic, 1 item, 3 streaming kernel
std::atomic<int> g_force_u{0};     // heads per item (0: automatic)
std::atomic<int> g_force_tt{0};    // tokens per CTA (0: automatic)
std::atomic<int> g_force_s{0};     // streaming ring depth (0: automatic)
std::atomic<int> g_force_lpr{0};   // lanes per row, GPT-J layout (0: automatic)

// Opts `fn` in to `bytes` of dynamic shared memory on the current device.
// The largest size already granted per (device, kernel) is cached, so a
// launch after the first costs no driver call.
cudaError_t allow_smem(KernelFn fn, size_t bytes)
{
    struct Entry {
        int dev;
        KernelFn fn;
        size_t bytes;
    };
    static std::mutex mu;
    static std::vector<Entry> granted;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lock(mu);
    Entry *hit = nullptr;
    for (Entry &g : granted)
        if (g.dev == dev && g.fn == fn) {
            if (g.bytes >= bytes)
                return cudaSuccess;
            hit = &g;
        }
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess)
        return e;
    if (hit)
        hit->bytes = bytes;
    else
        granted.push_back({dev, fn, bytes});
    return cudaSuccess;
}

// CTAs of `fn` (256 threads, `smem` bytes of dynamic shared memory) resident
// on the whole current device at once.  Cached per (device, kernel, smem).
cudaError_t resident_slots(KernelFn fn, size_t smem, int *slots)
{
    struct Entry {
        int dev;
        KernelFn fn;
        size_t smem;
        int slots;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (const Entry &c : cache)
            if (c.dev == dev && c.fn == fn && c.smem == smem) {
                *slots = c.slots;
                return cudaSuccess;
            }
    }
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem);
    if (e != cudaSuccess)
        return e;
    *slots = (per_sm > 0 ? per_sm : 1) * sms;
    std::lock_guard<std::mutex> lock(mu);
    cache.push_back({dev, fn, smem, *slots});
    return cudaSuccess;
}

// Streaming kernel (rope_stream.cuh): heads per item U in {1, 2, 4}, ring
// depth S, at most kStreamTokens tokens per CTA (their staged angles share
// the CTA's shared memory with the ring).
constexpr int kStreamTokens = 64;

cudaError_t launch_rope_stream(RopeParams p, int layout, int lpr, int ns, cudaStream_t stream,
                               LaunchRecord *rec)
{
    // U = 2 heads per item with a two-pass ring was the best streaming shape
    // in the sweeps (deeper rings and U = 4 cost resident CTAs).
    const int fu = g_force_u, fs = g_force_s;
    int u = fu > 0 ? fu : 2;
    if (u == 3)
        u = 2;
    const int S = fs > 1 ? fs : 2;
    p.stages = S;
    p.pw = layout == VECTOR ? p.D / 2 : p.P;
    const int cs_ld = (p.pw + 3) & ~3;
    const bool norm = p.norm != 0;
    KernelFn fn = layout == PAIRED ? pick_stream_paired(lpr, ns, u, norm)
                                   : pick_stream_vector(lpr, ns, u, norm);
    if (!fn)
        return cudaErrorInvalidConfiguration;
    const size_t ring = (size_t)S * u * ns * kThreads * 16;
    const size_t angles_max = (size_t)kStreamTokens * cs_ld * 2 * sizeof(float);
    cudaError_t e = allow_smem(fn, ring + angles_max);
    if (e != cudaSuccess)
        return e;
    // Token split: the fewest whole waves of resident CTAs at no more than 7
    // tokens per CTA, tokens shared out evenly (at least 4 per CTA).  A sweep
    // of interleaved mRoPE launches (16+8 heads, T = 2400 .. 8192, 4 .. 16
    // tokens per CTA) put the best split there: a partly filled last wave
    // costs most (2400 tokens: 6.5 us at 5 per CTA, one wave, against 7.6 us
    // at 4, 1.01 waves; 5000: 12.1 us at 5, two waves, against 13.2 at 8),
    // and more than about 8 tokens per CTA exposes each CTA's staging
    // prologue (8192: 17.5 us at 7 against 20.2 at 12).  Against the
    // previous rule (4 per CTA below 8 x the resident CTAs, else 8) only
    // 6000 and 7000 tokens lost, 2-4%.
    int64_t grid;
    int tt = g_force_tt;
    if (tt <= 0) {
        int slots = 0;
        e = resident_slots(fn, ring + (size_t)8 * cs_ld * 2 * sizeof(float), &slots);
        if (e != cudaSuccess)
            return e;
        const int64_t waves = (p.T + 7 * (int64_t)slots - 1) / (7 * (int64_t)slots);
        const int64_t even = (p.T + waves * slots - 1) / (waves * slots);
        tt = even < 4 ? 4 : (int)even;
        // Few heads per token (K-only scatter into a cache: 8 heads, 4
        // items per token) would leave one item per lane group at 8
        // tokens, so nothing overlaps the ring's first wait: up to 16
        // tokens per CTA (5% faster than 8 on 8192 x 8 heads of K), but no
        // more than fill one wave (14 there: 586 CTAs of 592 slots, 0.8%
        // faster than 16; 12 or 13 spill into a second wave, 20% slower).
        const int items_per_token = (p.Hq + u - 1) / u + (p.Hk + u - 1) / u;
        if (8 * items_per_token < 2 * (kThreads / lpr)) {
            const int64_t wave = (p.T + slots - 1) / slots;
            tt = wave < 8 ? 8 : (wave > 16 ? 16 : (int)wave);
        }
    }
    if (tt > kStreamTokens)
        tt = kStreamTokens;
    grid = (p.T + tt - 1) / tt;
    if (grid < 1)
        grid = 1;
    p.tokens_per_cta = (int)((p.T + grid - 1) / grid);
    p.tok_base = (int)(p.T / grid);
    p.tok_rem = (int)(p.T % grid);
    p.gpt_recip = 65536 / std::max(1, (p.Hq + u - 1) / u + (p.Hk + u - 1) / u);
    const size_t smem = ring + (size_t)p.tokens_per_cta * cs_ld * 2 * sizeof(float);
    e = launch(fn, dim3((unsigned)grid), dim3(kThreads), smem, stream, 1, p);
    if (e == cudaSuccess && rec) {
        *rec = LaunchRecord();
        rec->kernel = layout == PAIRED ? QKR_KERNEL_ROPE_PAIRED : QKR_KERNEL_ROPE_VECTOR;
        rec->lanes_per_row = lpr;
        rec->slots = ns;
        rec->tokens_per_cta = p.tokens_per_cta;
        rec->heads_per_item = u;
        rec->pipelined = 2;
        rec->stages = S;
        rec->cluster = 1;
        rec->block = kThreads;
        rec->grid = grid;
        rec->launches = 1;
    }
    return e;
}

// Resident CTAs of the automatic streaming shape (U = 2, S = 2, 8 tokens of
// staged angles) for this call's layout.
cudaError_t stream_slots(const RopeParams &p, int layout, int lpr, int ns, int *slots)
{
    const int pw = layout == VECTOR ? p.D / 2 : p.P;
    const int cs_ld = (pw + 3) & ~3;
    KernelFn fn = layout == PAIRED ? pick_stream_paired(lpr, ns, 2, p.norm != 0)
                                   : pick_stream_vector(lpr, ns, 2, p.norm != 0);
    if (!fn)
        return cudaErrorInvalidConfiguration;
    const size_t ring = (size_t)2 * 2 * ns * kThreads * 16;
    const size_t angles_max = (size_t)kStreamTokens * cs_ld * 2 * sizeof(float);
    const cudaError_t e = allow_smem(fn, ring + angles_max);
    if (e != cudaSuccess)
        return e;
    return resident_slots(fn, ring + (size_t)8 * cs_ld * 2 * sizeof(float), slots);
}

int pow2_ceil(int v)
{
    int p = 1;
    while (p < v)
        p <<= 1;
    return p;
}

// Heads per work item (U) and tokens per CTA (tt) for one-vector GPT-J rows
// with table angles read per item.  A CTA of tt tokens holds
// tt * (ceil(Hq / U) + ceil(Hk / U)) work items for its lane groups, taken
// in passes of one item per group.  The split keeps the largest share of
// lane-group row slots that carry a row (the last pass part empty, or the
// last item of a head set short of U heads, wastes slots), then the fewest
// passes per CTA, then the most heads per item, over U in {4, 6} (6 only
// for 16-lane rows; a forced U alone) and at most 3 passes.  The grid is
// then as many such CTAs as the tokens need, usually several waves, so a
// partly filled last wave is a small share of the launch.  Measured on B200
// (fp32 table, head_dim 128, ~100 MB per launch; the previous rule, whole
// passes in at most two waves, in brackets):
//   * joint 512+4096 tokens x 24+24 heads: 6 x 2 (one pass) 19.1-19.3 us
//     (4 x 4, three passes: 19.8); 24+24 at 4 x 1 or 4 x 2 (a quarter of the
//     slots empty) 21.8-22.7;
//   * 32+8 heads: 4 x 3 (30 of 32 slots) 17.9 us (22.1: 611 CTAs, one
//     wave and 19 CTAs); 64+8: 6 x 1 18.8 (23.3: 339 CTAs); 6+6: 6 x 8
//     18.2 (21.1); 12+12: 6 x 4 17.5 (18.2); 16+16, 28+4, 32+32, 40+8 and
//     8+8 within 1% of the best measured shape.
void pick_item_split(int hq, int hk, int groups, bool six, int force_u, int *u_out, int *tt_out)
{
    const int cand[2] = {4, 6};
    const int ncand = force_u > 0 ? 1 : (six ? 2 : 1);
    double best = -1.0;
    int bu = force_u > 0 ? force_u : 4, btt = 1, bpass = 0;
    for (int i = 0; i < ncand; ++i) {
        const int u = force_u > 0 ? force_u : cand[i];
        const int gpt = (hq + u - 1) / u + (hk + u - 1) / u;
        if (gpt < 1)
            continue;
        const double row_share = (double)(hq + hk) / ((double)u * gpt);
        const int ttmax = std::max(1, 3 * groups / gpt);
        for (int tt = 1; tt <= ttmax; ++tt) {
            const int items = tt * gpt;
            const int passes = (items + groups - 1) / groups;
            const double score = row_share * items / ((double)passes * groups);
            const bool better = score > best + 1e-9 ||
                                (score > best - 1e-9 &&
                                 (passes < bpass || (passes == bpass && u > bu)));
            if (better) {
                best = score;
                bu = u;
                btt = tt;
                bpass = passes;
            }
        }
    }
    *u_out = bu;
    *tt_out = btt;
}

}  // namespace

void set_rope_lanes_override(int lanes) { g_force_lpr = lanes; }

void set_rope_shape_override(int pipeline, int heads_per_item, int tokens_per_cta, int stages)
{
    g_force_pipe = pipeline;
    g_force_u = heads_per_item;
    g_force_tt = tokens_per_cta;
    g_force_s = stages;
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
        // GPT-J: one 16-byte vector per lane where the row allows (up to 16
        // lanes, D <= 128): the smaller per-lane state admits 4 CTAs per SM at
        // 4 heads per item, measured 3% faster than two vectors per lane on
        // the joint 512+4096-token workload.
        lpr = layout == VECTOR ? pow2_ceil(nvec) : pow2_ceil((nvec + 1) / 2);
        if (lpr > 16)
            lpr = 16;
        if (layout == VECTOR && g_force_lpr > 0 && (nvec + g_force_lpr - 1) / g_force_lpr <= 2)
            lpr = g_force_lpr;
        ns = (nvec + lpr - 1) / lpr;
    }
    if (p.T > INT_MAX)
        return cudaErrorInvalidConfiguration;
    // Angles from positions: the streaming kernel (sincosf once per token of a
    // CTA's whole range, overlapped with the first row copies) measured ~4%
    // faster than the item kernel's per-4-token staging on interleaved mRoPE
    // (8192 x (16+8) heads); angles from a table: the item kernel with direct
    // 16-byte table reads measured ~12% faster than the streaming kernel.
    // Below a wave of streaming CTAs at 4 tokens each the item kernel with
    // 4-token staging is the faster one: 1024 tokens of interleaved mRoPE
    // (16+8 heads) took 3.7 us against 4.3 us, 16 tokens of 4+4 heads 2.5
    // against 2.8.  Above it the gain is small (2457 tokens: 8.3 against
    // 8.5 us) and is lost when a streaming launch follows directly: two
    // chunks of 2457 and 5735 tokens took 24.2 us with the first on the item
    // kernel against 23.7 us with both streaming.  With the per-head norm,
    // launches of 8192 tokens or more take the item kernel: 8192 / 16384
    // tokens of NeoX 16+16 heads 26.4 / 49.7 us against 30.2 / 57.7, 8+8
    // heads 15.9 / 29.4 against 19.9 / 36.9, 32+8 heads 34.0 / 64.7 against
    // 35.4 / 68.1, GPT-J 32+8 heads 34.8 / 65.8 against 35.8 / 70.8; 64+8
    // heads tie.  (Below 8192 tokens the two trade places by head count.)
    bool stream_auto = g_force_pipe == 0 && p.angle_kind == QKR_ANGLE_POSITIONS &&
                       !(p.norm && p.T >= 8192);
    if (stream_auto && layout != EXCHANGE && g_force_tt <= 0) {
        int slots = 0;
        const cudaError_t e = stream_slots(p, layout, lpr, ns, &slots);
        if (e != cudaSuccess)
            return e;
        stream_auto = p.T >= 4 * (int64_t)slots;
    }
    if (layout != EXCHANGE && (g_force_pipe == 3 || stream_auto))
        return launch_rope_stream(p, layout, lpr, ns, stream, rec);
    // Table angles are read per item by the item kernel (nothing staged) when
    // four consecutive pairs always come from one 16-byte aligned row segment
    // of one plane: aligned rows, P % 4 == 0, and no section boundary inside
    // a group of four pairs under a contiguous (or no) section map.
    bool direct = layout != EXCHANGE && p.angle_kind == QKR_ANGLE_TABLE && p.tab_vec4 &&
                  p.P % 4 == 0;
    if (direct && p.section_mode != QKR_SECTIONS_NONE)
        direct = p.section_mode == QKR_SECTIONS_CONTIGUOUS && p.sec[0] % 4 == 0 &&
                 (p.sec[0] + p.sec[1]) % 4 == 0;
    // NeoX rows of head_dim 64 rotated whole, with staged angles, take the
    // PAIRX lane mapping: one vector per lane and the partner half by
    // shuffle (8 lanes per row instead of 4 with two vectors each),
    // bit-identical to the paired layout.  Positions launches of 4+4 heads:
    // 16 / 256 / 1024 tokens 2.09 / 2.17 / 2.92 us against 2.20 / 2.27 /
    // 3.30.  With table angles read per item it was 18-60% slower, and at
    // head_dim 128 (16 lanes per row) slower everywhere: the per-row role
    // selects and the partner's unpacking cost more than the occupancy gained.
    if (layout == PAIRED && !direct && p.rot == p.D && p.rot == 64) {
        layout = PAIRX;
        lpr = p.rot / 8;
        ns = 1;
    }
    // staged (cos, sin) columns: GPT-J stages every pair of the head so pairs
    // past rot_dim rotate by the identity
    p.pw = layout == VECTOR ? p.D / 2 : p.P;
    const int cs_ld = (p.pw + 3) & ~3;
    const int groups = kThreads / lpr;

    // Heads per work item (U) and the token split.  Sweeps on B200 (joint
    // 512+4096 x 24 heads with both pairings, interleaved mRoPE 8192 x
    // (16+8) heads, ViT 16268 x 16 heads of D=80) gave:
    //   * direct angles, one-vector GPT-J rows: U and the token split from
    //     pick_item_split (4 or 6 heads, CTAs of one to three passes);
    //   * direct angles, other rows: U = 4 heads per item (U = 2 with four
    //     slots per lane) and one wave of resident CTAs, each owning T / grid
    //     tokens.  The balanced single wave matters most there: a grid that
    //     leaves a partly filled last wave costs up to 20%;
    //   * staged angles: U = 2 and 1-4 tokens per CTA (below).
    const bool staged = !direct;
    const int max_tt_smem = staged && cs_ld > 0 ? 16384 / (8 * cs_ld) : 64;
    int best_u = layout == EXCHANGE ? 1 : direct ? (ns <= 3 ? 4 : 2) : 2;
    if (g_force_u > 0 && layout != EXCHANGE)
        best_u = g_force_u;
    // one-vector GPT-J rows with per-item table angles: U and the token split together
    int item_tt = 0;
    if (direct && layout == VECTOR && ns == 1 && g_force_tt <= 0)
        pick_item_split(p.Hq, p.Hk, groups, lpr == 16, g_force_u, &best_u, &item_tt);
    const bool norm = p.norm != 0;
    const int rmode = p.round_norm;
    KernelFn fn;
    if (layout == PAIRED)
        fn = direct ? pick_fast_paired_direct(lpr, ns, best_u, norm, rmode)
                    : pick_fast_paired_staged(lpr, ns, best_u, norm, rmode);
    else if (layout == VECTOR)
        fn = direct ? pick_fast_vector_direct(lpr, ns, best_u, norm, rmode)
                    : pick_fast_vector_staged(lpr, ns, best_u, norm, rmode);
    else if (layout == PAIRX)
        fn = pick_fast_pairx_staged(lpr, ns, best_u, norm, rmode);
    else
        fn = pick_exchange(lpr, ns);
    if (!fn)
        return cudaErrorInvalidConfiguration;

    int64_t grid;
    if (g_force_tt > 0) {
        const int ftt = g_force_tt;
        const int tt = ftt < max_tt_smem ? ftt : max_tt_smem;
        grid = (p.T + tt - 1) / tt;
    } else if (direct) {
        int slots = 0;
        cudaError_t e = resident_slots(fn, 0, &slots);
        if (e != cudaSuccess)
            return e;
        if (item_tt > 0) {
            grid = (p.T + item_tt - 1) / item_tt;
        } else {
            // The other direct-angle rows (NeoX pairs, two-vector GPT-J
            // lanes; 2 CTAs per SM): tokens per CTA a multiple of the count
            // that gives every lane group the same number of work items
            // (whole passes), the smallest whose grid fits in one wave of
            // resident CTAs.  NeoX joint 512+4096 tokens x 24 heads at 16 per
            // CTA (288 CTAs, 6 passes) 21.03 us against 21.2 at 15-16 and
            // 21.44 at 8 (two waves); ViT apply lost 8% on two waves.
            const int items = (p.Hq + best_u - 1) / best_u + (p.Hk + best_u - 1) / best_u;
            int a = items, b = groups;
            while (b) {
                const int r = a % b;
                a = b;
                b = r;
            }
            const int64_t unit = groups / (a > 0 ? a : 1);  // tokens per CTA for whole passes
            int64_t tt = unit;
            if ((p.T + tt - 1) / tt > slots)
                tt = ((p.T + slots - 1) / slots + unit - 1) / unit * unit;
            grid = (p.T + tt - 1) / tt;
        }
        // launches of fewer tokens than resident CTAs: one token per CTA
        // spreads them over the most SMs
        if (p.T < slots)
            grid = p.T;
    } else if (layout == EXCHANGE) {
        const int tt = 4 < max_tt_smem ? 4 : max_tt_smem;
        grid = (p.T + tt - 1) / tt;
    } else {
        // Staged angles: tokens per CTA that give the lane groups about one
        // pass of work items, doubled while the grid would exceed one wave
        // of resident CTAs, and at most 4 (several CTAs per SM keep one CTA's
        // staging prologue under another's row traffic).  Positions launches
        // (fp32 angles from int32 positions, B200, against 4 per CTA):
        // GPT-J 16+16 heads x 128 at 1 per CTA, 16 / 256 tokens 2.08 / 2.75
        // us against 3.91 / 5.46, and at 2 per CTA, 1024 tokens 5.58 against
        // 6.86; NeoX 16+16 heads at 2 per CTA, 16 / 256 tokens 2.27 / 3.16
        // against 3.15 / 4.22; interleaved mRoPE 16+8 heads at 2 per CTA,
        // 64 / 512 tokens 2.04 / 2.49 against 2.55 / 2.68.  Rows of few heads
        // (4+4 heads x 64) keep 4 per CTA.
        int slots = 0;
        const size_t smem4 = (size_t)4 * cs_ld * 2 * sizeof(float);
        cudaError_t e = resident_slots(fn, smem4, &slots);
        if (e != cudaSuccess)
            return e;
        const int gpt = (p.Hq + best_u - 1) / best_u + (p.Hk + best_u - 1) / best_u;
        int tt = std::max(1, std::min(4, groups / std::max(1, gpt)));
        while (tt < 4 && (p.T + tt - 1) / tt > slots)
            tt = std::min(4, 2 * tt);
        if (tt > max_tt_smem)
            tt = max_tt_smem;
        grid = (p.T + tt - 1) / tt;
    }
    if (grid < 1)
        grid = 1;
    // the exchange kernel walks fixed tiles; the item kernels take balanced ranges
    p.tokens_per_cta = (int)((p.T + grid - 1) / grid);
    p.tok_base = (int)(p.T / grid);
    p.tok_rem = (int)(p.T % grid);
    {
        const int ug = layout == EXCHANGE ? 1 : best_u;
        p.gpt_recip = 65536 / std::max(1, (p.Hq + ug - 1) / ug + (p.Hk + ug - 1) / ug);
    }

    size_t smem = staged ? (size_t)p.tokens_per_cta * cs_ld * 2 * sizeof(float) : 0;
    if (layout == EXCHANGE)
        smem += (size_t)groups * p.D * sizeof(float);
    smem = (smem + 15) & ~(size_t)15;
    if (smem > 48 * 1024) {
        const cudaError_t e = allow_smem(fn, smem);
        if (e != cudaSuccess)
            return e;
    }
    cudaError_t err = launch(fn, dim3((unsigned)grid), dim3(kThreads), smem, stream, 1, p);
    if (err == cudaSuccess && rec) {
        *rec = LaunchRecord();
        rec->kernel = layout == PAIRED || layout == PAIRX ? QKR_KERNEL_ROPE_PAIRED
                    : layout == VECTOR   ? QKR_KERNEL_ROPE_VECTOR
                                         : QKR_KERNEL_ROPE_EXCHANGE;
        rec->lanes_per_row = lpr;
        rec->slots = ns;
        rec->tokens_per_cta = p.tokens_per_cta;
        rec->heads_per_item = layout == EXCHANGE ? 1 : best_u;
        rec->cluster = 1;
        rec->block = kThreads;
        rec->direct_angles = direct ? 1 : 0;
        rec->grid = grid;
        rec->launches = 1;
    }
    return err;
}

}  // namespace qkr
