// qkr_api.cu -- the C ABI of include/qkr.h: host-side validation and launch.
//
// Every entry point validates all arguments before enqueuing anything and
// refuses (never degrades) when it cannot serve a call exactly; it never
// allocates, frees or synchronises.

#include <atomic>
#include <climits>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <string>

#include "qkr_internal.cuh"

namespace qkr {
namespace {
std::atomic<int> g_overlap{1};
}
int launch_overlap() { return g_overlap.load(std::memory_order_relaxed); }
void set_launch_overlap(int enable) { g_overlap.store(enable ? 1 : 0); }
}  // namespace qkr

namespace {

thread_local std::string g_error;
thread_local qkr::LaunchRecord g_last;

qkr_status fail(qkr_status st, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_error = buf;
    return st;
}

qkr_status cuda_result(cudaError_t e, const char *what)
{
    if (e != cudaSuccess)
        return fail(QKR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    g_error.clear();
    return QKR_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Byte span [lo, hi) touched by a [T, H, D] bf16 view with positive strides.
struct Span {
    uintptr_t lo = 0, hi = 0;
};
Span view_span(const void *base, int64_t T, int64_t ts, int64_t H, int64_t hs, int64_t D)
{
    Span s;
    if (T <= 0 || H <= 0)
        return s;
    s.lo = reinterpret_cast<uintptr_t>(base);
    const int64_t last = (T - 1) * ts + (H - 1) * hs + D;  // elements
    s.hi = s.lo + (uintptr_t)last * 2u;
    return s;
}
bool overlap(const Span &a, const Span &b)
{
    return a.lo < a.hi && b.lo < b.hi && a.lo < b.hi && b.lo < a.hi;
}

// A strided bf16 [T, H, D] view: element (t, h, d) at base + t*ts + h*hs + d.
struct View {
    const void *base = nullptr;
    int64_t T = 0, ts = 0, H = 0, hs = 0, D = 0;
};
Span span(const View &v) { return view_span(v.base, v.T, v.ts, v.H, v.hs, v.D); }

// True when two views share no element.  Either their byte spans do not
// intersect, or both advance by the same token stride and, within that
// stride, the columns one view's token row covers lie outside the other's
// (Q and K as column windows of one packed [T, 3, H, D] buffer, say): then no
// row of one reaches a byte of the other, whatever tokens they cover.
bool views_disjoint(const View &a, const View &b)
{
    const Span sa = span(a), sb = span(b);
    if (!overlap(sa, sb))
        return true;
    if (a.ts != b.ts || a.ts <= 0)
        return false;
    const int64_t TS = 2 * a.ts;                        // token stride in bytes
    const int64_t wa = 2 * ((a.H - 1) * a.hs + a.D);    // bytes of a token row
    const int64_t wb = 2 * ((b.H - 1) * b.hs + b.D);
    if (wa > TS || wb > TS)
        return false;
    const int64_t diff = (int64_t)(reinterpret_cast<uintptr_t>(b.base) -
                                   reinterpret_cast<uintptr_t>(a.base));
    const int64_t rel = ((diff % TS) + TS) % TS;        // b's row start inside a's row grid
    return rel >= wa && rel + wb <= TS;
}

// Largest element offset a view reaches must stay far from int64 overflow.
bool view_fits(int64_t T, int64_t ts, int64_t H, int64_t hs, int64_t D)
{
    const __int128 last = (__int128)(T > 0 ? T - 1 : 0) * ts + (__int128)(H > 0 ? H - 1 : 0) * hs + D;
    return last < ((__int128)1 << 60);
}

int rows_for_mode(int mode)
{
    return mode == QKR_SECTIONS_NONE ? 1 : (mode == QKR_SECTIONS_IMROPE ? 4 : 3);
}

qkr_status check_sections(int mode, const int32_t *sec, int64_t P, int (&out)[4])
{
    for (int i = 0; i < 4; ++i)
        out[i] = 0;
    if (mode < QKR_SECTIONS_NONE || mode > QKR_SECTIONS_IMROPE)
        return fail(QKR_ERR_INVALID_ARG, "unknown section mode %d", mode);
    if (mode == QKR_SECTIONS_NONE)
        return QKR_OK;
    if (!sec)
        return fail(QKR_ERR_INVALID_ARG,
                    "section mode %d needs its sections: refusing rather than rotating every "
                    "pair by one row", mode);
    int64_t sum = 0;
    for (int i = 0; i < 4; ++i) {
        if (sec[i] < 0 || sec[i] > (1 << 20))
            return fail(QKR_ERR_INVALID_ARG, "section %d = %d out of range", i, sec[i]);
        sum += sec[i];
        out[i] = sec[i];
    }
    if (mode != QKR_SECTIONS_IMROPE && sec[3] != 0)
        return fail(QKR_ERR_INVALID_ARG, "a fourth section is only read by the IMROPE mode");
    if (P > 0 && (sum < P || sum > 2 * P))
        return fail(QKR_ERR_INVALID_ARG,
                    "sections sum to %lld; %lld rotated pairs need P <= sum <= 2P",
                    (long long)sum, (long long)P);
    if (P == 0 && sum == 0 && mode == QKR_SECTIONS_IMROPE)
        return fail(QKR_ERR_INVALID_ARG, "IMROPE sections must not all be zero");
    return QKR_OK;
}

// Angle descriptor checks; fills the device-side fields of RopeParams.
qkr_status check_angle(const qkr_angle_desc *a, int64_t P, int64_t T, qkr::RopeParams &p)
{
    if (!a)
        return fail(QKR_ERR_INVALID_ARG, "angle descriptor is NULL");
    int sec[4];
    qkr_status st = check_sections(a->section_mode, a->sections, P, sec);
    if (st != QKR_OK)
        return st;
    p.section_mode = a->section_mode;
    for (int i = 0; i < 4; ++i)
        p.sec[i] = sec[i];
    p.angle_kind = a->kind;
    p.token_offset = a->token_offset;
    if (a->token_offset < 0)
        return fail(QKR_ERR_INVALID_ARG, "token_offset must be >= 0");
    if (P == 0)
        return QKR_OK;  // nothing is rotated: the angle source is never read
    if (a->kind == QKR_ANGLE_POSITIONS) {
        if (!a->positions || !a->inv_freq)
            return fail(QKR_ERR_INVALID_ARG, "positions and inv_freq must be non-NULL");
        if (!aligned4(a->positions) || !aligned4(a->inv_freq))
            return fail(QKR_ERR_UNSUPPORTED, "positions / inv_freq must be 4-byte aligned");
        if (a->pos_row_stride < 0 || a->token_offset + T > a->pos_row_stride)
            return fail(QKR_ERR_INVALID_ARG,
                        "token_offset (%lld) + tokens (%lld) exceeds the positions row length "
                        "(%lld)", (long long)a->token_offset, (long long)T,
                        (long long)a->pos_row_stride);
        p.pos = a->positions;
        p.pos_rs = a->pos_row_stride;
        p.inv_freq = a->inv_freq;
    } else if (a->kind == QKR_ANGLE_TABLE) {
        if (!a->cos || !a->sin)
            return fail(QKR_ERR_INVALID_ARG, "cos and sin tables must be non-NULL");
        if (!aligned4(a->cos) || !aligned4(a->sin))
            return fail(QKR_ERR_UNSUPPORTED, "cos / sin tables must be 4-byte aligned");
        if (a->ld < P)
            return fail(QKR_ERR_INVALID_ARG, "table ld (%lld) < rotated pairs (%lld)",
                        (long long)a->ld, (long long)P);
        if (a->table_rows < 0 || a->token_offset + T > a->table_rows)
            return fail(QKR_ERR_INVALID_ARG,
                        "token_offset (%lld) + tokens (%lld) exceeds the table rows (%lld)",
                        (long long)a->token_offset, (long long)T, (long long)a->table_rows);
        const int planes = rows_for_mode(a->section_mode);
        if (planes > 1 && a->plane_stride < a->table_rows * a->ld)
            return fail(QKR_ERR_INVALID_ARG, "plane_stride (%lld) smaller than one plane",
                        (long long)a->plane_stride);
        p.cos = a->cos;
        p.sin = a->sin;
        p.ld = a->ld;
        p.plane_stride = a->plane_stride;
        // four consecutive pairs of a row in one 16-byte load when every row
        // (and plane) start keeps 16-byte alignment
        p.tab_vec4 = aligned16(a->cos) && aligned16(a->sin) && a->ld % 4 == 0 &&
                     (planes == 1 || a->plane_stride % 4 == 0);
    } else {
        return fail(QKR_ERR_INVALID_ARG, "unknown angle kind %d", a->kind);
    }
    return QKR_OK;
}

qkr_status check_geometry(int64_t Hq, int64_t Hk, int64_t D, int64_t rot, int32_t pairing,
                          float eps, bool k_only = false)
{
    if (Hq < (k_only ? 0 : 1) || Hk < 1 || Hq + Hk > 65536)
        return fail(QKR_ERR_INVALID_ARG, "head counts must be >= 1 and Hq + Hk <= 65536");
    if (D < 8 || D > 256 || D % 8)
        return fail(QKR_ERR_UNSUPPORTED, "head_dim %lld: need a multiple of 8 in [8, 256]",
                    (long long)D);
    if (rot < 0 || rot > D || rot % 2)
        return fail(QKR_ERR_INVALID_ARG, "rot_dim %lld: need an even value in [0, head_dim]",
                    (long long)rot);
    if (pairing != QKR_PAIRING_NEOX && pairing != QKR_PAIRING_GPTJ)
        return fail(QKR_ERR_INVALID_ARG, "unknown pairing %d", pairing);
    if (!(eps >= 0.f) || eps > 1.f)
        return fail(QKR_ERR_INVALID_ARG, "eps must be finite and in [0, 1]");
    return QKR_OK;
}

// Shared body of fused_qk_norm_rope, fused_qkv_norm_rope and mrope_apply.
// `inplace_ok` admits outputs equal to the inputs with identical strides
// (mrope_apply).  Hv > 0 routes each stream's V rows into v_out unchanged.
qkr_status rope_call(void *stream, const qkr_stream_desc *streams, int32_t n_streams,
                     void *q_out, void *k_out, int64_t qo_ts, int64_t ko_ts, int64_t Hq,
                     int64_t Hk, int64_t D, int64_t rot, int32_t pairing, float eps,
                     const qkr_angle_desc *angle, uint32_t flags, bool norm, bool inplace_ok,
                     int64_t Hv = 0, void *v_out = nullptr, int64_t vo_ts = 0,
                     bool k_only = false, const int64_t *k_rows = nullptr,
                     int64_t k_out_rows = 0)
{
    // k_only: K-only scatter (rope_set_rows): no Q heads, K row n goes to
    // output row k_rows[n] of a k_out buffer with k_out_rows rows.
    qkr_status st = check_geometry(Hq, Hk, D, rot, pairing, eps, k_only);
    if (st != QKR_OK)
        return st;
    if (k_only && (Hq != 0 || Hv != 0 || k_out_rows < 1 || k_out_rows > ((int64_t)1 << 40)))
        return fail(QKR_ERR_INVALID_ARG, "scatter: need Hq == 0, no V and 1 <= cache rows");
    if (k_only && (reinterpret_cast<uintptr_t>(k_rows) & 7u))
        return fail(QKR_ERR_UNSUPPORTED, "row indices must be 8-byte aligned");
    if (Hv < 0 || Hq + Hk + Hv > 65536)
        return fail(QKR_ERR_INVALID_ARG, "V head count out of range");
    if (!streams || n_streams < 1 || n_streams > 2)
        return fail(QKR_ERR_INVALID_ARG, "need 1 or 2 stream descriptors");
    if (flags & ~(uint32_t)(QKR_FLAG_ROUND_NORMALIZED_BF16 | QKR_FLAG_EAGER_ROUNDING |
                            QKR_FLAG_INDEPENDENT))
        return fail(QKR_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
    if ((flags & QKR_FLAG_ROUND_NORMALIZED_BF16) && (flags & QKR_FLAG_EAGER_ROUNDING))
        return fail(QKR_ERR_INVALID_ARG, "one rounding contract at a time: ROUND_NORMALIZED_BF16 "
                                         "or EAGER_ROUNDING");
    if (!norm && (flags & (QKR_FLAG_ROUND_NORMALIZED_BF16 | QKR_FLAG_EAGER_ROUNDING)))
        return fail(QKR_ERR_INVALID_ARG, "the rounding contracts need normalisation (gammas)");
    int64_t T_all = 0;
    for (int s = 0; s < n_streams; ++s) {
        if (streams[s].n_tokens < 0 || streams[s].n_tokens > ((int64_t)1 << 40))
            return fail(QKR_ERR_INVALID_ARG, "stream %d: token count out of range", s);
        T_all += streams[s].n_tokens;
    }
    if (T_all == 0) {  // nothing to do: enqueue nothing
        g_last = qkr::LaunchRecord();
        g_error.clear();
        return QKR_OK;
    }
    if ((Hq > 0 && !q_out) || !k_out)
        return fail(QKR_ERR_INVALID_ARG, "q_out and k_out must be non-NULL");
    if ((Hq > 0 && !aligned16(q_out)) || !aligned16(k_out))
        return fail(QKR_ERR_UNSUPPORTED, "outputs must be 16-byte aligned");
    if ((Hq > 0 && (qo_ts < Hq * D || qo_ts % 8)) || ko_ts < Hk * D || ko_ts % 8)
        return fail(QKR_ERR_UNSUPPORTED,
                    "output token strides must be multiples of 8 and hold a token's heads");
    if (Hv > 0) {
        if (!v_out)
            return fail(QKR_ERR_INVALID_ARG, "v_out must be non-NULL");
        if (!aligned16(v_out))
            return fail(QKR_ERR_UNSUPPORTED, "v_out must be 16-byte aligned");
        if (vo_ts < Hv * D || vo_ts % 8)
            return fail(QKR_ERR_UNSUPPORTED,
                        "v_out token stride must be a multiple of 8 and hold a token's heads");
    }

    qkr::RopeParams p = {};
    int64_t T = 0;
    const __nv_bfloat16 *qb[2] = {nullptr, nullptr}, *kb[2] = {nullptr, nullptr},
                        *vb[2] = {nullptr, nullptr};
    for (int s = 0; s < n_streams; ++s) {
        const qkr_stream_desc &d = streams[s];
        if (d.n_tokens < 0)
            return fail(QKR_ERR_INVALID_ARG, "stream %d: negative token count", s);
        if (d.n_tokens == 0) {
            qb[s] = kb[s] = nullptr;
            p.st[s] = qkr::RopeStreamDev{};
            continue;
        }
        qkr_stream_desc dd = d;
        if (Hq == 0) {  // K-only call: Q is never read
            dd.q = d.k;
            dd.q_offset = d.k_offset;
            dd.q_tok_stride = d.k_tok_stride;
            dd.q_head_stride = d.k_head_stride;
        }
        if (!dd.q || !d.k)
            return fail(QKR_ERR_INVALID_ARG, "stream %d: q and k must be non-NULL", s);
        if (dd.q_offset < 0 || d.k_offset < 0)
            return fail(QKR_ERR_INVALID_ARG, "stream %d: storage offsets must be >= 0", s);
        if (dd.q_tok_stride <= 0 || d.k_tok_stride <= 0 || dd.q_head_stride < D ||
            d.k_head_stride < D)
            return fail(QKR_ERR_UNSUPPORTED,
                        "stream %d: strides must be positive and heads must not overlap", s);
        if (dd.q_tok_stride % 8 || d.k_tok_stride % 8 || dd.q_head_stride % 8 ||
            d.k_head_stride % 8 || dd.q_offset % 8 || d.k_offset % 8)
            return fail(QKR_ERR_UNSUPPORTED,
                        "stream %d: offsets and strides must be multiples of 8 elements "
                        "(16-byte vectors)", s);
        if (!view_fits(d.n_tokens, dd.q_tok_stride, Hq, dd.q_head_stride, D) ||
            !view_fits(d.n_tokens, d.k_tok_stride, Hk, d.k_head_stride, D) ||
            dd.q_offset > ((int64_t)1 << 60) || d.k_offset > ((int64_t)1 << 60))
            return fail(QKR_ERR_INVALID_ARG, "stream %d: view exceeds the address range", s);
        qb[s] = static_cast<const __nv_bfloat16 *>(dd.q) + dd.q_offset;
        kb[s] = static_cast<const __nv_bfloat16 *>(d.k) + d.k_offset;
        if (!aligned16(qb[s]) || !aligned16(kb[s]))
            return fail(QKR_ERR_UNSUPPORTED, "stream %d: q/k must be 16-byte aligned", s);
        if (norm) {
            if ((Hq > 0 && !d.gamma_q) || !d.gamma_k)
                return fail(QKR_ERR_INVALID_ARG, "stream %d: gamma_q and gamma_k are required",
                            s);
            if ((Hq > 0 && !aligned16(d.gamma_q)) || !aligned16(d.gamma_k))
                return fail(QKR_ERR_UNSUPPORTED, "stream %d: gammas must be 16-byte aligned", s);
        }
        p.st[s].q = qb[s];
        p.st[s].k = kb[s];
        p.st[s].q_ts = dd.q_tok_stride;
        p.st[s].q_hs = dd.q_head_stride;
        p.st[s].k_ts = d.k_tok_stride;
        p.st[s].k_hs = d.k_head_stride;
        p.st[s].gq = static_cast<const __nv_bfloat16 *>(d.gamma_q);
        p.st[s].gk = static_cast<const __nv_bfloat16 *>(d.gamma_k);
        if (Hv > 0) {
            if (!d.v)
                return fail(QKR_ERR_INVALID_ARG, "stream %d: v must be non-NULL", s);
            if (d.v_offset < 0 || d.v_offset > ((int64_t)1 << 60))
                return fail(QKR_ERR_INVALID_ARG, "stream %d: v storage offset out of range", s);
            if (d.v_tok_stride <= 0 || d.v_head_stride < D)
                return fail(QKR_ERR_UNSUPPORTED,
                            "stream %d: v strides must be positive and heads must not overlap",
                            s);
            if (d.v_tok_stride % 8 || d.v_head_stride % 8 || d.v_offset % 8)
                return fail(QKR_ERR_UNSUPPORTED,
                            "stream %d: v offset and strides must be multiples of 8 elements", s);
            if (!view_fits(d.n_tokens, d.v_tok_stride, Hv, d.v_head_stride, D))
                return fail(QKR_ERR_INVALID_ARG, "stream %d: v view exceeds the address range",
                            s);
            vb[s] = static_cast<const __nv_bfloat16 *>(d.v) + d.v_offset;
            if (!aligned16(vb[s]))
                return fail(QKR_ERR_UNSUPPORTED, "stream %d: v must be 16-byte aligned", s);
            p.st[s].v = vb[s];
            p.st[s].v_ts = d.v_tok_stride;
            p.st[s].v_hs = d.v_head_stride;
        }
        T += d.n_tokens;
    }
    if (T > ((int64_t)1 << 40))
        return fail(QKR_ERR_INVALID_ARG, "token count too large");
    if (T > INT32_MAX)
        return fail(QKR_ERR_UNSUPPORTED,
                    "%lld tokens in one launch: the kernels take at most 2^31 - 1; split the "
                    "call into chunks with a token offset", (long long)T);
    const int64_t k_rows_out = k_only ? k_out_rows : T;
    if (!view_fits(T, qo_ts, 1, 0, Hq * D) || !view_fits(k_rows_out, ko_ts, 1, 0, Hk * D))
        return fail(QKR_ERR_INVALID_ARG, "output view exceeds the address range");

    // Aliasing: outputs may equal inputs only where allowed (exact in-place),
    // and must share no element with any other view.
    const View vo_q{q_out, T, qo_ts, Hq, D, D};
    const View vo_k{k_out, k_rows_out, ko_ts, Hk, D, D};
    if (!views_disjoint(vo_q, vo_k))
        return fail(QKR_ERR_UNSUPPORTED, "q_out and k_out overlap");
    View vo_v;
    if (Hv > 0) {
        if (!view_fits(T, vo_ts, 1, 0, Hv * D))
            return fail(QKR_ERR_INVALID_ARG, "v_out view exceeds the address range");
        vo_v = View{v_out, T, vo_ts, Hv, D, D};
        if (!views_disjoint(vo_v, vo_q) || !views_disjoint(vo_v, vo_k))
            return fail(QKR_ERR_UNSUPPORTED, "v_out overlaps q_out or k_out");
    }
    for (int s = 0; s < n_streams; ++s) {
        const qkr_stream_desc &d = streams[s];
        if (d.n_tokens == 0)
            continue;
        const View vi_q{qb[s], d.n_tokens, d.q_tok_stride, Hq, d.q_head_stride, D};
        const View vi_k{kb[s], d.n_tokens, d.k_tok_stride, Hk, d.k_head_stride, D};
        const bool q_same = inplace_ok && n_streams == 1 && qb[s] == q_out &&
                            d.q_tok_stride == qo_ts && d.q_head_stride == D;
        const bool k_same = inplace_ok && n_streams == 1 && kb[s] == k_out &&
                            d.k_tok_stride == ko_ts && d.k_head_stride == D;
        if ((!views_disjoint(vo_q, vi_q) && !q_same) || !views_disjoint(vo_q, vi_k) ||
            (!views_disjoint(vo_k, vi_k) && !k_same) || !views_disjoint(vo_k, vi_q))
            return fail(QKR_ERR_UNSUPPORTED,
                        inplace_ok ? "outputs overlap inputs (only exact in-place is allowed)"
                                   : "outputs must not overlap the inputs (fresh outputs)");
        if (Hv > 0) {
            const View vi_v{vb[s], d.n_tokens, d.v_tok_stride, Hv, d.v_head_stride, D};
            if (!views_disjoint(vo_v, vi_q) || !views_disjoint(vo_v, vi_k) ||
                !views_disjoint(vo_v, vi_v) || !views_disjoint(vo_q, vi_v) ||
                !views_disjoint(vo_k, vi_v))
                return fail(QKR_ERR_UNSUPPORTED,
                            "outputs must not overlap the inputs (fresh outputs)");
        }
    }

    const int64_t P = rot / 2;
    st = check_angle(angle, P, T, p);
    if (st != QKR_OK)
        return st;

    p.split = n_streams == 2 ? streams[0].n_tokens : INT64_MAX;
    if (n_streams == 2 && streams[0].n_tokens == 0)
        p.split = 0;
    p.q_out = static_cast<__nv_bfloat16 *>(q_out);
    p.k_out = static_cast<__nv_bfloat16 *>(k_out);
    p.v_out = static_cast<__nv_bfloat16 *>(v_out);
    p.qo_ts = qo_ts;
    p.ko_ts = ko_ts;
    p.vo_ts = vo_ts;
    p.Hv = (int)Hv;
    p.T = T;
    p.Hq = (int)Hq;
    p.Hk = (int)Hk;
    p.D = (int)D;
    p.rot = (int)rot;
    p.P = (int)P;
    p.rows_per_token = (int)(Hq + Hk + Hv);
    p.k_rows = k_rows;
    p.k_out_rows = k_only ? k_out_rows : 0;
    if (k_only) {
        cudaError_t se = qkr::device_status_address(&p.status);
        if (se != cudaSuccess)
            return cuda_result(se, "device status address");
    }
    p.eps = eps;
    p.inv_D = 1.0f / (float)D;
    p.norm = norm ? 1 : 0;
    p.independent = (flags & QKR_FLAG_INDEPENDENT) ? 1 : 0;
    p.round_norm = (flags & QKR_FLAG_EAGER_ROUNDING)          ? 2   // kRoundEager
                 : (flags & QKR_FLAG_ROUND_NORMALIZED_BF16) ? 1   // kRoundNormalized
                                                            : 0;

    qkr::LaunchRecord rec;
    cudaError_t e = qkr::launch_rope_rows(p, pairing, static_cast<cudaStream_t>(stream), &rec);
    qkr_status r = cuda_result(e, "rope kernel launch");
    if (r == QKR_OK)
        g_last = rec;
    return r;
}

}  // namespace

extern "C" {

const char *qkr_last_error(void) { return g_error.c_str(); }

const char *qkr_version(void) { return "qkr 0.1.0 (sm_100a)"; }

qkr_status qkr_last_launch(qkr_launch_info *info)
{
    if (!info)
        return fail(QKR_ERR_INVALID_ARG, "info is NULL");
    info->kernel = g_last.kernel;
    info->lanes_per_row = g_last.lanes_per_row;
    info->slots = g_last.slots;
    info->tokens_per_cta = g_last.tokens_per_cta;
    info->heads_per_item = g_last.heads_per_item;
    info->pipelined = g_last.pipelined;
    info->cluster = g_last.cluster;
    info->block = g_last.block;
    info->direct_angles = g_last.direct_angles;
    info->overlap = g_last.launches > 0 ? qkr::launch_overlap() : 0;
    info->stages = g_last.stages;
    info->reserved = 0;
    info->grid = g_last.grid;
    info->launches = g_last.launches;
    return QKR_OK;
}

qkr_status qkr_launch_overlap(int32_t enable)
{
    if (enable != 0 && enable != 1)
        return fail(QKR_ERR_INVALID_ARG, "enable must be 0 or 1");
    qkr::set_launch_overlap(enable);
    g_error.clear();
    return QKR_OK;
}

qkr_status qkr_tune_rms(int32_t cluster, int32_t threads)
{
    if (cluster != 0 && cluster != 1 && cluster != 2 && cluster != 4 && cluster != 8 &&
        cluster != 16)
        return fail(QKR_ERR_INVALID_ARG, "cluster must be 0 or a power of two up to 16");
    if (threads != 0 && (threads < 32 || threads > 1024 || threads % 32))
        return fail(QKR_ERR_INVALID_ARG, "threads must be 0 or a multiple of 32 in [32, 1024]");
    qkr::set_rms_cluster_override(cluster, threads);
    g_error.clear();
    return QKR_OK;
}

qkr_status qkr_tune_rope_lanes(int32_t lanes)
{
    if (lanes != 0 && lanes != 1 && lanes != 2 && lanes != 4 && lanes != 8 && lanes != 16)
        return fail(QKR_ERR_INVALID_ARG, "lanes must be 0 or a power of two up to 16");
    qkr::set_rope_lanes_override(lanes);
    g_error.clear();
    return QKR_OK;
}

qkr_status qkr_tune_rope(int32_t pipeline, int32_t heads_per_item, int32_t tokens_per_cta,
                         int32_t stages)
{
    if ((pipeline != 0 && pipeline != 1 && pipeline != 3) || heads_per_item < 0 ||
        (heads_per_item > 4 && heads_per_item != 6) || tokens_per_cta < 0 ||
        tokens_per_cta > 64 || stages < 0 || stages > 4)
        return fail(QKR_ERR_INVALID_ARG,
                    "pipeline 0, 1 or 3, heads_per_item in [0, 4] or 6, tokens_per_cta in "
                    "[0, 64], stages in [0, 4]");
    qkr::set_rope_shape_override(pipeline, heads_per_item, tokens_per_cta, stages);
    g_error.clear();
    return QKR_OK;
}

qkr_status qkr_null_launch(void *stream, int64_t grid, int32_t block)
{
    if (grid < 1 || grid > INT32_MAX || block < 32 || block > 1024 || block % 32)
        return fail(QKR_ERR_INVALID_ARG, "grid in [1, 2^31), block a multiple of 32 in [32, 1024]");
    qkr::LaunchRecord rec;
    qkr_status r = cuda_result(qkr::launch_null(grid, block, static_cast<cudaStream_t>(stream),
                                                &rec),
                               "null kernel launch");
    if (r == QKR_OK)
        g_last = rec;
    return r;
}

qkr_status qkr_device_status(uint32_t *status, int32_t reset)
{
    if (!status)
        return fail(QKR_ERR_INVALID_ARG, "status is NULL");
    unsigned v = 0;
    qkr_status r = cuda_result(qkr::read_device_status(&v, reset != 0), "device status read");
    *status = v;
    return r;
}

qkr_status fused_qk_norm_rope(void *stream, const qkr_stream_desc *streams, int32_t n_streams,
                              void *q_out, void *k_out, int64_t q_out_tok_stride,
                              int64_t k_out_tok_stride, int64_t Hq, int64_t Hk, int64_t D,
                              int64_t rot_dim, int32_t pairing, float eps,
                              const qkr_angle_desc *angle, uint32_t flags)
{
    return rope_call(stream, streams, n_streams, q_out, k_out, q_out_tok_stride,
                     k_out_tok_stride, Hq, Hk, D, rot_dim, pairing, eps, angle, flags,
                     /*norm=*/true, /*inplace_ok=*/false);
}

qkr_status fused_qkv_norm_rope(void *stream, const qkr_stream_desc *streams, int32_t n_streams,
                               void *q_out, void *k_out, void *v_out, int64_t q_out_tok_stride,
                               int64_t k_out_tok_stride, int64_t v_out_tok_stride, int64_t Hq,
                               int64_t Hk, int64_t Hv, int64_t D, int64_t rot_dim,
                               int32_t pairing, float eps, const qkr_angle_desc *angle,
                               uint32_t flags)
{
    if (Hv < 1)
        return fail(QKR_ERR_INVALID_ARG, "Hv must be >= 1 (use fused_qk_norm_rope without V)");
    return rope_call(stream, streams, n_streams, q_out, k_out, q_out_tok_stride,
                     k_out_tok_stride, Hq, Hk, D, rot_dim, pairing, eps, angle, flags,
                     /*norm=*/true, /*inplace_ok=*/false, Hv, v_out, v_out_tok_stride);
}

qkr_status mrope_apply(void *stream, const void *q, const void *k, void *q_out, void *k_out,
                       int64_t T, int64_t Hq, int64_t Hkv, int64_t D, int64_t rot_dim,
                       int64_t q_tok_stride, int64_t k_tok_stride, int64_t q_out_tok_stride,
                       int64_t k_out_tok_stride, const int32_t *positions, int64_t n_rows,
                       int64_t T_total, int64_t token_offset, const float *inv_freq,
                       const int32_t *sections, int32_t section_mode, int32_t pairing,
                       const void *gamma_q, const void *gamma_k, float eps, uint32_t flags)
{
    if ((gamma_q == nullptr) != (gamma_k == nullptr))
        return fail(QKR_ERR_INVALID_ARG, "gamma_q and gamma_k must be both set or both NULL");
    const bool norm = gamma_q != nullptr;
    if (!norm && (flags & (QKR_FLAG_ROUND_NORMALIZED_BF16 | QKR_FLAG_EAGER_ROUNDING)))
        return fail(QKR_ERR_INVALID_ARG, "the rounding contracts need normalisation (gammas)");
    if (section_mode < QKR_SECTIONS_NONE || section_mode > QKR_SECTIONS_IMROPE)
        return fail(QKR_ERR_INVALID_ARG, "unknown section mode %d", section_mode);
    if (rot_dim > 0 && n_rows != rows_for_mode(section_mode))
        return fail(QKR_ERR_INVALID_ARG, "section mode %d reads %d position rows, got %lld",
                    section_mode, rows_for_mode(section_mode), (long long)n_rows);
    qkr_stream_desc d = {};
    d.q = q;
    d.k = k;
    d.q_tok_stride = q_tok_stride;
    d.q_head_stride = D;
    d.k_tok_stride = k_tok_stride;
    d.k_head_stride = D;
    d.n_tokens = T;
    d.gamma_q = gamma_q;
    d.gamma_k = gamma_k;
    qkr_angle_desc a = {};
    a.kind = QKR_ANGLE_POSITIONS;
    a.section_mode = section_mode;
    if (sections)
        for (int i = 0; i < 4; ++i)
            a.sections[i] = sections[i];
    a.positions = positions;
    a.pos_row_stride = T_total;
    a.inv_freq = inv_freq;
    a.token_offset = token_offset;
    if (section_mode != QKR_SECTIONS_NONE && !sections)
        return fail(QKR_ERR_INVALID_ARG,
                    "section mode %d needs its sections: refusing rather than rotating every "
                    "pair by one row", section_mode);
    return rope_call(stream, &d, 1, q_out, k_out, q_out_tok_stride, k_out_tok_stride, Hq, Hkv,
                     D, rot_dim, pairing, eps, &a, flags, norm, /*inplace_ok=*/true);
}

static qkr_status vit_common(const int32_t *cu, const int32_t *grids, int64_t G, int64_t N,
                             int64_t m, qkr::VitParams &p)
{
    if (G < 0 || N < 0)
        return fail(QKR_ERR_INVALID_ARG, "G and N must be >= 0");
    if (G > (1 << 24) || N > ((int64_t)1 << 40))
        return fail(QKR_ERR_INVALID_ARG, "G or N too large");
    if (G == 0 && N != 0)
        return fail(QKR_ERR_INVALID_ARG, "N = %lld tokens with no grids", (long long)N);
    if (m < 1 || m > 64)
        return fail(QKR_ERR_INVALID_ARG, "spatial_merge must be in [1, 64]");
    if (N > 0 && (!cu || !grids))
        return fail(QKR_ERR_INVALID_ARG, "cu_seqlens and grids must be non-NULL");
    if (N > 0 && (!aligned4(cu) || !aligned4(grids)))
        return fail(QKR_ERR_UNSUPPORTED, "cu_seqlens / grids must be 4-byte aligned");
    p.cu = cu;
    p.grids = grids;
    p.G = (int)G;
    p.N = N;
    p.m = (int)m;
    return QKR_OK;
}

qkr_status rope_set_rows(void *stream, const void *x, void *cache, const int64_t *row_idx,
                         int64_t T, int64_t H, int64_t D, int64_t rot_dim, int64_t x_tok_stride,
                         int64_t cache_row_stride, int64_t cache_rows, const int32_t *positions,
                         int64_t n_rows, int64_t T_total, int64_t token_offset,
                         const float *inv_freq, const int32_t *sections, int32_t section_mode,
                         int32_t pairing, const void *gamma, float eps, uint32_t flags)
{
    const bool norm = gamma != nullptr;
    if (!norm && (flags & (QKR_FLAG_ROUND_NORMALIZED_BF16 | QKR_FLAG_EAGER_ROUNDING)))
        return fail(QKR_ERR_INVALID_ARG, "the rounding contracts need normalisation (gamma)");
    if (section_mode < QKR_SECTIONS_NONE || section_mode > QKR_SECTIONS_IMROPE)
        return fail(QKR_ERR_INVALID_ARG, "unknown section mode %d", section_mode);
    if (rot_dim > 0 && n_rows != rows_for_mode(section_mode))
        return fail(QKR_ERR_INVALID_ARG, "section mode %d reads %d position rows, got %lld",
                    section_mode, rows_for_mode(section_mode), (long long)n_rows);
    if (section_mode != QKR_SECTIONS_NONE && !sections)
        return fail(QKR_ERR_INVALID_ARG,
                    "section mode %d needs its sections: refusing rather than rotating every "
                    "pair by one row", section_mode);
    if (T > 0 && !row_idx)
        return fail(QKR_ERR_INVALID_ARG, "row_idx must be non-NULL");
    qkr_stream_desc d = {};
    d.k = x;
    d.k_tok_stride = x_tok_stride;
    d.k_head_stride = D;
    d.n_tokens = T;
    d.gamma_k = gamma;
    qkr_angle_desc a = {};
    a.kind = QKR_ANGLE_POSITIONS;
    a.section_mode = section_mode;
    if (sections)
        for (int i = 0; i < 4; ++i)
            a.sections[i] = sections[i];
    a.positions = positions;
    a.pos_row_stride = T_total;
    a.inv_freq = inv_freq;
    a.token_offset = token_offset;
    return rope_call(stream, &d, 1, nullptr, cache, 0, cache_row_stride, 0, H, D, rot_dim,
                     pairing, eps, &a, flags, norm, /*inplace_ok=*/false, 0, nullptr, 0,
                     /*k_only=*/true, row_idx, cache_rows);
}

qkr_status vit_mrope_setup(void *stream, const float *inv_t, const float *inv_h,
                           const float *inv_w, int64_t half_t, int64_t half_h, int64_t half_w,
                           const int32_t *cu_seqlens, const int32_t *grids, int64_t G, int64_t N,
                           int64_t spatial_merge, float *cos_out, float *sin_out)
{
    qkr::VitParams p = {};
    qkr_status st = vit_common(cu_seqlens, grids, G, N, spatial_merge, p);
    if (st != QKR_OK)
        return st;
    if (half_t < 0 || half_h < 0 || half_w < 0 || half_t + half_h + half_w < 1 ||
        half_t + half_h + half_w > 4096)
        return fail(QKR_ERR_INVALID_ARG, "per-axis lengths must be >= 0 and sum to [1, 4096]");
    if ((half_t && !inv_t) || (half_h && !inv_h) || (half_w && !inv_w))
        return fail(QKR_ERR_INVALID_ARG, "inv_freq of a non-empty axis is NULL");
    if (N > 0 && (!cos_out || !sin_out))
        return fail(QKR_ERR_INVALID_ARG, "cos_out and sin_out must be non-NULL");
    if (!aligned4(cos_out) || !aligned4(sin_out) || !aligned4(inv_t) || !aligned4(inv_h) ||
        !aligned4(inv_w))
        return fail(QKR_ERR_UNSUPPORTED, "fp32 buffers must be 4-byte aligned");
    p.inv[0] = inv_t;
    p.inv[1] = inv_h;
    p.inv[2] = inv_w;
    p.half[0] = (int)half_t;
    p.half[1] = (int)half_h;
    p.half[2] = (int)half_w;
    p.P = (int)(half_t + half_h + half_w);
    p.cos_out = cos_out;
    p.sin_out = sin_out;
    if (N == 0) {
        g_last = qkr::LaunchRecord();
        g_error.clear();
        return QKR_OK;
    }
    qkr::LaunchRecord rec;
    qkr_status r = cuda_result(qkr::launch_vit_setup(p, static_cast<cudaStream_t>(stream), &rec),
                               "vit setup launch");
    if (r == QKR_OK)
        g_last = rec;
    return r;
}

qkr_status rms_norm_residual(void *stream, const void *x, void *residual, const void *gamma,
                             void *out, int64_t R, int64_t hidden, int64_t x_stride,
                             int64_t res_stride, int64_t out_stride, float eps)
{
    if (R < 0)
        return fail(QKR_ERR_INVALID_ARG, "R must be >= 0");
    if (hidden < 8 || hidden > 65536 || hidden % 8)
        return fail(QKR_ERR_UNSUPPORTED, "hidden %lld: need a multiple of 8 in [8, 65536]",
                    (long long)hidden);
    if (!(eps >= 0.f) || eps > 1.f)
        return fail(QKR_ERR_INVALID_ARG, "eps must be finite and in [0, 1]");
    if (R == 0) {
        g_last = qkr::LaunchRecord();
        g_error.clear();
        return QKR_OK;
    }
    if (R > ((int64_t)1 << 31) - 1)
        return fail(QKR_ERR_INVALID_ARG, "too many rows");
    if (!x || !residual || !gamma || !out)
        return fail(QKR_ERR_INVALID_ARG, "x, residual, gamma and out must be non-NULL");
    if (!aligned16(x) || !aligned16(residual) || !aligned16(gamma) || !aligned16(out))
        return fail(QKR_ERR_UNSUPPORTED, "pointers must be 16-byte aligned");
    if (x_stride < hidden || res_stride < hidden || out_stride < hidden || x_stride % 8 ||
        res_stride % 8 || out_stride % 8)
        return fail(QKR_ERR_UNSUPPORTED,
                    "row strides must be >= hidden and multiples of 8 elements");
    if (!view_fits(R, x_stride, 1, 0, hidden) || !view_fits(R, res_stride, 1, 0, hidden) ||
        !view_fits(R, out_stride, 1, 0, hidden))
        return fail(QKR_ERR_INVALID_ARG, "view exceeds the address range");
    const Span sx = view_span(x, R, x_stride, 1, 0, hidden);
    const Span sr = view_span(residual, R, res_stride, 1, 0, hidden);
    const Span so = view_span(out, R, out_stride, 1, 0, hidden);
    if (overlap(sr, so) || overlap(sr, sx))
        return fail(QKR_ERR_UNSUPPORTED, "residual must not overlap x or out");
    if (overlap(sx, so) && !(x == out && x_stride == out_stride))
        return fail(QKR_ERR_UNSUPPORTED, "out may only alias x exactly (same stride)");
    qkr::RmsParams p = {};
    p.x = static_cast<const __nv_bfloat16 *>(x);
    p.res = static_cast<__nv_bfloat16 *>(residual);
    p.gamma = static_cast<const __nv_bfloat16 *>(gamma);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.R = R;
    p.hidden = (int)hidden;
    p.xs = x_stride;
    p.rs = res_stride;
    p.os = out_stride;
    p.eps = eps;
    p.inv_hidden = 1.0f / (float)hidden;
    qkr::LaunchRecord rec;
    qkr_status r = cuda_result(
        qkr::launch_rms_norm_residual(p, static_cast<cudaStream_t>(stream), &rec),
        "rms norm launch");
    if (r == QKR_OK)
        g_last = rec;
    return r;
}

qkr_status rms_norm_fp8(void *stream, const void *x, void *residual, const void *gamma,
                        void *out, const float *scale, int64_t R, int64_t hidden,
                        int64_t x_stride, int64_t res_stride, int64_t out_stride, float eps)
{
    if (R < 0)
        return fail(QKR_ERR_INVALID_ARG, "R must be >= 0");
    if (hidden < 8 || hidden > 65536 || hidden % 8)
        return fail(QKR_ERR_UNSUPPORTED, "hidden %lld: need a multiple of 8 in [8, 65536]",
                    (long long)hidden);
    if (!(eps >= 0.f) || eps > 1.f)
        return fail(QKR_ERR_INVALID_ARG, "eps must be finite and in [0, 1]");
    if (R == 0) {
        g_last = qkr::LaunchRecord();
        g_error.clear();
        return QKR_OK;
    }
    if (R > ((int64_t)1 << 31) - 1)
        return fail(QKR_ERR_INVALID_ARG, "too many rows");
    if (!x || !gamma || !out || !scale)
        return fail(QKR_ERR_INVALID_ARG, "x, gamma, out and scale must be non-NULL");
    if (!aligned16(x) || (residual && !aligned16(residual)) || !aligned16(gamma) ||
        (reinterpret_cast<uintptr_t>(out) & 7u) || !aligned4(scale))
        return fail(QKR_ERR_UNSUPPORTED,
                    "x, residual, gamma 16-byte aligned; out 8-byte; scale 4-byte");
    if (x_stride < hidden || x_stride % 8 || out_stride < hidden || out_stride % 8 ||
        (residual && (res_stride < hidden || res_stride % 8)))
        return fail(QKR_ERR_UNSUPPORTED,
                    "row strides must be >= hidden and multiples of 8 elements");
    if (!view_fits(R, x_stride, 1, 0, hidden) || !view_fits(R, out_stride, 1, 0, hidden) ||
        (residual && !view_fits(R, res_stride, 1, 0, hidden)))
        return fail(QKR_ERR_INVALID_ARG, "view exceeds the address range");
    const Span sx = view_span(x, R, x_stride, 1, 0, hidden);
    Span so;  // FP8 rows: one byte per element
    so.lo = reinterpret_cast<uintptr_t>(out);
    so.hi = so.lo + (uintptr_t)((R - 1) * out_stride + hidden);
    const Span ss{reinterpret_cast<uintptr_t>(scale), reinterpret_cast<uintptr_t>(scale) + 4};
    if (overlap(sx, so) || overlap(so, ss))
        return fail(QKR_ERR_UNSUPPORTED, "out must not overlap x or scale");
    if (residual) {
        const Span sr = view_span(residual, R, res_stride, 1, 0, hidden);
        if (overlap(sr, so) || overlap(sr, sx) || overlap(sr, ss))
            return fail(QKR_ERR_UNSUPPORTED, "residual must not overlap x, out or scale");
    }
    qkr::RmsParams p = {};
    p.x = static_cast<const __nv_bfloat16 *>(x);
    p.res = static_cast<__nv_bfloat16 *>(residual);
    p.gamma = static_cast<const __nv_bfloat16 *>(gamma);
    p.out8 = static_cast<uint8_t *>(out);
    p.scale = scale;
    p.R = R;
    p.hidden = (int)hidden;
    p.xs = x_stride;
    p.rs = res_stride;
    p.os = out_stride;
    p.eps = eps;
    p.inv_hidden = 1.0f / (float)hidden;
    qkr::LaunchRecord rec;
    qkr_status r = cuda_result(
        qkr::launch_rms_norm_residual(p, static_cast<cudaStream_t>(stream), &rec),
        "rms norm fp8 launch");
    if (r == QKR_OK)
        g_last = rec;
    return r;
}

qkr_status qkr_section_map(void *stream, int32_t section_mode, const int32_t *sections,
                           int64_t P, int8_t *axis_out)
{
    if (P < 1 || P > 4096)
        return fail(QKR_ERR_INVALID_ARG, "P must be in [1, 4096]");
    if (!axis_out)
        return fail(QKR_ERR_INVALID_ARG, "axis_out is NULL");
    int sec[4];
    qkr_status st = check_sections(section_mode, sections, P, sec);
    if (st != QKR_OK)
        return st;
    qkr::LaunchRecord rec;
    qkr_status r = cuda_result(qkr::launch_section_map(section_mode, sec, (int)P, axis_out,
                                                       static_cast<cudaStream_t>(stream), &rec),
                               "section map launch");
    if (r == QKR_OK)
        g_last = rec;
    return r;
}

qkr_status qkr_vit_positions(void *stream, const int32_t *cu_seqlens, const int32_t *grids,
                             int64_t G, int64_t N, int64_t spatial_merge, int32_t *pos_out)
{
    qkr::VitParams p = {};
    qkr_status st = vit_common(cu_seqlens, grids, G, N, spatial_merge, p);
    if (st != QKR_OK)
        return st;
    if (N > 0 && (!pos_out || !aligned4(pos_out)))
        return fail(QKR_ERR_INVALID_ARG, "pos_out must be a non-NULL 4-byte aligned pointer");
    if (N == 0) {
        g_last = qkr::LaunchRecord();
        g_error.clear();
        return QKR_OK;
    }
    qkr::LaunchRecord rec;
    qkr_status r = cuda_result(
        qkr::launch_vit_positions(p, pos_out, static_cast<cudaStream_t>(stream), &rec),
        "vit positions launch");
    if (r == QKR_OK)
        g_last = rec;
    return r;
}

}  // extern "C"
