/*
 * qkr.h -- C ABI of the B200 (sm_100a) normalise-then-rotate library.
 *
 * The four operations of the path and their extensions, each one CUDA kernel
 * launch on the caller's stream:
 *
 *   fused_qk_norm_rope  per-head RMSNorm of Q and K, optional text/image
 *                       concatenation, RoPE (NeoX or GPT-J pairing), one launch.
 *   fused_qkv_norm_rope the same, with V concatenated (copied unchanged)
 *                       into a joint V output in the same launch.
 *   mrope_apply         multi-section RoPE (contiguous or interleaved
 *                       sections) with a token offset for chunked launches,
 *                       optional per-head RMSNorm.
 *   vit_mrope_setup     fp32 (3, N, P) cos/sin t/h/w planes computed from
 *                       per-image [t, h, w] grids.
 *   rms_norm_residual   hidden-size RMSNorm with a fused residual add; splits
 *                       a wide row across a thread-block cluster when rows are few.
 *   rms_norm_fp8        the same with a static-scale FP8 E4M3 output.
 *   rope_set_rows       mrope_apply's rotation of K rows, scattered into cache
 *                       rows by index.
 *
 * Conventions shared by every entry point:
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - Pointers marked "device" are CUDA device (or managed) memory; pointers
 *     marked "host" are read during the call and may be freed after it returns.
 *   - bf16 tensors are passed as void* to IEEE bfloat16 data; strides and
 *     offsets are in elements, never bytes; all sizes are int64_t.
 *   - The caller owns all memory.  No entry point allocates, frees or
 *     synchronises; each enqueues its work on `stream` and returns.
 *   - Arguments are validated on the host before anything is enqueued.  A
 *     call that cannot be served exactly returns an error; there is no
 *     fallback path and no silent degradation.
 *   - A call with zero tokens (or rows) enqueues nothing and returns QKR_OK.
 *   - Errors: QKR_ERR_INVALID_ARG (bad sizes, null pointers, inconsistent
 *     descriptors), QKR_ERR_UNSUPPORTED (valid but outside what the kernels
 *     serve: alignment, head_dim range, aliasing), QKR_ERR_CUDA (the launch
 *     failed).  qkr_last_error() returns a message for the calling thread's
 *     most recent failure.
 *   - Results are deterministic: fixed launch shape for a given call, no
 *     atomics, fixed reduction order.
 */
#ifndef QKR_H
#define QKR_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qkr_status {
    QKR_OK = 0,
    QKR_ERR_INVALID_ARG = 1,
    QKR_ERR_UNSUPPORTED = 2,
    QKR_ERR_CUDA = 3
} qkr_status;

/* Rotary pairing.  NeoX ("rotate half") pairs dim j with dim j + rot/2;
 * GPT-J ("interleaved") pairs dim 2j with dim 2j+1 (vllm-omni #7600: the
 * single-stream op is called with interleaved=True).  Pair j is rotated by
 * angle theta_j: a' = a cos - b sin, b' = b cos + a sin. */
enum { QKR_PAIRING_NEOX = 0, QKR_PAIRING_GPTJ = 1 };

/* Which position row (t = 0, h = 1, w = 2, e = 3) each rotated pair j < P
 * reads.  sections[] = {s_t, s_h, s_w, s_e}.
 *   NONE                every pair reads row 0 (plain 1-D RoPE).
 *   CONTIGUOUS          pairs [0,s_t) -> t, [s_t, s_t+s_h) -> h, rest -> w
 *                       (vLLM mrope_vit_setup: section columns of the planes).
 *   INTERLEAVED         pair j -> j mod 3 while j < 3*min(s_t,s_h,s_w),
 *                       else the axis of its contiguous section.
 *   INTERLEAVED_QUOTA   same head; each later pair goes to the first axis
 *                       (t, h, w order) whose section count is not used up.
 *   IMROPE              llama.cpp fork #286 sector rule: sector = j mod
 *                       (s_t+s_h+s_w+s_e); sector mod 3 == 1 -> h while
 *                       sector < 3*s_h, == 2 -> w while < 3*s_w, == 0 -> t
 *                       while < 3*s_t, otherwise e.  Needs four rows.
 * Admission (llama.cpp fork #286, review of the claim predicate): for every
 * mode but NONE, each section >= 0 and P <= sum(sections) <= 2P; s_e must be
 * 0 unless the mode is IMROPE. */
enum {
    QKR_SECTIONS_NONE = 0,
    QKR_SECTIONS_CONTIGUOUS = 1,
    QKR_SECTIONS_INTERLEAVED = 2,
    QKR_SECTIONS_INTERLEAVED_QUOTA = 3,
    QKR_SECTIONS_IMROPE = 4
};

/* Where the cos/sin of pair j for a token come from. */
enum {
    /* theta = fp32(pos) * inv_freq[j] (one fp32 multiply), cos/sin by the
     * accurate single-precision sincos; pos = positions[row(j) *
     * pos_row_stride + token_offset + t] (vLLM mrope_vit_setup kernel: fp32
     * position times fp32 inverse frequency). */
    QKR_ANGLE_POSITIONS = 0,
    /* cos/sin read from fp32 tables: element [plane(j)][token_offset + t][j]
     * at plane(j) * plane_stride + (token_offset + t) * ld + j.  With
     * QKR_SECTIONS_NONE this is the single packed table of vllm-omni #7600
     * (one [cos | sin] table per forward); with CONTIGUOUS it reads the
     * (3, N, P) planes written by vit_mrope_setup. */
    QKR_ANGLE_TABLE = 1
};

/* Flags for fused_qk_norm_rope / fused_qkv_norm_rope / mrope_apply /
 * rope_set_rows.  The first two set the rounding points of the normalised
 * value: without either, every intermediate stays in fp32 (gamma folded into
 * the rotation) and only the output is rounded; at most one of them, and
 * either needs the norm. */
enum {
    /* Round the normalised value to bf16 before rotating (the rounding
     * contract of the vllm-omni #7600 Triton tile: bf16-rounded normalised
     * value, fp32 rotation, one final rounding). */
    QKR_FLAG_ROUND_NORMALIZED_BF16 = 1u,
    /* The eager chain's rounding points (vllm-omni #7600, numerics follow-up:
     * a preset that reproduces the unfused RMSNorm and RoPE chain; vLLM
     * #26234 quotes the rms_norm_kernel line that fixes them): the normalised
     * value x r (r = rsqrt(mean(x^2) + eps), fp32) is rounded to bf16, its
     * product with the bf16 gamma is rounded to bf16 again, and the rotation
     * a c - b s, b c + a s takes every product and sum in fp32 without fused
     * multiply-adds; one final rounding.  The rounding points, not bitwise
     * equality with any other implementation: the order of the fp32 sum of
     * squares is this library's. */
    QKR_FLAG_EAGER_ROUNDING = 2u,
    /* A launch-order contract, not a rounding point: the caller declares
     * that this call reads no memory the previous kernel on the stream
     * writes, and writes no memory that kernel reads or writes (the chunks
     * of one chunked step, llama.cpp fork #286, "The change": a launch over
     * part of the tokens).  The kernel then starts its rows while the
     * previous kernel's last CTAs drain (with qkr_launch_overlap on) and
     * waits for that kernel only before it completes, so everything after
     * it on the stream still sees the writes of both.  Results are
     * bit-identical with and without the flag; a call that breaks the
     * contract races with the previous kernel.  Combines with either
     * rounding flag. */
    QKR_FLAG_INDEPENDENT = 4u
};

/* One input stream of fused_qk_norm_rope / fused_qkv_norm_rope.  q, k and v
 * are bf16 device pointers; element (t, h, d) of Q is at q + q_offset +
 * t*q_tok_stride + h*q_head_stride + d (d contiguous), likewise K and V.
 * Offsets may exceed 2^31 elements: all address arithmetic is 64-bit
 * (vllm-omni #7600, 64-bit row addressing for large storage offsets).
 * gamma_q / gamma_k: bf16 [D] device.  The v fields are read only by
 * fused_qkv_norm_rope (zero them otherwise). */
typedef struct qkr_stream_desc {
    const void *q;
    const void *k;
    int64_t q_offset;
    int64_t k_offset;
    int64_t q_tok_stride;
    int64_t q_head_stride;
    int64_t k_tok_stride;
    int64_t k_head_stride;
    int64_t n_tokens;
    const void *gamma_q;
    const void *gamma_k;
    const void *v;
    int64_t v_offset;
    int64_t v_tok_stride;
    int64_t v_head_stride;
} qkr_stream_desc;

/* Angle source (see QKR_ANGLE_*).  Unused fields are ignored.
 *   positions      device int32 [rows, pos_row_stride]; rows = 1 (NONE),
 *                  3 (CONTIGUOUS / INTERLEAVED*), 4 (IMROPE).
 *   pos_row_stride elements between rows = tokens the buffer covers
 *                  (llama.cpp fork #286: a launch over part of the tokens
 *                  indexes the full-length rows from token_offset on).
 *   inv_freq       device fp32 [P], P = rot_dim / 2.
 *   cos, sin       device fp32 tables; table_rows tokens per plane, ld >= P
 *                  elements between token rows, plane_stride elements
 *                  between planes (planes: 1 for NONE, 3 for CONTIGUOUS and
 *                  INTERLEAVED*, 4 for IMROPE).
 *   token_offset   added to the launch-local token index before the
 *                  positions / tables are indexed; token_offset + tokens
 *                  of the launch must not exceed pos_row_stride (table_rows).
 */
typedef struct qkr_angle_desc {
    int32_t kind;
    int32_t section_mode;
    int32_t sections[4];
    const int32_t *positions;
    int64_t pos_row_stride;
    const float *inv_freq;
    const float *cos;
    const float *sin;
    int64_t table_rows;
    int64_t ld;
    int64_t plane_stride;
    int64_t token_offset;
} qkr_angle_desc;

/*
 * fused_qk_norm_rope -- vllm-omni #7600 ("Fuse text/image QK RMSNorm + cat +
 * RoPE into one Triton launch", Purpose and the kernel review): for every
 * token and head, y = x / sqrt(mean(x^2) + eps) * gamma over the head dim
 * (fp32 sum of squares), then RoPE on the first rot_dim dims; dims
 * [rot_dim, D) are normalised only.  With n_streams == 2 the streams are
 * concatenated text first: stream 0's tokens occupy joint rows
 * [0, T0), stream 1's [T0, T0+T1), and the angle of joint row n is that of
 * token token_offset + n.
 *
 *   streams          host array of n_streams (1 or 2) descriptors.
 *   q_out, k_out     bf16 device [T0+T1, Hq, D] and [T0+T1, Hk, D]; row n
 *                    of Q starts at q_out + n*q_out_tok_stride (heads dense).
 *                    Fresh outputs: they must not overlap any input.
 *   D                head dim, a multiple of 8, 8 <= D <= 256.
 *   rot_dim          even, 0 <= rot_dim <= D.
 *   flags            0, QKR_FLAG_ROUND_NORMALIZED_BF16 or QKR_FLAG_EAGER_ROUNDING,
 *                    optionally with QKR_FLAG_INDEPENDENT.
 * Alignment: q/k (after offsets), gammas and outputs 16-byte aligned; all
 * token and head strides multiples of 8 elements (else QKR_ERR_UNSUPPORTED).
 */
qkr_status fused_qk_norm_rope(void *stream, const qkr_stream_desc *streams, int32_t n_streams,
                              void *q_out, void *k_out, int64_t q_out_tok_stride,
                              int64_t k_out_tok_stride, int64_t Hq, int64_t Hk, int64_t D,
                              int64_t rot_dim, int32_t pairing, float eps,
                              const qkr_angle_desc *angle, uint32_t flags);

/*
 * fused_qkv_norm_rope -- the joint Q/K/V form of the same op (vllm-omni #7600,
 * Purpose: the fused joint op takes Q, K and V as zero-copy strided views and
 * writes the concatenated joint Q, K and V in one launch).  Q and K exactly as
 * fused_qk_norm_rope; each stream's V rows are copied bit for bit, text first,
 * into v_out, with no norm and no rotation.
 *
 *   v_out            bf16 device [T0+T1, Hv, D]; row n starts at
 *                    v_out + n*v_out_tok_stride (heads dense).  Fresh: must
 *                    not overlap any input or the other outputs.
 *   Hv               V heads per token, >= 1 (V shares D with Q and K).
 * Every stream with tokens needs v (and its strides, same rules as q / k).
 * Errors, alignment and the remaining arguments as fused_qk_norm_rope.
 */
qkr_status fused_qkv_norm_rope(void *stream, const qkr_stream_desc *streams, int32_t n_streams,
                               void *q_out, void *k_out, void *v_out, int64_t q_out_tok_stride,
                               int64_t k_out_tok_stride, int64_t v_out_tok_stride, int64_t Hq,
                               int64_t Hk, int64_t Hv, int64_t D, int64_t rot_dim,
                               int32_t pairing, float eps, const qkr_angle_desc *angle,
                               uint32_t flags);

/*
 * mrope_apply -- multi-section RoPE (llama.cpp fork #286, "The change":
 * the section a pair falls in picks the position row its angle comes from;
 * a launch over part of the tokens indexes the full-length position rows from
 * its first token).  Rotates Q [T, Hq, D] and K [T, Hkv, D] (heads dense, token
 * strides given) with angles from positions + inv_freq, pair j reading row
 * section(j) at column token_offset + t.  If gamma_q and gamma_k are both
 * non-NULL each head is RMS-normalised first (as fused_qk_norm_rope); both
 * NULL means no normalisation; one NULL is an error.
 *
 *   q, k             bf16 device inputs; q_out, k_out bf16 device outputs.
 *                    In-place is allowed: q_out == q with the same token
 *                    stride (likewise k).  Views that share no element are
 *                    accepted even where their byte ranges interleave (Q and
 *                    K as column windows of one packed [T, 3, H, D] buffer
 *                    with one token stride, rotated in place); any other
 *                    overlap is refused.
 *   positions        device int32 [n_rows, T_total]; n_rows must match the
 *                    section mode (1 NONE, 3 sectioned, 4 IMROPE).
 *   token_offset     first token of this launch within positions;
 *                    token_offset + T <= T_total.
 *   inv_freq         device fp32 [rot_dim / 2].
 *   sections         host int32[4] {s_t, s_h, s_w, s_e} (may be NULL for
 *                    QKR_SECTIONS_NONE; NULL with any other mode is an error).
 * Same D / rot_dim / alignment rules as fused_qk_norm_rope.
 */
qkr_status mrope_apply(void *stream, const void *q, const void *k, void *q_out, void *k_out,
                       int64_t T, int64_t Hq, int64_t Hkv, int64_t D, int64_t rot_dim,
                       int64_t q_tok_stride, int64_t k_tok_stride, int64_t q_out_tok_stride,
                       int64_t k_out_tok_stride, const int32_t *positions, int64_t n_rows,
                       int64_t T_total, int64_t token_offset, const float *inv_freq,
                       const int32_t *sections, int32_t section_mode, int32_t pairing,
                       const void *gamma_q, const void *gamma_k, float eps, uint32_t flags);

/*
 * rope_set_rows -- rotate K rows and scatter them into cache rows (llama.cpp
 * fork #286, "The change": the rotation kernels rope_f32 and rope_set_rows_f32
 * both gain the sectioned mode; the second writes each rotated row into the
 * destination row its index names, as ggml's ROPE + SET_ROWS pair does when
 * a decoder stores K in its cache).  For every token t < T and head h:
 *   cache[row_idx[t], h, :] = rope(norm(x[t, h, :]))
 * with exactly mrope_apply's angle rules (positions rows, sections, token
 * offset, pairing) and, when gamma is non-NULL, the per-head RMSNorm first.
 *
 *   x                bf16 device [T, H, D], token stride x_tok_stride, heads dense.
 *   cache            bf16 device [cache_rows, H, D], row stride cache_row_stride
 *                    (a multiple of 8, >= H*D), heads dense.  Must not overlap x.
 *   row_idx          int64 device [T], 8-byte aligned: destination row of each
 *                    token.  Rows must be distinct within a call (two tokens
 *                    naming one row race).  A row outside [0, cache_rows) is
 *                    not written and sets bit 4 of the device status word
 *                    (qkr_device_status); the host cannot see device indices
 *                    without synchronising, so this is reported, not refused.
 *   gamma            nullable bf16 [D].
 * Other arguments, alignment and errors as mrope_apply.
 */
qkr_status rope_set_rows(void *stream, const void *x, void *cache, const int64_t *row_idx,
                         int64_t T, int64_t H, int64_t D, int64_t rot_dim, int64_t x_tok_stride,
                         int64_t cache_row_stride, int64_t cache_rows, const int32_t *positions,
                         int64_t n_rows, int64_t T_total, int64_t token_offset,
                         const float *inv_freq, const int32_t *sections, int32_t section_mode,
                         int32_t pairing, const void *gamma, float eps, uint32_t flags);

/*
 * vit_mrope_setup -- vLLM mrope_vit_setup (VitMropeSetup.forward and
 * _vit_mrope_setup_kernel): the (3, N, P) fp32 cos/sin t/h/w planes,
 * P = half_t + half_h + half_w.  Token n of grid g (cu_seqlens[g] <= n <
 * cu_seqlens[g+1], grid [t, h, w]) has local index l = n - cu_seqlens[g];
 * frames hold h*w tokens ordered by spatial-merge block: merge-block row,
 * merge-block column, then the m x m patch in row-major order, so
 * t_pos = l / (h*w), h_pos = block_row*m + patch_row, w_pos = block_col*m +
 * patch_col.  Plane a holds, in its own section columns only ([0, half_t)
 * for t, [half_t, half_t+half_h) for h, the rest for w),
 * cos/sin(fp32(pos_a) * inv_a[col - offset_a]); other columns are not
 * written.
 *
 *   inv_t/h/w        device fp32 [half_t], [half_h], [half_w].
 *   cu_seqlens       device int32 [G+1], nondecreasing, cu[0] = 0,
 *                    cu[G] = N (the caller uploads it with grids in one copy).
 *   grids            device int32 [G, 3] (t, h, w); h and w multiples of
 *                    spatial_merge (not checked on the device; a violating
 *                    grid yields positions but never an out-of-bounds access).
 *   cos_out, sin_out device fp32 [3, N, P], 4-byte aligned.
 */
qkr_status vit_mrope_setup(void *stream, const float *inv_t, const float *inv_h,
                           const float *inv_w, int64_t half_t, int64_t half_h, int64_t half_w,
                           const int32_t *cu_seqlens, const int32_t *grids, int64_t G, int64_t N,
                           int64_t spatial_merge, float *cos_out, float *sin_out);

/*
 * rms_norm_residual -- hidden-size RMSNorm with fused residual add
 * (vllm.cpp #185, "decode RmsNorm ran on ONE workgroup"; vLLM #26234
 * rms_norm_kernel): per row, s = bf16(x + residual) is written back to
 * residual, then out = s / sqrt(mean(s^2) + eps) * gamma (fp32 sum of
 * squares, one final bf16 rounding).  A row that fits one CTA (hidden <=
 * 8192) is one CTA wide enough to have every 16-byte vector of the row in
 * flight at once; a wider row at decode sizes (up to 32 rows) is split
 * across a thread-block cluster of 8 (up to 16 rows) or 4 CTAs whose partial
 * sums meet in distributed shared memory.
 *
 *   x                bf16 device [R, hidden], row stride x_stride.
 *   residual         bf16 device [R, hidden], in/out, row stride res_stride.
 *   gamma            bf16 device [hidden].
 *   out              bf16 device [R, hidden], row stride out_stride; may be
 *                    x itself (same stride); must not overlap residual.
 *   hidden           multiple of 8, 8 <= hidden <= 65536.
 * Alignment: pointers 16-byte aligned, strides multiples of 8 elements.
 */
qkr_status rms_norm_residual(void *stream, const void *x, void *residual, const void *gamma,
                             void *out, int64_t R, int64_t hidden, int64_t x_stride,
                             int64_t res_stride, int64_t out_stride, float eps);

/*
 * rms_norm_fp8 -- rms_norm_residual with a static FP8 output (vLLM #26234,
 * Purpose: the same vectorised variance read serves rms_norm_kernel and
 * rms_norm_static_fp8_quant_kernel).  With a residual, s = bf16(x + residual)
 * is written back to residual as in rms_norm_residual; without one
 * (residual == NULL) s = x.  Then y = s * rsqrt(mean(s^2) + eps) * gamma in
 * fp32, and out holds the FP8 E4M3 (OCP "FN": no infinities, max 448) code of
 * y / scale (computed as y * fp32(1 / scale)), rounded to nearest even and
 * saturated to +-448.
 *
 *   out              device uint8 [R, hidden] E4M3 codes, row stride out_stride
 *                    bytes (a multiple of 8), 8-byte aligned.
 *   scale            device fp32 [1]: the static per-tensor scale (read on the
 *                    device, so the call never synchronises).
 *   residual         nullable; res_stride is ignored when NULL.
 * Other arguments and errors as rms_norm_residual; out must not overlap any input.
 */
qkr_status rms_norm_fp8(void *stream, const void *x, void *residual, const void *gamma,
                        void *out, const float *scale, int64_t R, int64_t hidden,
                        int64_t x_stride, int64_t res_stride, int64_t out_stride, float eps);

/* ------------------------------------------------------------------------
 * Introspection and debug entry points (used by the tests).
 * ------------------------------------------------------------------------ */

/* Message for the calling thread's most recent failed call ("" if none). */
const char *qkr_last_error(void);

/* Library version string. */
const char *qkr_version(void);

/* What the calling thread's most recent successful call enqueued, in the
 * spirit of vllm.cpp #185's dispatch histogram (which kernel, what shape). */
enum {
    QKR_KERNEL_NONE = 0,
    QKR_KERNEL_ROPE_PAIRED = 1,    /* NeoX, rot_dim % 16 == 0: lane holds both halves */
    QKR_KERNEL_ROPE_VECTOR = 2,    /* GPT-J: pairs inside a lane's vector */
    QKR_KERNEL_ROPE_EXCHANGE = 3,  /* NeoX with rot_dim % 16 != 0: shared-memory partner */
    QKR_KERNEL_VIT_SETUP = 4,
    QKR_KERNEL_RMS_ROWS = 5,       /* one CTA per row */
    QKR_KERNEL_RMS_CLUSTER = 6,    /* one cluster per row */
    QKR_KERNEL_SECTION_MAP = 7,
    QKR_KERNEL_VIT_POSITIONS = 8,
    QKR_KERNEL_NULL = 9            /* qkr_null_launch */
};
typedef struct qkr_launch_info {
    int32_t kernel;          /* QKR_KERNEL_* */
    int32_t lanes_per_row;   /* rope kernels: lanes that share one head row */
    int32_t slots;           /* rope: 16-byte vectors per lane per row (NeoX rows of
                                head_dim 64 with staged angles: 1, the lane taking its
                                partner half from another lane); rms: per thread */
    int32_t tokens_per_cta;  /* rope / vit: tokens one CTA covers */
    int32_t heads_per_item;  /* rope: head rows of one token a lane group loads
                                together */
    int32_t pipelined;       /* rope: 0 rows loaded straight into registers (item
                                kernel); 2 rows streamed by every thread into a
                                cp.async ring (streaming kernel) */
    int32_t cluster;         /* rms: CTAs per row (cluster size); else 1 */
    int32_t block;           /* threads per CTA */
    int32_t direct_angles;   /* rope: 1 if each work item read its (cos, sin) straight
                                from the fp32 table (16-byte loads), 0 if the angles
                                were staged per token in shared memory */
    int32_t overlap;         /* 1 if launched with programmatic stream serialisation
                                (see qkr_launch_overlap) */
    int32_t stages;          /* streaming kernel: passes in the row ring; else 0 */
    int32_t reserved;        /* 0 */
    int64_t grid;            /* CTAs launched */
    int64_t launches;        /* kernel launches enqueued (0 for an empty call) */
} qkr_launch_info;
qkr_status qkr_last_launch(qkr_launch_info *info);

/* Programmatic dependent launch for every kernel of this library (default 1).
 * With 1, a kernel is launched with programmatic stream serialisation: it
 * may become resident while the previous kernel of the stream drains, and
 * its first action is a grid-dependency wait that returns once the previous
 * kernel has completed and its writes are visible; stream order therefore
 * holds exactly as without it, and results are bit-identical.  What it saves
 * is the launch gap between back-to-back kernels.  0 launches plainly.
 * Process-wide.  Returns QKR_ERR_INVALID_ARG for other values. */
qkr_status qkr_launch_overlap(int32_t enable);

/* Launch-shape override for the rope kernels, for tuning sweeps.  pipeline:
 * 0 automatic, 1 item kernel (rows straight into registers), 3 streaming
 * kernel (cp.async row ring); calls a forced kernel cannot serve fail with
 * QKR_ERR_CUDA.  heads per work item (1..4, or 6 for GPT-J rows of 128
 * elements with angles from a table whose rows allow 16-byte reads; the
 * streaming kernel takes 1, 2 or 4), tokens per CTA (1..64; kernels that stage angles cap it by their shared
 * memory) and ring depth of the streaming kernel (2..4; 1 counts as 2); 0
 * keeps the automatic choice.  Process-wide; a launch racing a change on
 * another thread takes the old or the new value of each knob.  Every shape
 * computes bit-identical results: a row's arithmetic does not depend on it.
 * Returns QKR_ERR_INVALID_ARG out of range. */
qkr_status qkr_tune_rope(int32_t pipeline, int32_t heads_per_item, int32_t tokens_per_cta,
                         int32_t stages);

/* Lanes sharing one head row in the GPT-J (VECTOR) layout of the rope
 * kernels, for tuning sweeps: 0 automatic, else 1, 2, 4, 8 or 16 (ignored
 * where a lane would need more than two 16-byte vectors of the row).
 * Process-wide.  The lane count sets the order of the fp32 sum of squares
 * (per-lane partial sums, then a shuffle tree), so results can differ in the
 * last bit between choices; each choice is deterministic. */
qkr_status qkr_tune_rope_lanes(int32_t lanes);

/* CTAs that share one row in rms_norm_residual / rms_norm_fp8, and the
 * threads of each CTA, for tuning sweeps.  cluster: 0 automatic, else 1, 2,
 * 4, 8 or 16 (a thread-block cluster when > 1).  threads: 0 automatic, else a
 * multiple of 32 in [32, 1024]: the CTA width the row slice is spread over
 * (each thread keeps its 16-byte vectors of the slice in registers, so a
 * wider CTA holds fewer per thread).  Process-wide.  The split and the width
 * set the order of the fp32 sum of squares, so the normalised output can
 * differ in the last bit between choices; the residual stream is
 * bit-identical. */
qkr_status qkr_tune_rms(int32_t cluster, int32_t threads);

/* Device status word of the library on the current device (0 = healthy).
 * Bit 4: rope_set_rows met a row index outside the cache (that row was not
 * written).  The word is shared by every call of the process on that device,
 * so a bit cannot be traced to the call that raised it; it stays set until a
 * read with reset != 0 clears it.  The read (and the clear) is one atomic
 * exchange on the device, ordered after the work of every blocking stream:
 * a bit raised concurrently by a kernel on a non-blocking stream is returned
 * by this read or by the next, never lost.  Synchronous (copies the word to
 * the host); concurrent reads from several host threads are serialised.  Not
 * for the hot path. */
qkr_status qkr_device_status(uint32_t *status, int32_t reset);

/* The launch floor, for measurement: enqueues one kernel of `grid` CTAs of
 * `block` threads (a multiple of 32, at most 1024) that does nothing but the
 * programmatic-launch wait and trigger every library kernel begins with,
 * launched with the same attributes (qkr_launch_overlap).  Back-to-back
 * launches of it show the per-launch cost no kernel of this library can go
 * below (vllm.cpp #185 measures its decode RMSNorm per call; a call that
 * moves kilobytes costs what a launch costs).  Touches no memory. */
qkr_status qkr_null_launch(void *stream, int64_t grid, int32_t block);

/* Writes the axis (0 t, 1 h, 2 w, 3 e) of pairs 0..P-1 under a section mode
 * to axis_out (device int8 [P]) with the kernels' own section rule.
 * sections: host int32[4].  Same admission rules as mrope_apply. */
qkr_status qkr_section_map(void *stream, int32_t section_mode, const int32_t *sections,
                           int64_t P, int8_t *axis_out);

/* Writes the (t, h, w) position of every token to pos_out (device int32
 * [3, N]) with vit_mrope_setup's own grid-to-position mapping. */
qkr_status qkr_vit_positions(void *stream, const int32_t *cu_seqlens, const int32_t *grids,
                             int64_t G, int64_t N, int64_t spatial_merge, int32_t *pos_out);

#ifdef __cplusplus
}
#endif

#endif /* QKR_H */
