"""Python binding of libqkr.so (include/qkr.h) -- argument marshalling only.

Every function here takes torch tensors already on a CUDA device, checks
their dtype/device, passes raw pointers, sizes and strides to the C ABI on
the current torch stream, and raises ``QkrError`` on a non-zero status.  All
arithmetic runs in the library's CUDA kernels; there is no CPU path.  The shared
library is loaded on first use; if it is missing every call raises
ImportError -- build it with ``python mrope_qk_norm_b200/build.py``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqkr.so")

QKR_OK, QKR_ERR_INVALID_ARG, QKR_ERR_UNSUPPORTED, QKR_ERR_CUDA = range(4)
PAIRING_NEOX, PAIRING_GPTJ = 0, 1
(SECTIONS_NONE, SECTIONS_CONTIGUOUS, SECTIONS_INTERLEAVED, SECTIONS_INTERLEAVED_QUOTA,
 SECTIONS_IMROPE) = range(5)
ANGLE_POSITIONS, ANGLE_TABLE = 0, 1
FLAG_ROUND_NORMALIZED_BF16 = 1
FLAG_EAGER_ROUNDING = 2
FLAG_INDEPENDENT = 4
KERNEL_NAMES = {0: "none", 1: "rope_paired", 2: "rope_vector", 3: "rope_exchange",
                4: "vit_setup", 5: "rms_rows", 6: "rms_cluster", 7: "section_map",
                8: "vit_positions", 9: "null"}

EXPORTS = ("fused_qk_norm_rope", "fused_qkv_norm_rope", "mrope_apply", "rope_set_rows",
           "vit_mrope_setup", "rms_norm_residual", "rms_norm_fp8", "qkr_last_error", "qkr_version", "qkr_last_launch", "qkr_section_map",
           "qkr_vit_positions", "qkr_tune_rope", "qkr_tune_rope_lanes", "qkr_tune_rms", "qkr_device_status",
           "qkr_launch_overlap", "qkr_null_launch")


class QkrError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("qkr status %d: %s" % (status, message))
        self.status = status


class StreamDesc(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("q_offset", ctypes.c_int64), ("k_offset", ctypes.c_int64),
                ("q_tok_stride", ctypes.c_int64), ("q_head_stride", ctypes.c_int64),
                ("k_tok_stride", ctypes.c_int64), ("k_head_stride", ctypes.c_int64),
                ("n_tokens", ctypes.c_int64),
                ("gamma_q", ctypes.c_void_p), ("gamma_k", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("v_offset", ctypes.c_int64),
                ("v_tok_stride", ctypes.c_int64), ("v_head_stride", ctypes.c_int64)]


class AngleDesc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("section_mode", ctypes.c_int32),
                ("sections", ctypes.c_int32 * 4),
                ("positions", ctypes.c_void_p), ("pos_row_stride", ctypes.c_int64),
                ("inv_freq", ctypes.c_void_p),
                ("cos", ctypes.c_void_p), ("sin", ctypes.c_void_p),
                ("table_rows", ctypes.c_int64), ("ld", ctypes.c_int64),
                ("plane_stride", ctypes.c_int64), ("token_offset", ctypes.c_int64)]


class LaunchInfo(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("lanes_per_row", ctypes.c_int32),
                ("slots", ctypes.c_int32), ("tokens_per_cta", ctypes.c_int32),
                ("heads_per_item", ctypes.c_int32), ("pipelined", ctypes.c_int32),
                ("cluster", ctypes.c_int32), ("block", ctypes.c_int32),
                ("direct_angles", ctypes.c_int32), ("overlap", ctypes.c_int32),
                ("stages", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("grid", ctypes.c_int64), ("launches", ctypes.c_int64)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError("libqkr.so not built (%s); run python -m mrope_qk_norm_b200.build"
                          % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    V, I64, I32, U32, F = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32,
                           ctypes.c_float)
    sig = {
        "fused_qk_norm_rope": [V, ctypes.POINTER(StreamDesc), I32, V, V, I64, I64, I64, I64, I64,
                               I64, I32, F, ctypes.POINTER(AngleDesc), U32],
        "fused_qkv_norm_rope": [V, ctypes.POINTER(StreamDesc), I32, V, V, V, I64, I64, I64, I64,
                                I64, I64, I64, I64, I32, F, ctypes.POINTER(AngleDesc), U32],
        "mrope_apply": [V, V, V, V, V, I64, I64, I64, I64, I64, I64, I64, I64, I64, V, I64, I64,
                        I64, V, V, I32, I32, V, V, F, U32],
        "rope_set_rows": [V, V, V, V, I64, I64, I64, I64, I64, I64, I64, V, I64, I64, I64, V, V,
                          I32, I32, V, F, U32],
        "vit_mrope_setup": [V, V, V, V, I64, I64, I64, V, V, I64, I64, I64, V, V],
        "rms_norm_residual": [V, V, V, V, V, I64, I64, I64, I64, I64, F],
        "rms_norm_fp8": [V, V, V, V, V, V, I64, I64, I64, I64, I64, F],
        "qkr_last_launch": [ctypes.POINTER(LaunchInfo)],
        "qkr_section_map": [V, I32, V, I64, V],
        "qkr_vit_positions": [V, V, V, I64, I64, I64, V],
        "qkr_tune_rope": [I32, I32, I32, I32],
        "qkr_tune_rope_lanes": [I32],
        "qkr_tune_rms": [I32, I32],
        "qkr_launch_overlap": [I32],
        "qkr_device_status": [ctypes.POINTER(ctypes.c_uint32), I32],
        "qkr_null_launch": [V, I64, I32],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.qkr_last_error.restype = ctypes.c_char_p
    lib.qkr_last_error.argtypes = []
    lib.qkr_version.restype = ctypes.c_char_p
    lib.qkr_version.argtypes = []
    return lib


_lib_handle = None


def lib() -> ctypes.CDLL:
    """The loaded libqkr.so (loaded on first use; raises if it is missing)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load()
    return _lib_handle


class _LazyLib:
    def __getattr__(self, name):
        return getattr(lib(), name)


_lib = _LazyLib()


def version() -> str:
    return _lib.qkr_version().decode()


def _check(status: int) -> None:
    if status != QKR_OK:
        raise QkrError(status, _lib.qkr_last_error().decode())


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t, dtype=None, what="tensor") -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % what)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (what, dtype, t.dtype))
    return t.data_ptr()


def _ptr_base(t, dtype, what):
    """Pointer to the start of the tensor's storage plus the element offset."""
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % what)
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (what, dtype, t.dtype))
    return t.untyped_storage().data_ptr(), t.storage_offset()


def tune_rope(pipeline: int = 0, heads_per_item: int = 0, tokens_per_cta: int = 0,
              stages: int = 0) -> None:
    """Override the rope kernels' launch shape (0 = automatic), for tuning.
    pipeline: 1 item kernel, 3 streaming kernel; heads_per_item: 1 to 4, or
    6 (GPT-J rows of 128 elements with per-item table angles only); stages:
    depth of the streaming kernel's row ring (0 automatic, 1 and 2 both mean
    2, up to 4)."""
    _check(_lib.qkr_tune_rope(pipeline, heads_per_item, tokens_per_cta, stages))


def tune_rope_lanes(lanes: int = 0) -> None:
    """Lanes per head row of the GPT-J layout (0 = automatic), for tuning."""
    _check(_lib.qkr_tune_rope_lanes(lanes))


def tune_rms(cluster: int = 0, threads: int = 0) -> None:
    """CTAs per row and threads per CTA of the RMSNorm kernels (0 = automatic),
    for tuning."""
    _check(_lib.qkr_tune_rms(cluster, threads))


def launch_overlap(enable: bool) -> None:
    """Programmatic dependent launch for every kernel of the library (default on)."""
    _check(_lib.qkr_launch_overlap(1 if enable else 0))


def null_launch(grid: int = 1, block: int = 128, stream=None) -> None:
    """The launch-floor probe: an empty kernel with the library's launch attributes."""
    _check(_lib.qkr_null_launch(_stream(stream), grid, block))


def device_status(reset: bool = False) -> int:
    """The library's device status word (0 = healthy); synchronous."""
    v = ctypes.c_uint32(0)
    _check(_lib.qkr_device_status(ctypes.byref(v), int(reset)))
    return int(v.value)


def last_launch() -> dict:
    info = LaunchInfo()
    _check(_lib.qkr_last_launch(ctypes.byref(info)))
    d = {f: getattr(info, f) for f, _ in LaunchInfo._fields_}
    d["kernel_name"] = KERNEL_NAMES.get(d["kernel"], "?")
    return d


# --------------------------------------------------------------------------
# fused_qk_norm_rope
# --------------------------------------------------------------------------

def stream_desc(q, k, gamma_q, gamma_k, v=None) -> StreamDesc:
    """Descriptor for [T, H, D] Q/K (and optionally V) views (any token/head
    strides, D dense)."""
    bf = torch.bfloat16
    if q.dim() != 3 or k.dim() != 3 or q.shape[0] != k.shape[0]:
        raise ValueError("q and k must be [T, H, D] views with the same T")
    if q.stride(2) != 1 or k.stride(2) != 1:
        raise ValueError("the head dim must be contiguous")
    d = StreamDesc()
    d.q, d.q_offset = _ptr_base(q, bf, "q")
    d.k, d.k_offset = _ptr_base(k, bf, "k")
    d.q_tok_stride, d.q_head_stride = q.stride(0), q.stride(1)
    d.k_tok_stride, d.k_head_stride = k.stride(0), k.stride(1)
    d.n_tokens = q.shape[0]
    d.gamma_q = _ptr(gamma_q, bf, "gamma_q")
    d.gamma_k = _ptr(gamma_k, bf, "gamma_k")
    if v is not None:
        if v.dim() != 3 or v.shape[0] != q.shape[0] or v.stride(2) != 1:
            raise ValueError("v must be a [T, Hv, D] view with the same T and a contiguous D")
        d.v, d.v_offset = _ptr_base(v, bf, "v")
        d.v_tok_stride, d.v_head_stride = v.stride(0), v.stride(1)
    d._keep = (q, k, gamma_q, gamma_k, v)  # the descriptor holds raw pointers into these
    return d


def angle_positions(positions, inv_freq, section_mode=SECTIONS_NONE, sections=None,
                    token_offset=0) -> AngleDesc:
    a = AngleDesc()
    a.kind = ANGLE_POSITIONS
    a.section_mode = section_mode
    for i, s in enumerate(list(sections or []) + [0] * (4 - len(sections or []))):
        a.sections[i] = int(s)
    if positions.dim() == 1:
        positions = positions.view(1, -1)
    if positions.stride(-1) != 1 or (positions.shape[0] > 1 and positions.stride(0) != positions.shape[1]):
        raise ValueError("positions must be a contiguous [rows, T_total] tensor")
    a.positions = _ptr(positions, torch.int32, "positions")
    a.pos_row_stride = positions.shape[-1]
    a.inv_freq = _ptr(inv_freq, torch.float32, "inv_freq")
    a.token_offset = token_offset
    a._keep = (positions, inv_freq)  # the descriptor holds raw pointers into these
    return a


def angle_table(cos, sin, section_mode=SECTIONS_NONE, sections=None, token_offset=0) -> AngleDesc:
    """cos/sin: fp32 [rows, ld] (one table) or [planes, rows, ld] (contiguous)."""
    if cos.shape != sin.shape:
        raise ValueError("cos and sin must have the same shape")
    c3 = cos if cos.dim() == 3 else cos.unsqueeze(0)
    s3 = sin if sin.dim() == 3 else sin.unsqueeze(0)
    if c3.stride(2) != 1 or s3.stride() != c3.stride():
        raise ValueError("tables must have a contiguous last dim and equal strides")
    a = AngleDesc()
    a.kind = ANGLE_TABLE
    a.section_mode = section_mode
    for i, s in enumerate(list(sections or []) + [0] * (4 - len(sections or []))):
        a.sections[i] = int(s)
    a.cos = _ptr(c3, torch.float32, "cos")
    a.sin = _ptr(s3, torch.float32, "sin")
    a.table_rows = c3.shape[1]
    a.ld = c3.stride(1)
    a.plane_stride = c3.stride(0) if c3.shape[0] > 1 else c3.shape[1] * c3.stride(1)
    a.token_offset = token_offset
    a._keep = (c3, s3)  # the descriptor holds raw pointers into these
    return a


def fused_qk_norm_rope(streams, q_out, k_out, rot_dim, pairing, eps, angle: AngleDesc,
                       flags=0, stream=None):
    """streams: list of (q, k, gamma_q, gamma_k) tuples or StreamDesc objects.

    q_out: [T_total, Hq, D], k_out: [T_total, Hk, D] bf16 (heads dense).
    """
    descs = [s if isinstance(s, StreamDesc) else stream_desc(*s) for s in streams]
    arr = (StreamDesc * len(descs))(*descs)
    if q_out.stride(2) != 1 or q_out.stride(1) != q_out.shape[2] or \
            k_out.stride(2) != 1 or k_out.stride(1) != k_out.shape[2]:
        raise ValueError("outputs must have dense heads")
    _check(_lib.fused_qk_norm_rope(
        _stream(stream), arr, len(descs), _ptr(q_out, torch.bfloat16, "q_out"),
        _ptr(k_out, torch.bfloat16, "k_out"), q_out.stride(0), k_out.stride(0),
        q_out.shape[1], k_out.shape[1], q_out.shape[2], rot_dim, pairing, eps,
        ctypes.byref(angle), flags))


def fused_qkv_norm_rope(streams, q_out, k_out, v_out, rot_dim, pairing, eps,
                        angle: AngleDesc, flags=0, stream=None):
    """streams: list of (q, k, gamma_q, gamma_k, v) tuples or StreamDesc objects
    with v set.  q_out / k_out / v_out: [T_total, H, D] bf16 (heads dense); V
    rows are copied unchanged, text first."""
    descs = [s if isinstance(s, StreamDesc) else stream_desc(*s) for s in streams]
    arr = (StreamDesc * len(descs))(*descs)
    for name, t in (("q_out", q_out), ("k_out", k_out), ("v_out", v_out)):
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError("%s must be [T, H, D] with dense heads" % name)
    _check(_lib.fused_qkv_norm_rope(
        _stream(stream), arr, len(descs), _ptr(q_out, torch.bfloat16, "q_out"),
        _ptr(k_out, torch.bfloat16, "k_out"), _ptr(v_out, torch.bfloat16, "v_out"),
        q_out.stride(0), k_out.stride(0), v_out.stride(0), q_out.shape[1], k_out.shape[1],
        v_out.shape[1], q_out.shape[2], rot_dim, pairing, eps, ctypes.byref(angle), flags))


# --------------------------------------------------------------------------
# mrope_apply
# --------------------------------------------------------------------------

def mrope_apply(q, k, q_out, k_out, positions, inv_freq, rot_dim, section_mode=SECTIONS_NONE,
                sections=None, pairing=PAIRING_NEOX, token_offset=0, gamma_q=None,
                gamma_k=None, eps=1e-6, flags=0, stream=None):
    """q: [T, Hq, D], k: [T, Hkv, D] (heads dense); positions int32 [rows, T_total]."""
    for name, t in (("q", q), ("k", k), ("q_out", q_out), ("k_out", k_out)):
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError("%s must be [T, H, D] with dense heads" % name)
    if positions.dim() == 1:
        positions = positions.view(1, -1)
    if not positions.is_contiguous():
        raise ValueError("positions must be contiguous [rows, T_total]")
    sec = None
    if sections is not None:
        sec = (ctypes.c_int32 * 4)(*(list(sections) + [0] * (4 - len(sections))))
    _check(_lib.mrope_apply(
        _stream(stream), _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
        _ptr(q_out, torch.bfloat16, "q_out"), _ptr(k_out, torch.bfloat16, "k_out"),
        q.shape[0], q.shape[1], k.shape[1], q.shape[2], rot_dim, q.stride(0), k.stride(0),
        q_out.stride(0), k_out.stride(0), _ptr(positions, torch.int32, "positions"),
        positions.shape[0], positions.shape[1], token_offset,
        _ptr(inv_freq, torch.float32, "inv_freq"),
        ctypes.cast(sec, ctypes.c_void_p) if sec is not None else None, section_mode, pairing,
        _ptr(gamma_q, torch.bfloat16, "gamma_q"), _ptr(gamma_k, torch.bfloat16, "gamma_k"),
        eps, flags))




def rope_set_rows(x, cache, row_idx, positions, inv_freq, rot_dim, section_mode=SECTIONS_NONE,
                  sections=None, pairing=PAIRING_NEOX, token_offset=0, gamma=None, eps=1e-6,
                  flags=0, stream=None):
    """cache[row_idx[t]] = rope(norm(x[t])): x [T, H, D] bf16 (heads dense),
    cache [R, H, D] bf16 (heads dense), row_idx int64 [T]; positions int32
    [rows, T_total]."""
    for name, t in (("x", x), ("cache", cache)):
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError("%s must be [T, H, D] with dense heads" % name)
    if x.shape[1:] != cache.shape[1:]:
        raise ValueError("x and cache must have the same heads and head dim")
    if row_idx.dim() != 1 or row_idx.shape[0] != x.shape[0] or row_idx.stride(0) != 1:
        raise ValueError("row_idx must be a contiguous int64 [T] tensor")
    if positions.dim() == 1:
        positions = positions.view(1, -1)
    if not positions.is_contiguous():
        raise ValueError("positions must be contiguous [rows, T_total]")
    sec = None
    if sections is not None:
        sec = (ctypes.c_int32 * 4)(*(list(sections) + [0] * (4 - len(sections))))
    T, H, D = x.shape
    _check(_lib.rope_set_rows(
        _stream(stream), _ptr(x, torch.bfloat16, "x"), _ptr(cache, torch.bfloat16, "cache"),
        _ptr(row_idx, torch.int64, "row_idx"), T, H, D, rot_dim, x.stride(0), cache.stride(0),
        cache.shape[0], _ptr(positions, torch.int32, "positions"), positions.shape[0],
        positions.shape[1], token_offset, _ptr(inv_freq, torch.float32, "inv_freq"),
        ctypes.cast(sec, ctypes.c_void_p) if sec is not None else None, section_mode, pairing,
        _ptr(gamma, torch.bfloat16, "gamma") if gamma is not None else None, eps, flags))
# --------------------------------------------------------------------------
# vit_mrope_setup
# --------------------------------------------------------------------------

def vit_mrope_setup(inv_t, inv_h, inv_w, cu_seqlens, grids, n_tokens, spatial_merge, cos_out,
                    sin_out, stream=None):
    """cu_seqlens int32 [G+1], grids int32 [G, 3] (device); cos/sin_out fp32 [3, N, P]."""
    G = grids.shape[0]
    for name, t in (("cos_out", cos_out), ("sin_out", sin_out)):
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous (3, N, P)" % name)
    _check(_lib.vit_mrope_setup(
        _stream(stream), _ptr(inv_t, torch.float32, "inv_t"), _ptr(inv_h, torch.float32, "inv_h"),
        _ptr(inv_w, torch.float32, "inv_w"), inv_t.numel(), inv_h.numel(), inv_w.numel(),
        _ptr(cu_seqlens, torch.int32, "cu_seqlens"), _ptr(grids, torch.int32, "grids"), G,
        n_tokens, spatial_merge, _ptr(cos_out, torch.float32, "cos_out"),
        _ptr(sin_out, torch.float32, "sin_out")))


# --------------------------------------------------------------------------
# rms_norm_residual
# --------------------------------------------------------------------------

def rms_norm_residual(x, residual, gamma, out, eps, stream=None):
    """x, residual, out: [R, hidden] bf16 (row strides free); residual updated in place."""
    for name, t in (("x", x), ("residual", residual), ("out", out)):
        if t.dim() != 2 or t.stride(1) != 1:
            raise ValueError("%s must be [R, hidden] with a contiguous hidden dim" % name)
    R, hidden = x.shape
    _check(_lib.rms_norm_residual(
        _stream(stream), _ptr(x, torch.bfloat16, "x"), _ptr(residual, torch.bfloat16, "residual"),
        _ptr(gamma, torch.bfloat16, "gamma"), _ptr(out, torch.bfloat16, "out"), R, hidden,
        x.stride(0), residual.stride(0), out.stride(0), eps))


# --------------------------------------------------------------------------
# debug entry points
# --------------------------------------------------------------------------

def section_map(mode, sections, P, out, stream=None):
    sec = (ctypes.c_int32 * 4)(*(list(sections) + [0] * (4 - len(sections))))
    _check(_lib.qkr_section_map(_stream(stream), mode, ctypes.cast(sec, ctypes.c_void_p), P,
                                _ptr(out, torch.int8, "axis_out")))


def vit_positions(cu_seqlens, grids, n_tokens, spatial_merge, out, stream=None):
    _check(_lib.qkr_vit_positions(_stream(stream), _ptr(cu_seqlens, torch.int32, "cu_seqlens"),
                                  _ptr(grids, torch.int32, "grids"), grids.shape[0], n_tokens,
                                  spatial_merge, _ptr(out, torch.int32, "pos_out")))


def rms_norm_fp8(x, residual, gamma, out, scale, eps, stream=None):
    """x: [R, hidden] bf16; residual: [R, hidden] bf16 updated in place, or None;
    out: [R, hidden] uint8 (E4M3 codes; view as torch.float8_e4m3fn); scale:
    fp32 [1] device tensor."""
    for name, t in (("x", x), ("out", out)) + ((("residual", residual),) if residual is not None else ()):
        if t.dim() != 2 or t.stride(1) != 1:
            raise ValueError("%s must be [R, hidden] with a contiguous hidden dim" % name)
    if out.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise ValueError("out must be uint8 or float8_e4m3fn")
    if scale.dtype != torch.float32 or scale.numel() != 1 or not scale.is_cuda:
        raise ValueError("scale must be a one-element fp32 CUDA tensor")
    R, hidden = x.shape
    _check(_lib.rms_norm_fp8(
        _stream(stream), _ptr(x, torch.bfloat16, "x"),
        _ptr(residual, torch.bfloat16, "residual") if residual is not None else None,
        _ptr(gamma, torch.bfloat16, "gamma"), out.data_ptr(), scale.data_ptr(), R, hidden,
        x.stride(0), residual.stride(0) if residual is not None else 0, out.stride(0), eps))
