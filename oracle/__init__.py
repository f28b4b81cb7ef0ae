"""CPU oracle for the normalise-then-rotate path (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  It wraps ``oracle.c`` (plain
fp64 C, compiled with gcc into ``liboracle.so``) through ctypes and shares no
code with the CUDA library.

Parity pins for every function are in ``tests/test_oracle_pins.py``.  Absolute
values of the rotation sign convention are fixed by the textbook
complex-multiplication form of RoPE (pinned), not by the pages, which print no
worked numeric example.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

SEC_NONE, SEC_CONTIGUOUS, SEC_INTERLEAVED, SEC_INTERLEAVED_QUOTA, SEC_IMROPE = range(5)
# Rounding points of the normalised value (oracle.c rms_norm_head).
ROUND_NONE, ROUND_NORMALIZED, ROUND_EAGER = range(3)


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared",
                               "-ffp-contract=off", "-fno-fast-math", _SRC, "-lm", "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


class _Angle(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("section_mode", ctypes.c_int32),
                ("sections", ctypes.c_int32 * 4),
                ("positions", ctypes.c_void_p), ("pos_row_stride", ctypes.c_int64),
                ("inv_freq", ctypes.c_void_p),
                ("cos_tab", ctypes.c_void_p), ("sin_tab", ctypes.c_void_p),
                ("plane_stride", ctypes.c_int64), ("ld", ctypes.c_int64),
                ("token_offset", ctypes.c_int64)]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.oracle_bf16_round.restype = ctypes.c_uint16
        lib.oracle_bf16_round.argtypes = [ctypes.c_double]
        lib.oracle_section_axis.restype = I32
        lib.oracle_section_axis.argtypes = [I32, P, I64]
        lib.oracle_section_map.restype = None
        lib.oracle_section_map.argtypes = [I32, P, I64, P]
        lib.oracle_qk_norm_rope.restype = I32
        lib.oracle_qk_norm_rope.argtypes = [I32, P, P, P, P, P, I64, I64, I64, I64, I32,
                                            ctypes.c_double, I32, I32,
                                            ctypes.POINTER(_Angle), P, P, P, P]
        lib.oracle_vit_positions.restype = I64
        lib.oracle_vit_positions.argtypes = [P, I64, ctypes.c_int32, P, I64]
        lib.oracle_vit_planes.restype = None
        lib.oracle_vit_planes.argtypes = [P, I64, P, I64, P, I64, P, I64, P, P, P]
        lib.oracle_rms_norm_residual.restype = None
        lib.oracle_rms_norm_residual.argtypes = [P, P, P, I64, I64, ctypes.c_double, P, P]
        lib.oracle_fp8_e4m3.restype = ctypes.c_uint8
        lib.oracle_fp8_e4m3.argtypes = [ctypes.c_double]
        lib.oracle_fp8_e4m3_array.restype = None
        lib.oracle_fp8_e4m3_array.argtypes = [P, I64, P]
        lib.oracle_rms_norm_fp8.restype = None
        lib.oracle_rms_norm_fp8.argtypes = [P, P, P, I64, I64, ctypes.c_double, ctypes.c_double,
                                            P, P, P]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def bits(t) -> np.ndarray:
    """bf16 tensor -> contiguous uint16 numpy array of its bit patterns."""
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.uint16)
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy()
                                .view(np.uint16))


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_round(v) -> np.ndarray:
    """Round-to-nearest-even of each fp64 value to bf16 (bit patterns)."""
    lib = _load()
    flat = np.asarray(v, dtype=np.float64).reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint16)
    for i, x in enumerate(flat):
        out[i] = lib.oracle_bf16_round(float(x))
    return out.reshape(np.shape(v))


def section_axis(mode: int, sections, j: int) -> int:
    s = (ctypes.c_int32 * 4)(*(list(sections) + [0] * (4 - len(sections))))
    return _load().oracle_section_axis(mode, ctypes.cast(s, ctypes.c_void_p), j)


def section_map(mode: int, sections, P: int) -> np.ndarray:
    s = np.array(list(sections) + [0] * (4 - len(sections)), dtype=np.int32)
    out = np.empty(P, dtype=np.int8)
    _load().oracle_section_map(mode, _ptr(s), P, _ptr(out))
    return out


def _make_angle(angle, keep: list) -> _Angle:
    A = _Angle()
    A.kind = int(angle.kind)
    A.section_mode = int(angle.section_mode)
    secs = list(angle.sections) + [0] * (4 - len(angle.sections))
    for i in range(4):
        A.sections[i] = int(secs[i])
    A.token_offset = int(angle.token_offset)
    if A.kind == 0:
        pos = np.ascontiguousarray(np.asarray(angle.positions, dtype=np.int32))
        inv = np.ascontiguousarray(np.asarray(angle.inv_freq, dtype=np.float32))
        keep += [pos, inv]
        A.positions = _ptr(pos)
        A.pos_row_stride = pos.shape[-1]
        A.inv_freq = _ptr(inv)
    else:
        cos = np.ascontiguousarray(np.asarray(angle.cos, dtype=np.float32))
        sin = np.ascontiguousarray(np.asarray(angle.sin, dtype=np.float32))
        if cos.ndim == 2:
            cos, sin = cos[None], sin[None]
        keep += [cos, sin]
        A.cos_tab, A.sin_tab = _ptr(cos), _ptr(sin)
        A.plane_stride = cos.shape[1] * cos.shape[2]
        A.ld = cos.shape[2]
    return A


def qk_norm_rope(streams, Hq: int, Hk: int, D: int, rot: int, pairing: int, eps: float,
                 angle, norm: bool = True, round_normalized: bool = False,
                 eager_rounding: bool = False, return_ties: bool = False):
    """Joint (text-first) RMSNorm + RoPE of Q and K; returns fp64 [T, H, D] arrays.

    ``streams`` is a list of objects with ``q``, ``k`` ([T, H, D] bf16) and
    ``gamma_q``, ``gamma_k`` ([D] bf16) attributes.  ``round_normalized``:
    y = bf16(x r gamma) before the rotation; ``eager_rounding``: y =
    bf16(bf16(x r) gamma).  With ``return_ties`` also returns two uint8 masks
    of the output elements that depend on a value sitting within 1e-3 bf16
    quanta of a rounding midpoint (where an fp32 evaluation may take the
    other neighbour).
    """
    if round_normalized and eager_rounding:
        raise ValueError("one rounding contract at a time")
    mode = ROUND_EAGER if eager_rounding else (ROUND_NORMALIZED if round_normalized else ROUND_NONE)
    lib = _load()
    keep = []
    T_s = np.array([int(s.q.shape[0]) for s in streams], dtype=np.int64)
    arrs = {name: [bits(getattr(s, name)) for s in streams]
            for name in ("q", "k", "gamma_q", "gamma_k")}
    keep += [T_s] + sum(arrs.values(), [])
    ptrs = {name: (ctypes.c_void_p * len(streams))(*[_ptr(a) for a in v])
            for name, v in arrs.items()}
    T = int(T_s.sum())
    q_out = np.empty((T, Hq, D), dtype=np.float64)
    k_out = np.empty((T, Hk, D), dtype=np.float64)
    tq = np.zeros((T, Hq, D), dtype=np.uint8) if return_ties else None
    tk = np.zeros((T, Hk, D), dtype=np.uint8) if return_ties else None
    A = _make_angle(angle, keep)
    rc = lib.oracle_qk_norm_rope(len(streams), _ptr(T_s),
                                 ctypes.cast(ptrs["q"], ctypes.c_void_p),
                                 ctypes.cast(ptrs["k"], ctypes.c_void_p),
                                 ctypes.cast(ptrs["gamma_q"], ctypes.c_void_p),
                                 ctypes.cast(ptrs["gamma_k"], ctypes.c_void_p),
                                 Hq, Hk, D, rot, pairing, float(eps), int(norm), mode,
                                 ctypes.byref(A), _ptr(q_out), _ptr(k_out),
                                 _ptr(tq) if return_ties else None,
                                 _ptr(tk) if return_ties else None)
    if rc != 0:
        raise ValueError("oracle_qk_norm_rope rejected its arguments")
    if return_ties:
        return q_out, k_out, tq.astype(bool), tk.astype(bool)
    return q_out, k_out


def joint_v(v_streams) -> np.ndarray:
    """V of the joint Q/K/V op (vllm-omni #7600, Purpose): every stream's V
    rows, unchanged, text first -- the bf16 bit patterns [T0+T1, Hv, D]."""
    return np.concatenate([bits(v) for v in v_streams], axis=0)


def scatter_rows(rows: np.ndarray, row_idx, n_rows: int, fill=np.nan) -> np.ndarray:
    """rope_set_rows's destination (llama.cpp fork #286, "The change": rotated
    rows written to the rows their indices name): out[row_idx[t]] = rows[t];
    rows no index names hold `fill`."""
    idx = np.asarray(row_idx, dtype=np.int64)
    out = np.full((n_rows,) + rows.shape[1:], fill, dtype=rows.dtype)
    for t, r in enumerate(idx):
        out[r] = rows[t]
    return out


def vit_positions(grids, spatial_merge: int) -> np.ndarray:
    """int32 [3, N] (t, h, w) positions of every token, by nested loops."""
    lib = _load()
    g = np.ascontiguousarray(np.asarray(grids, dtype=np.int32).reshape(-1, 3))
    N = int(lib.oracle_vit_positions(_ptr(g), g.shape[0], spatial_merge, None, 0))
    if N < 0:
        raise ValueError("grid h and w must be multiples of spatial_merge")
    pos = np.empty((3, N), dtype=np.int32)
    lib.oracle_vit_positions(_ptr(g), g.shape[0], spatial_merge, _ptr(pos), N)
    return pos


def vit_planes(pos: np.ndarray, inv_t, inv_h, inv_w):
    """(cos, sin, written): fp32 (3, N, P) planes and a uint8 mask of written cells."""
    lib = _load()
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    invs = [np.ascontiguousarray(np.asarray(v, dtype=np.float32)) for v in (inv_t, inv_h, inv_w)]
    N = pos.shape[1]
    P = sum(len(v) for v in invs)
    cos = np.full((3, N, P), np.nan, dtype=np.float32)
    sin = np.full((3, N, P), np.nan, dtype=np.float32)
    written = np.zeros((3, N, P), dtype=np.uint8)
    lib.oracle_vit_planes(_ptr(pos), N, _ptr(invs[0]), len(invs[0]), _ptr(invs[1]),
                          len(invs[1]), _ptr(invs[2]), len(invs[2]), _ptr(cos), _ptr(sin),
                          _ptr(written))
    return cos, sin, written


def rms_norm_residual(x, residual, gamma, eps: float):
    """(new_residual bf16 bits [R, hidden], out fp64 [R, hidden])."""
    lib = _load()
    xb, rb, gb = bits(x), bits(residual), bits(gamma)
    R, hidden = xb.shape
    res_out = np.empty((R, hidden), dtype=np.uint16)
    out = np.empty((R, hidden), dtype=np.float64)
    lib.oracle_rms_norm_residual(_ptr(xb), _ptr(rb), _ptr(gb), R, hidden, float(eps),
                                 _ptr(res_out), _ptr(out))
    return res_out, out


def fp8_e4m3(values) -> np.ndarray:
    """E4M3 ("FN") codes of fp64 values: round to nearest even, saturate at 448."""
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float64))
    out = np.empty(v.shape, dtype=np.uint8)
    _load().oracle_fp8_e4m3_array(_ptr(v), v.size, _ptr(out))
    return out


def rms_norm_fp8(x, residual, gamma, eps: float, scale: float):
    """(new residual bf16 bits or None, y / scale in fp64, E4M3 codes), [R, hidden]."""
    lib = _load()
    xb, gb = bits(x), bits(gamma)
    R, hidden = xb.shape
    rb = bits(residual) if residual is not None else None
    res_out = np.empty((R, hidden), dtype=np.uint16)
    ys = np.empty((R, hidden), dtype=np.float64)
    codes = np.empty((R, hidden), dtype=np.uint8)
    lib.oracle_rms_norm_fp8(_ptr(xb), _ptr(rb) if rb is not None else None, _ptr(gb), R,
                            hidden, float(eps), float(scale), _ptr(res_out), _ptr(ys),
                            _ptr(codes))
    return (res_out if rb is not None else None), ys, codes
