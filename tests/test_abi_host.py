"""Host-side checks of the C ABI that need no GPU.

The library must load, export every function include/qkr.h declares, and
refuse invalid arguments on the host before touching CUDA (these calls
enqueue nothing, so they run on a machine without a device).
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qkr.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\([^;{]*\)\s*;",
                       src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def qkr():
    import mrope_qk_norm_b200 as m
    return m


def test_header_declares_the_four_operations():
    names = _declared_functions()
    for n in ("fused_qk_norm_rope", "mrope_apply", "vit_mrope_setup", "rms_norm_residual"):
        assert n in names


def test_library_exports_every_declared_symbol(qkr):
    lib = ctypes.CDLL(qkr.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_declared_functions()) == set(qkr.EXPORTS)
    assert qkr.version().startswith("qkr")


def _err(qkr):
    return qkr.lib().qkr_last_error().decode()


FAKE = 1 << 32  # a 16-byte aligned non-null address; never dereferenced on refusal


def test_rms_norm_residual_refusals(qkr):
    L = qkr.lib()
    # hidden not a multiple of 8
    assert L.rms_norm_residual(None, FAKE, FAKE + 4096, FAKE, FAKE + 8192, 2, 12, 12, 12, 12,
                               1e-6) == qkr.QKR_ERR_UNSUPPORTED
    assert "hidden" in _err(qkr)
    # null pointer
    assert L.rms_norm_residual(None, 0, FAKE, FAKE, FAKE, 2, 16, 16, 16, 16, 1e-6) == \
        qkr.QKR_ERR_INVALID_ARG
    # misaligned
    assert L.rms_norm_residual(None, FAKE + 2, FAKE + 4096, FAKE, FAKE + 8192, 2, 16, 16, 16, 16,
                               1e-6) == qkr.QKR_ERR_UNSUPPORTED
    # residual overlapping out
    assert L.rms_norm_residual(None, FAKE, FAKE + 4096, FAKE + 65536, FAKE + 4096 + 16, 2, 16, 16,
                               16, 16, 1e-6) == qkr.QKR_ERR_UNSUPPORTED
    # negative eps / NaN eps
    assert L.rms_norm_residual(None, FAKE, FAKE + 4096, FAKE, FAKE + 8192, 2, 16, 16, 16, 16,
                               -1.0) == qkr.QKR_ERR_INVALID_ARG
    assert L.rms_norm_residual(None, FAKE, FAKE + 4096, FAKE, FAKE + 8192, 2, 16, 16, 16, 16,
                               float("nan")) == qkr.QKR_ERR_INVALID_ARG
    # empty call: nothing enqueued, OK
    assert L.rms_norm_residual(None, 0, 0, 0, 0, 0, 16, 16, 16, 16, 1e-6) == qkr.QKR_OK
    assert qkr.last_launch()["launches"] == 0


def _mrope(qkr, **kw):
    a = dict(stream=None, q=FAKE, k=FAKE + (1 << 20), q_out=FAKE + (2 << 20), k_out=FAKE + (3 << 20),
             T=4, Hq=2, Hkv=1, D=64, rot=64, qts=128, kts=64, qots=128, kots=64, pos=FAKE + (4 << 20),
             n_rows=3, T_total=4, off=0, inv=FAKE + (5 << 20), sec=(16, 8, 8, 0),
             mode=qkr.SECTIONS_INTERLEAVED, pairing=0, gq=None, gk=None, eps=1e-6, flags=0)
    a.update(kw)
    sec = None
    if a["sec"] is not None:
        sec = ctypes.cast((ctypes.c_int32 * 4)(*a["sec"]), ctypes.c_void_p)
    return qkr.lib().mrope_apply(a["stream"], a["q"], a["k"], a["q_out"], a["k_out"], a["T"],
                                 a["Hq"], a["Hkv"], a["D"], a["rot"], a["qts"], a["kts"],
                                 a["qots"], a["kots"], a["pos"], a["n_rows"], a["T_total"],
                                 a["off"], a["inv"], sec, a["mode"], a["pairing"], a["gq"],
                                 a["gk"], a["eps"], a["flags"])


def test_mrope_apply_refusals(qkr):
    E, U = qkr.QKR_ERR_INVALID_ARG, qkr.QKR_ERR_UNSUPPORTED
    # sections requested but missing: refuse rather than rotate by one row
    assert _mrope(qkr, sec=None) == E and "sections" in _err(qkr)
    # section sum outside [P, 2P]
    assert _mrope(qkr, sec=(10, 8, 8, 0)) == E
    assert _mrope(qkr, sec=(40, 40, 40, 0)) == E
    # fourth section outside IMROPE
    assert _mrope(qkr, sec=(16, 8, 4, 4)) == E
    # IMROPE needs four rows
    assert _mrope(qkr, mode=qkr.SECTIONS_IMROPE, sec=(16, 8, 4, 4)) == E
    # chunk past the positions buffer (token_offset + T > T_total)
    assert _mrope(qkr, off=1) == E and "exceeds" in _err(qkr)
    # rot_dim > head_dim, odd rot_dim, head_dim not a multiple of 8, head_dim > 256
    assert _mrope(qkr, rot=80) == E
    assert _mrope(qkr, rot=63, sec=(11, 10, 10, 0)) == E
    assert _mrope(qkr, D=60, rot=60, qts=120, kts=60, qots=120, kots=60, sec=(10, 10, 10, 0)) == U
    assert _mrope(qkr, D=264, rot=64, qts=528, kts=264, qots=528, kots=264) == U
    # one gamma only
    assert _mrope(qkr, gq=FAKE + (6 << 20)) == E
    # misaligned q
    assert _mrope(qkr, q=FAKE + 8) == U
    # partial overlap of output with input (not exact in-place)
    assert _mrope(qkr, q_out=FAKE + 16) == U
    # unknown mode / pairing / flags
    assert _mrope(qkr, mode=9) == E
    assert _mrope(qkr, pairing=3) == E
    assert _mrope(qkr, flags=8) == E
    # the rounding contracts need the norm, and only one at a time
    assert _mrope(qkr, flags=2) == E and "normalisation" in _err(qkr)
    assert _mrope(qkr, flags=3, gq=FAKE + (6 << 20), gk=FAKE + (7 << 20)) == E
    # empty chunk: OK, nothing enqueued
    assert _mrope(qkr, T=0) == qkr.QKR_OK
    assert qkr.last_launch()["launches"] == 0


def test_fused_refusals(qkr):
    E, U = qkr.QKR_ERR_INVALID_ARG, qkr.QKR_ERR_UNSUPPORTED
    L = qkr.lib()
    d = qkr.StreamDesc(q=FAKE, k=FAKE + (1 << 20), q_offset=0, k_offset=0, q_tok_stride=256,
                       q_head_stride=64, k_tok_stride=256, k_head_stride=64, n_tokens=4,
                       gamma_q=FAKE + (2 << 20), gamma_k=FAKE + (2 << 20))
    a = qkr.AngleDesc(kind=qkr.ANGLE_TABLE, section_mode=0, cos=FAKE + (3 << 20),
                      sin=FAKE + (4 << 20), table_rows=4, ld=32, plane_stride=128)
    arr = (qkr.StreamDesc * 2)(d, d)

    def call(n=1, q_out=FAKE + (5 << 20), k_out=FAKE + (6 << 20), qots=256, kots=256, rot=64,
             angle=a, flags=0):
        return L.fused_qk_norm_rope(None, arr, n, q_out, k_out, qots, kots, 4, 4, 64, rot, 0,
                                    1e-6, ctypes.byref(angle), flags)
    # outputs overlapping inputs are refused (fresh outputs)
    assert call(q_out=FAKE) == U
    # two streams need table rows for all 8 joint tokens
    assert call(n=2) == E
    # ld smaller than the rotated pairs
    a2 = qkr.AngleDesc(kind=qkr.ANGLE_TABLE, section_mode=0, cos=FAKE + (3 << 20),
                       sin=FAKE + (4 << 20), table_rows=4, ld=16, plane_stride=64)
    assert call(angle=a2) == E
    # missing gamma
    arr[0].gamma_q = 0
    assert call() == E
    arr[0].gamma_q = FAKE + (2 << 20)
    # storage offset not a multiple of 8 elements
    arr[0].q_offset = 4
    assert call() == U
    arr[0].q_offset = 0
    # n_streams out of range
    assert call(n=3) == E
    # output stride too small for the heads
    assert call(qots=128) == U


def test_fused_qkv_refusals(qkr):
    E, U = qkr.QKR_ERR_INVALID_ARG, qkr.QKR_ERR_UNSUPPORTED
    L = qkr.lib()
    d = qkr.StreamDesc(q=FAKE, k=FAKE + (1 << 20), q_offset=0, k_offset=0, q_tok_stride=256,
                       q_head_stride=64, k_tok_stride=256, k_head_stride=64, n_tokens=4,
                       gamma_q=FAKE + (2 << 20), gamma_k=FAKE + (2 << 20), v=FAKE + (7 << 20),
                       v_offset=0, v_tok_stride=192, v_head_stride=64)
    a = qkr.AngleDesc(kind=qkr.ANGLE_TABLE, section_mode=0, cos=FAKE + (3 << 20),
                      sin=FAKE + (4 << 20), table_rows=8, ld=32, plane_stride=256)
    arr = (qkr.StreamDesc * 2)(d, d)

    def call(n=1, v_out=FAKE + (8 << 20), vots=192, Hv=3):
        return L.fused_qkv_norm_rope(None, arr, n, FAKE + (5 << 20), FAKE + (6 << 20), v_out,
                                     256, 256, vots, 4, 4, Hv, 64, 64, 0, 1e-6,
                                     ctypes.byref(a), 0)
    # Hv must be >= 1 (the Q/K-only op is fused_qk_norm_rope)
    assert call(Hv=0) == E and "Hv" in _err(qkr)
    # v_out missing, misaligned, too narrow, overlapping an input or another output
    assert call(v_out=0) == E
    assert call(v_out=FAKE + (8 << 20) + 8) == U
    assert call(vots=128) == U
    assert call(v_out=FAKE + (7 << 20)) == U
    assert call(v_out=FAKE + (5 << 20) + 64) == U
    # a stream without v
    arr[0].v = 0
    assert call() == E and "v must be non-NULL" in _err(qkr)
    arr[0].v = FAKE + (7 << 20)
    # v stride not a multiple of 8 elements, v heads overlapping
    arr[0].v_tok_stride = 196
    assert call() == U
    arr[0].v_tok_stride = 192
    arr[0].v_head_stride = 32
    assert call() == U
    arr[0].v_head_stride = 64
    # an empty call enqueues nothing
    arr[0].n_tokens = 0
    assert call() == qkr.QKR_OK
    assert qkr.last_launch()["launches"] == 0


def test_launch_switch_refusals(qkr):
    L = qkr.lib()
    assert L.qkr_launch_overlap(2) == qkr.QKR_ERR_INVALID_ARG
    assert L.qkr_launch_overlap(-1) == qkr.QKR_ERR_INVALID_ARG
    assert L.qkr_tune_rope(4, 0, 0, 0) == qkr.QKR_ERR_INVALID_ARG
    assert L.qkr_tune_rope(2, 0, 0, 0) == qkr.QKR_ERR_INVALID_ARG   # 1 item, 3 streaming only
    assert L.qkr_tune_rope(3, 0, 0, 5) == qkr.QKR_ERR_INVALID_ARG
    assert L.qkr_tune_rope(1, 0, 0, -1) == qkr.QKR_ERR_INVALID_ARG
    assert L.qkr_tune_rope(3, 5, 0, 0) == qkr.QKR_ERR_INVALID_ARG
    assert L.qkr_tune_rope(1, 7, 0, 0) == qkr.QKR_ERR_INVALID_ARG
    assert L.qkr_tune_rope(1, 8, 0, 0) == qkr.QKR_ERR_INVALID_ARG
    assert L.qkr_tune_rope(1, 6, 0, 0) == qkr.QKR_OK  # GPT-J rows of 128 with table angles
    assert L.qkr_tune_rope(3, 0, 65, 0) == qkr.QKR_ERR_INVALID_ARG
    assert L.qkr_tune_rope(0, 0, 0, 0) == qkr.QKR_OK
    assert L.qkr_launch_overlap(1) == qkr.QKR_OK


def test_rope_set_rows_refusals(qkr):
    E, U = qkr.QKR_ERR_INVALID_ARG, qkr.QKR_ERR_UNSUPPORTED
    L = qkr.lib()
    sec = ctypes.cast((ctypes.c_int32 * 4)(24, 20, 20, 0), ctypes.c_void_p)

    def call(x=FAKE, cache=FAKE + (1 << 20), rows=FAKE + (2 << 20), T=4, R=16, cstride=1024,
             n_rows=3, mode=qkr.SECTIONS_INTERLEAVED, gamma=None, flags=0):
        return L.rope_set_rows(None, x, cache, rows, T, 8, 128, 128, 1024, cstride, R,
                               FAKE + (3 << 20), n_rows, 4, 0, FAKE + (4 << 20), sec, mode, 0,
                               gamma, 1e-6, flags)
    assert call(rows=None) == E and "row_idx" in _err(qkr)
    assert call(rows=FAKE + (2 << 20) + 4) == U        # not 8-byte aligned
    assert call(R=0) == E                               # empty cache
    assert call(cache=FAKE + 512) == U                  # cache overlaps x
    assert call(cstride=1000) == U                      # row stride not a multiple of 8
    assert call(n_rows=1) == E                          # interleaved mode reads 3 rows
    assert call(flags=qkr.FLAG_ROUND_NORMALIZED_BF16) == E  # rounding contract needs gamma
    assert call(T=0, rows=None) == qkr.QKR_OK           # empty: nothing enqueued
    assert qkr.last_launch()["launches"] == 0


def test_rms_norm_fp8_refusals(qkr):
    E, U = qkr.QKR_ERR_INVALID_ARG, qkr.QKR_ERR_UNSUPPORTED
    L = qkr.lib()

    def call(x=FAKE, res=FAKE + (1 << 20), gamma=FAKE + (2 << 20), out=FAKE + (3 << 20),
             scale=FAKE + (4 << 20), R=4, hidden=64, xs=64, rs=64, os=64):
        return L.rms_norm_fp8(None, x, res, gamma, out, scale, R, hidden, xs, rs, os, 1e-6)
    assert call(scale=None) == E                 # the static scale is required
    assert call(out=FAKE + (3 << 20) + 4) == U   # FP8 rows need 8-byte alignment
    assert call(os=60) == U                      # stride below hidden
    assert call(out=FAKE + 64) == U              # out overlaps x
    assert call(scale=FAKE + (1 << 20) + 8) == U  # scale inside the residual it rewrites
    assert call(scale=FAKE + (3 << 20) + 8) == U  # scale inside out
    assert call(hidden=60, xs=60, rs=60, os=60) == U
    assert call(R=0) == qkr.QKR_OK
    assert qkr.last_launch()["launches"] == 0


def test_too_many_tokens_is_refused_not_launched(qkr):
    L = qkr.lib()
    T = 1 << 31  # one past what a launch takes
    d = qkr.StreamDesc(q=FAKE, k=FAKE + (1 << 40), q_offset=0, k_offset=0, q_tok_stride=64,
                       q_head_stride=64, k_tok_stride=64, k_head_stride=64, n_tokens=T,
                       gamma_q=FAKE + (2 << 40), gamma_k=FAKE + (2 << 40))
    a = qkr.AngleDesc(kind=qkr.ANGLE_TABLE, section_mode=0, cos=FAKE + (3 << 40),
                      sin=FAKE + (4 << 40), table_rows=T, ld=32, plane_stride=32 * T)
    arr = (qkr.StreamDesc * 1)(d)
    st = L.fused_qk_norm_rope(None, arr, 1, FAKE + (5 << 40), FAKE + (6 << 40), 64, 64, 1, 1, 64,
                              64, 0, 1e-6, ctypes.byref(a), 0)
    assert st == qkr.QKR_ERR_UNSUPPORTED and "2^31" in _err(qkr)


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="an accepted call would launch on the fake addresses")
def test_packed_qkv_in_place_passes_validation(qkr):
    """Q and K as column windows of one packed [T, 3, H, D] buffer, rotated in
    place: their byte ranges interleave but share no element, so the host
    accepts the call (here it then fails only at the launch, with no device);
    windows that do share elements are still refused."""
    T, H, D = 4, 2, 64
    ts = 3 * H * D
    base = FAKE
    q, k = base, base + 2 * H * D          # columns [0, HD) and [HD, 2HD) of each token row
    st = _mrope(qkr, q=q, k=k, q_out=q, k_out=k, T=T, Hq=H, Hkv=H, D=D, rot=D, qts=ts, kts=ts,
                qots=ts, kots=ts, T_total=T, sec=(16, 8, 8, 0))
    assert st == qkr.QKR_ERR_CUDA, _err(qkr)   # validation passed; no device to launch on
    # K window shifted by 8 elements into Q's columns: shared elements, refused
    st = _mrope(qkr, q=q, k=q + 2 * (H * D - 8), q_out=q, k_out=q + 2 * (H * D - 8), T=T, Hq=H,
                Hkv=H, D=D, rot=D, qts=ts, kts=ts, qots=ts, kots=ts, T_total=T, sec=(16, 8, 8, 0))
    assert st == qkr.QKR_ERR_UNSUPPORTED
    # an output window laid over the other input's columns: refused
    st = _mrope(qkr, q=q, k=k, q_out=k, k_out=q, T=T, Hq=H, Hkv=H, D=D, rot=D, qts=ts, kts=ts,
                qots=ts, kots=ts, T_total=T, sec=(16, 8, 8, 0))
    assert st == qkr.QKR_ERR_UNSUPPORTED
