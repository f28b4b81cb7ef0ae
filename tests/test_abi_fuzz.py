"""Host-side fuzz of the C ABI's argument validation (no GPU needed).

Random sizes, strides, offsets, pointers (never dereferenced: nothing is
launched on a machine without a device, and a call that passes validation
there fails only at the launch with QKR_ERR_CUDA) and modes must always come
back as one of the four status codes with a message for every refusal --
never a crash, never an exception.
"""
import ctypes

import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import mrope_qk_norm_b200 as qkr

STATUSES = {qkr.QKR_OK, qkr.QKR_ERR_INVALID_ARG, qkr.QKR_ERR_UNSUPPORTED, qkr.QKR_ERR_CUDA}
BASE = 1 << 36
ptrs = st.one_of(st.just(0), st.integers(0, 1 << 24).map(lambda o: BASE + o))
small = st.integers(-3, 300)
big = st.integers(-(1 << 33), 1 << 33)

pytestmark = pytest.mark.skipif(
    __import__("torch").cuda.is_available(),
    reason="host-only fuzz: on a GPU machine a validated call would launch on fake pointers")


def _check(status):
    assert status in STATUSES
    if status in (qkr.QKR_ERR_INVALID_ARG, qkr.QKR_ERR_UNSUPPORTED):
        assert qkr.lib().qkr_last_error().decode()


@settings(max_examples=400, deadline=None, suppress_health_check=list(HealthCheck))
@given(x=ptrs, res=ptrs, g=ptrs, out=ptrs, R=small, hidden=st.integers(-8, 70000),
       xs=big, rs=big, os_=big, eps=st.floats(allow_nan=True, allow_infinity=True))
def test_rms_norm_residual_fuzz(x, res, g, out, R, hidden, xs, rs, os_, eps):
    _check(qkr.lib().rms_norm_residual(None, x, res, g, out, R, hidden, xs, rs, os_, eps))


@settings(max_examples=400, deadline=None, suppress_health_check=list(HealthCheck))
@given(x=ptrs, res=ptrs, g=ptrs, out=ptrs, sc=ptrs, R=small, hidden=st.integers(-8, 70000),
       xs=big, rs=big, os_=big)
def test_rms_norm_fp8_fuzz(x, res, g, out, sc, R, hidden, xs, rs, os_):
    _check(qkr.lib().rms_norm_fp8(None, x, res, g, out, sc, R, hidden, xs, rs, os_, 1e-6))


@settings(max_examples=600, deadline=None, suppress_health_check=list(HealthCheck))
@given(q=ptrs, k=ptrs, qo=ptrs, ko=ptrs, T=small, Hq=st.integers(-2, 70), Hk=st.integers(-2, 70),
       D=st.integers(-8, 300), rot=st.integers(-4, 300), qts=big, kts=big, qots=big, kots=big,
       pos=ptrs, rows=st.integers(-1, 5), T_total=big, off=big, inv=ptrs,
       sec=st.one_of(st.none(), st.lists(st.integers(-5, 200), min_size=4, max_size=4)),
       mode=st.integers(-1, 6), pairing=st.integers(-1, 3), gq=ptrs, gk=ptrs,
       flags=st.integers(0, 4))
def test_mrope_apply_fuzz(q, k, qo, ko, T, Hq, Hk, D, rot, qts, kts, qots, kots, pos, rows,
                          T_total, off, inv, sec, mode, pairing, gq, gk, flags):
    s = None if sec is None else ctypes.cast((ctypes.c_int32 * 4)(*sec), ctypes.c_void_p)
    _check(qkr.lib().mrope_apply(None, q, k, qo, ko, T, Hq, Hk, D, rot, qts, kts, qots, kots,
                                 pos, rows, T_total, off, inv, s, mode, pairing, gq, gk, 1e-6,
                                 flags))


@settings(max_examples=400, deadline=None, suppress_health_check=list(HealthCheck))
@given(n=st.integers(-1, 3), T0=small, T1=small, qo=ptrs, ko=ptrs, vo=ptrs,
       Hq=st.integers(-1, 40), Hk=st.integers(-1, 40), Hv=st.integers(-1, 40),
       D=st.integers(-8, 300), rot=st.integers(-4, 300), strides=st.lists(big, min_size=6,
                                                                          max_size=6),
       kind=st.integers(-1, 2), mode=st.integers(-1, 5), ld=big, rows=big, off=big,
       use_v=st.booleans())
def test_fused_fuzz(n, T0, T1, qo, ko, vo, Hq, Hk, Hv, D, rot, strides, kind, mode, ld, rows,
                    off, use_v):
    d0 = qkr.StreamDesc(q=BASE, k=BASE + (1 << 26), q_offset=0, k_offset=0,
                        q_tok_stride=strides[0], q_head_stride=strides[1],
                        k_tok_stride=strides[2], k_head_stride=strides[3], n_tokens=T0,
                        gamma_q=BASE + (2 << 26), gamma_k=BASE + (2 << 26),
                        v=BASE + (3 << 26), v_offset=0, v_tok_stride=strides[4],
                        v_head_stride=strides[5])
    d1 = qkr.StreamDesc(q=BASE + (4 << 26), k=BASE + (5 << 26), q_offset=0, k_offset=0,
                        q_tok_stride=strides[0], q_head_stride=strides[1],
                        k_tok_stride=strides[2], k_head_stride=strides[3], n_tokens=T1,
                        gamma_q=BASE + (2 << 26), gamma_k=BASE + (2 << 26),
                        v=BASE + (6 << 26), v_offset=0, v_tok_stride=strides[4],
                        v_head_stride=strides[5])
    arr = (qkr.StreamDesc * 2)(d0, d1)
    a = qkr.AngleDesc(kind=kind, section_mode=mode, cos=BASE + (7 << 26), sin=BASE + (8 << 26),
                      positions=BASE + (9 << 26), inv_freq=BASE + (10 << 26), pos_row_stride=rows,
                      table_rows=rows, ld=ld, plane_stride=ld * 4, token_offset=off)
    a.sections[0], a.sections[1], a.sections[2] = 16, 8, 8
    L = qkr.lib()
    if use_v:
        st_ = L.fused_qkv_norm_rope(None, arr, n, qo, ko, vo, strides[0], strides[2], strides[4],
                                    Hq, Hk, Hv, D, rot, 0, 1e-6, ctypes.byref(a), 0)
    else:
        st_ = L.fused_qk_norm_rope(None, arr, n, qo, ko, strides[0], strides[2], Hq, Hk, D, rot,
                                   1, 1e-6, ctypes.byref(a), 0)
    _check(st_)
