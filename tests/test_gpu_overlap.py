"""Programmatic dependent launch (qkr_launch_overlap) keeps stream order.

Each case runs a chain of launches in which every call reads what the
previous call wrote (outputs fed back as inputs, a residual updated in place)
with no host synchronisation in between, once with the overlap switch on and
once with it off: the final bits must agree, and must agree with the oracle
where one applies.  A kernel that touched memory before its grid-dependency
wait would read stale data in the overlapped chain.
"""
import numpy as np
import pytest
import torch

import mrope_qk_norm_b200 as qkr
import oracle
import workloads as W
from tests._gpu_util import assert_bf16_close, to_dev

pytestmark = pytest.mark.gpu


def _both(run):
    outs = []
    try:
        for on in (True, False):
            qkr.launch_overlap(on)
            outs.append(run())
            torch.cuda.synchronize()
    finally:
        qkr.launch_overlap(True)
    return outs


def _bits(t):
    return t.contiguous().view(torch.int16)


def test_rope_chain_direct_and_staged():
    w = W.config3(seed=91, T_txt=100, img_h=12, img_w=17, H=8, D=128, pairing=W.PAIRING_GPTJ)
    cos = to_dev(torch.as_tensor(np.asarray(w.angle.cos), dtype=torch.float32))
    sin = to_dev(torch.as_tensor(np.asarray(w.angle.sin), dtype=torch.float32))
    T = w.n_tokens
    streams = [(to_dev(s.q), to_dev(s.k), to_dev(s.gamma_q), to_dev(s.gamma_k)) for s in w.streams]
    inv = W.inv_freq(1e4, 64, 128)
    pos = torch.arange(T, dtype=torch.int32).view(1, T)
    a_tab = qkr.angle_table(cos, sin)
    a_pos = qkr.angle_positions(to_dev(pos), to_dev(inv))

    def run():
        # step 0: joint launch from the two streams; steps 1..: rotate the
        # previous output again (alternating direct-table and staged angles)
        q = torch.empty(T, w.Hq, w.D, dtype=torch.bfloat16, device="cuda")
        k = torch.empty_like(q)
        qkr.fused_qk_norm_rope(streams, q, k, w.rot, w.pairing, w.eps, a_tab)
        g = streams[0][2]
        for i in range(12):
            q2, k2 = torch.empty_like(q), torch.empty_like(k)
            qkr.fused_qk_norm_rope([(q, k, g, g)], q2, k2, w.rot, w.pairing, w.eps,
                                   a_tab if i % 2 else a_pos)
            q, k = q2, k2
        return q, k

    (q1, k1), (q0, k0) = _both(run)
    assert torch.equal(_bits(q1), _bits(q0))
    assert torch.equal(_bits(k1), _bits(k0))


def test_mrope_in_place_chain():
    w = W.config4(T=777)
    q0 = to_dev(w.streams[0].q)
    k0 = to_dev(w.streams[0].k)
    pos = to_dev(w.angle.positions)
    inv = to_dev(w.angle.inv_freq)

    def run():
        q, k = q0.clone(), k0.clone()
        for _ in range(16):
            qkr.mrope_apply(q, k, q, k, pos, inv, 128, W.SECTIONS_INTERLEAVED, (24, 20, 20), 0)
        return q, k

    (q1, k1), (q2, k2) = _both(run)
    assert torch.equal(_bits(q1), _bits(q2))
    assert torch.equal(_bits(k1), _bits(k2))


@pytest.mark.parametrize("R,hidden", [(1, 5120), (3, 8192), (700, 2048)])
def test_rms_residual_chain(R, hidden):
    """The residual accumulates x over 20 calls: res_n = bf16(x + res_(n-1))."""
    w = W.config2(R=R, hidden=hidden, seed=93)
    x = to_dev(w.x)
    g = to_dev(w.gamma)
    n = 20

    def run():
        res = to_dev(w.residual).clone()
        out = torch.empty_like(x)
        for _ in range(n):
            qkr.rms_norm_residual(x, res, g, out, w.eps)
        return res, out

    (r1, o1), (r0, o0) = _both(run)
    assert torch.equal(_bits(r1), _bits(r0))
    assert torch.equal(_bits(o1), _bits(o0))
    # the oracle's residual stream after the same n accumulations
    ref = oracle.bits(w.residual)
    for _ in range(n):
        ref, ref_out = oracle.rms_norm_residual(w.x, ref, w.gamma, w.eps)
    assert np.array_equal(oracle.bits(r1), ref)
    assert_bf16_close(o1, ref_out, "rms chain out")


def test_launch_record_reports_overlap():
    x = torch.randn(4, 1024, device="cuda").to(torch.bfloat16)
    res = torch.zeros_like(x)
    g = torch.ones(1024, device="cuda", dtype=torch.bfloat16)
    try:
        for on in (False, True):
            qkr.launch_overlap(on)
            qkr.rms_norm_residual(x, res, g, torch.empty_like(x), 1e-6)
            assert qkr.last_launch()["overlap"] == int(on)
    finally:
        qkr.launch_overlap(True)
    with pytest.raises(qkr.QkrError):
        qkr._check(qkr.lib().qkr_launch_overlap(2))
