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


def test_independent_chunks_overlap_and_stay_ordered():
    """QKR_FLAG_INDEPENDENT on the second chunk of a chunked step (it reads
    and writes nothing the first chunk touches): bit-identical to the whole
    launch, and the next step -- which reads both chunks' outputs -- sees all
    of them.  Run as a chain of steps with no host synchronisation, with the
    overlap switch on (the flag's early start) and off (plain order)."""
    w = W.config4(seed=95, T=3000, Hq=8, Hkv=4)
    s = w.streams[0]
    q0, k0 = to_dev(s.q), to_dev(s.k)
    pos, inv = to_dev(w.angle.positions), to_dev(w.angle.inv_freq)
    T = q0.shape[0]
    cut = 1111

    def step(q, k, chunked):
        qo, ko = torch.empty_like(q), torch.empty_like(k)
        if chunked:
            for i, (t0, t1) in enumerate(((0, cut), (cut, T))):
                qkr.mrope_apply(q[t0:t1], k[t0:t1], qo[t0:t1], ko[t0:t1], pos, inv, w.rot,
                                w.angle.section_mode, w.angle.sections, w.pairing,
                                token_offset=t0, flags=qkr.FLAG_INDEPENDENT if i else 0)
        else:
            qkr.mrope_apply(q, k, qo, ko, pos, inv, w.rot, w.angle.section_mode,
                            w.angle.sections, w.pairing)
        return qo, ko

    def run(chunked):
        q, k = q0, k0
        for _ in range(10):  # each step rotates the previous step's output again
            q, k = step(q, k, chunked)
        return q, k

    (qa, ka), (qb, kb) = _both(lambda: run(True))
    qr, kr = run(False)
    torch.cuda.synchronize()
    for q, k in ((qa, ka), (qb, kb)):
        assert torch.equal(_bits(q), _bits(qr)) and torch.equal(_bits(k), _bits(kr))


def test_independent_flag_on_every_kernel():
    """The flag changes no bits on the item, streaming and exchange kernels,
    fused and rope_set_rows calls, and combines with a rounding flag."""
    pos = np.random.default_rng(96).integers(0, 9000, (1, 77)).astype(np.int32)
    cases = []
    for D, rot, pairing in ((128, 128, W.PAIRING_GPTJ), (128, 128, W.PAIRING_NEOX),
                            (64, 20, W.PAIRING_NEOX)):
        A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos,
                          inv_freq=W.inv_freq(1e4, rot // 2, rot).numpy())
        cases.append(W.random_rope_case(97 + D + rot, [77], 5, 3, D, rot, pairing, A))
    for w in cases:
        s = w.streams[0]
        d = (to_dev(s.q), to_dev(s.k), to_dev(s.gamma_q), to_dev(s.gamma_k))
        a = qkr.angle_positions(to_dev(torch.as_tensor(pos)),
                                to_dev(torch.as_tensor(np.asarray(w.angle.inv_freq))))
        outs = []
        try:
            for pipe in (1, 3):
                qkr.tune_rope(pipe, 0, 0, 0)
                for flags in (0, qkr.FLAG_INDEPENDENT, 2, 2 | qkr.FLAG_INDEPENDENT):
                    qo, ko = torch.empty_like(d[0]), torch.empty_like(d[1])
                    qkr.fused_qk_norm_rope([d], qo, ko, w.rot, w.pairing, w.eps, a, flags)
                    outs.append((flags, qo, ko))
        finally:
            qkr.tune_rope(0, 0, 0, 0)
        torch.cuda.synchronize()
        for flags, qo, ko in outs:
            ref = [o for o in outs if o[0] == (flags & 2)][0]
            assert torch.equal(_bits(qo), _bits(ref[1])) and torch.equal(_bits(ko), _bits(ref[2]))
