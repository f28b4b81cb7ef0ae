"""GPU parity of mrope_apply (multi-section RoPE) against the CPU oracle.

Full interleaved configuration: T=8192, Hq=16, Hkv=8, D=128, sections
(24, 20, 20), three independent position rows in [0, 8192), theta=5e6, NeoX,
also as two chunked launches split at token 2457, each with a token offset into the
full-length position rows.  Section maps and chunking are checked bit-exactly.
"""
import numpy as np
import pytest
import torch

import mrope_qk_norm_b200 as qkr
import oracle
import workloads as W
from tests._gpu_util import Guarded, assert_bf16_close, to_dev

pytestmark = pytest.mark.gpu


def _dev_inputs(w):
    s = w.streams[0]
    return (to_dev(s.q), to_dev(s.k), to_dev(w.angle.positions), to_dev(w.angle.inv_freq))


def run_mrope(w, chunks=None, norm=False, flags=0, inplace=False):
    q, k, pos, inv = _dev_inputs(w)
    T = q.shape[0]
    gq = to_dev(w.streams[0].gamma_q) if norm else None
    gk = to_dev(w.streams[0].gamma_k) if norm else None
    if inplace:
        qo, ko = q, k
    else:
        qo_g, ko_g = Guarded(q.shape), Guarded(k.shape)
        qo, ko = qo_g.tensor, ko_g.tensor
    for t0, t1 in (chunks or [(0, T)]):
        qkr.mrope_apply(q[t0:t1], k[t0:t1], qo[t0:t1], ko[t0:t1], pos, inv, w.rot,
                        w.angle.section_mode, w.angle.sections, w.pairing, token_offset=t0,
                        gamma_q=gq, gamma_k=gk, eps=w.eps, flags=flags)
    torch.cuda.synchronize()
    if not inplace:
        qo_g.check()
        ko_g.check()
    return qo, ko


def oracle_mrope(w, norm=False):
    return oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle,
                               norm=norm)


@pytest.mark.parametrize("mode", [W.SECTIONS_INTERLEAVED, W.SECTIONS_INTERLEAVED_QUOTA,
                                  W.SECTIONS_IMROPE, W.SECTIONS_CONTIGUOUS])
def test_config_full_size(mode):
    w = W.config4(section_mode=mode)
    q, k = run_mrope(w)
    rq, rk = oracle_mrope(w)
    assert_bf16_close(q, rq, "mrope q")
    assert_bf16_close(k, rk, "mrope k")
    assert qkr.last_launch()["kernel_name"] == "rope_paired"
    # the same launch split at token 2457 with a token offset is bit-identical
    qc, kc = run_mrope(w, chunks=[(0, 2457), (2457, 8192)])
    assert torch.equal(q.view(torch.int16), qc.view(torch.int16))
    assert torch.equal(k.view(torch.int16), kc.view(torch.int16))


@pytest.mark.parametrize("T", [2, 300, 2457, 4000, 5735, 8192])
def test_chunk_token_counts(T):
    # the token counts of the fork's known-answer cases; random chunk splits
    w = W.config4(seed=40 + T, T=T, Hq=4, Hkv=2)
    q, k = run_mrope(w)
    rq, rk = oracle_mrope(w)
    assert_bf16_close(q, rq, "T=%d q" % T)
    assert_bf16_close(k, rk, "T=%d k" % T)
    cuts = sorted(set([0, T] + list(np.random.default_rng(T).integers(1, T, 3))))
    qc, kc = run_mrope(w, chunks=list(zip(cuts[:-1], cuts[1:])))
    assert torch.equal(q.view(torch.int16), qc.view(torch.int16))
    assert torch.equal(k.view(torch.int16), kc.view(torch.int16))


def test_equal_rows_collapse_to_plain_rope_bit_exact():
    w = W.config4(seed=44, T=1000, Hq=4, Hkv=2)
    same = w.angle.positions[:1].repeat(3, 1)
    w.angle.positions = same
    q, k = run_mrope(w)
    plain = W.config4(seed=44, T=1000, Hq=4, Hkv=2)
    plain.angle = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=same[:1].contiguous(),
                                inv_freq=w.angle.inv_freq)
    qp, kp = run_mrope(plain)
    assert torch.equal(q.view(torch.int16), qp.view(torch.int16))
    assert torch.equal(k.view(torch.int16), kp.view(torch.int16))
    # distinct rows must not collapse (interleaved mode differs from plain rope)
    w2 = W.config4(seed=44, T=1000, Hq=4, Hkv=2)
    q2, _ = run_mrope(w2)
    assert not torch.equal(q2.view(torch.int16), qp.view(torch.int16))


def test_section_map_kernel_bit_exact():
    out = torch.empty(256, dtype=torch.int8, device="cuda")
    rng = np.random.default_rng(5)
    cases = [(W.SECTIONS_INTERLEAVED, (24, 20, 20, 0), 64),
             (W.SECTIONS_INTERLEAVED_QUOTA, (24, 20, 20, 0), 64),
             (W.SECTIONS_IMROPE, (24, 20, 20, 0), 64),
             (W.SECTIONS_CONTIGUOUS, (16, 24, 24, 0), 64),
             (W.SECTIONS_NONE, (0, 0, 0, 0), 64)]
    for P in range(1, 40):
        for _ in range(6):
            mode = int(rng.integers(1, 5))
            s = rng.multinomial(int(rng.integers(P, 2 * P + 1)), [0.3, 0.3, 0.3, 0.1] if mode == 4
                                else [1 / 3] * 3)
            s = tuple(int(v) for v in s) + ((0,) if mode != 4 else ())
            cases.append((mode, s, P))
    for mode, s, P in cases:
        qkr.section_map(mode, s, P, out)
        got = out[:P].cpu().numpy()
        assert np.array_equal(got, oracle.section_map(mode, s, P)), (mode, s, P)


def test_inplace_equals_out_of_place():
    w = W.config4(seed=45, T=777, Hq=6, Hkv=2)
    q, k = run_mrope(w)
    qi, ki = run_mrope(w, inplace=True)
    assert torch.equal(q.view(torch.int16), qi.view(torch.int16))
    assert torch.equal(k.view(torch.int16), ki.view(torch.int16))


def test_with_norm_and_rounding_contract():
    w = W.config4(seed=46, T=515, Hq=4, Hkv=2)
    g = torch.Generator().manual_seed(46)
    w.streams[0].gamma_q = W.bf16_uniform((128,), 0.5, 1.5, g)
    w.streams[0].gamma_k = W.bf16_uniform((128,), 0.5, 1.5, g)
    q, k = run_mrope(w, norm=True)
    rq, rk = oracle_mrope(w, norm=True)
    assert_bf16_close(q, rq, "norm q")
    assert_bf16_close(k, rk, "norm k")
    q, k = run_mrope(w, norm=True, flags=qkr.FLAG_ROUND_NORMALIZED_BF16)
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle,
                                 norm=True, round_normalized=True)
    assert_bf16_close(q, rq, "round-normalised q")
    assert_bf16_close(k, rk, "round-normalised k")


def test_gptj_sections_and_partial_rotary():
    g = torch.Generator().manual_seed(47)
    T, Hq, Hk, D, rot = 129, 3, 1, 128, 96
    P = rot // 2
    q, k = W.bf16_normal((T, Hq, D), g), W.bf16_normal((T, Hk, D), g)
    pos = W.random_positions(3, T, 0, 5000, 47)
    for pairing in (W.PAIRING_GPTJ, W.PAIRING_NEOX):
        A = W.AngleInputs(kind=W.ANGLE_POSITIONS, section_mode=W.SECTIONS_CONTIGUOUS,
                          sections=(16, 16, 16, 0), positions=pos,
                          inv_freq=W.inv_freq(1e4, P, rot))
        ones = torch.ones(D, dtype=torch.bfloat16)
        w = W.RopeWorkload("partial", [W.StreamInputs(q, k, ones, ones)], Hq, Hk, D, rot,
                           pairing, 1e-6, A, norm=False)
        qo, ko = run_mrope(w)
        rq, rk = oracle_mrope(w)
        assert_bf16_close(qo, rq, "partial q")
        assert_bf16_close(ko, rk, "partial k")


def test_packed_qkv_in_place():
    """Q and K rotated in place as column windows of one packed [T, 3, H, D]
    buffer: their byte ranges interleave but share no element, so the call is
    accepted, equals the fresh-output launch bit for bit and leaves V alone."""
    w = W.config4(seed=91, T=300, Hq=8, Hkv=8)
    q, k, pos, inv = _dev_inputs(w)
    T, H, D = q.shape
    g = torch.Generator(device="cuda").manual_seed(92)
    buf = torch.empty(T, 3, H, D, dtype=torch.bfloat16, device="cuda")
    buf[:, 0].copy_(q)
    buf[:, 1].copy_(k)
    buf[:, 2].copy_(torch.randn(T, H, D, device="cuda", generator=g).to(torch.bfloat16))
    v_before = buf[:, 2].clone()
    qv, kv = buf[:, 0], buf[:, 1]
    qkr.mrope_apply(qv, kv, qv, kv, pos, inv, w.rot, w.angle.section_mode, w.angle.sections,
                    w.pairing)
    torch.cuda.synchronize()
    ref_q, ref_k = run_mrope(w)
    assert torch.equal(qv.view(torch.int16), ref_q.view(torch.int16))
    assert torch.equal(kv.view(torch.int16), ref_k.view(torch.int16))
    assert torch.equal(buf[:, 2].view(torch.int16), v_before.view(torch.int16))


@pytest.mark.parametrize("pipeline", [0, 1, 3])
def test_row_offsets_past_2_31(pipeline):
    """Row offsets the kernel forms past 2^31 elements on the positions path:
    Q is a view whose token stride puts token 2 beyond 2^31 elements from its
    base.  Item kernel and streaming kernel alike equal the contiguous launch
    bit for bit.  About 4.3 GiB for the wide view."""
    free, _ = torch.cuda.mem_get_info()
    if free < 8 * 2 ** 30:
        pytest.skip("needs 8 GiB of free device memory")
    w = W.config4(seed=93, T=3, Hq=2, Hkv=1)
    q, k, pos, inv = _dev_inputs(w)
    T, Hq, D = q.shape
    ts = 2 ** 30 + 8
    assert (T - 1) * ts > 2 ** 31
    big = torch.empty((T - 1) * ts + Hq * D, dtype=torch.bfloat16, device="cuda")
    qw = big.as_strided((T, Hq, D), (ts, D, 1))
    qw.copy_(q)
    try:
        qkr.tune_rope(pipeline, 0, 0, 0)
        ref_q, ref_k = run_mrope(w)
        qo, ko = torch.empty_like(q), torch.empty_like(k)
        qkr.mrope_apply(qw, k, qo, ko, pos, inv, w.rot, w.angle.section_mode, w.angle.sections,
                        w.pairing)
        torch.cuda.synchronize()
        name = qkr.last_launch()["kernel_name"]
    finally:
        qkr.tune_rope(0, 0, 0, 0)
    assert name == "rope_paired"
    assert torch.equal(qo.view(torch.int16), ref_q.view(torch.int16))
    assert torch.equal(ko.view(torch.int16), ref_k.view(torch.int16))
    del big, qw
    torch.cuda.empty_cache()
