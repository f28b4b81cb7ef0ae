"""GPU parity of the eager-chain rounding preset (QKR_FLAG_EAGER_ROUNDING).

vllm-omni #7600's numerics follow-up measures a preset that keeps the rounding
points of the unfused RMSNorm and RoPE chain; vLLM #26234 quotes the
rms_norm_kernel line that fixes them: the normalised value is cast to bf16,
then multiplied by the bf16 weight with a bf16 result.  The kernels are
compared with the oracle's eager contract (tests/golden/eager_rounding.txt pins
it), at full size on the joint text/image configuration with both pairings, on
the single-stream configuration, on every kernel and layout, and against the
single-rounding contract it must differ from.
"""
import numpy as np
import pytest
import torch

import mrope_qk_norm_b200 as qkr
import oracle
import workloads as W
from tests._gpu_util import Guarded, assert_bf16_close_or_tie, to_dev
from tests.test_gpu_fused import run_fused

pytestmark = pytest.mark.gpu

EAGER = 2  # QKR_FLAG_EAGER_ROUNDING


def _check(w, flags, what):
    q, k = run_fused(w, flags)
    rq, rk, tq, tk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps,
                                         w.angle, norm=w.norm,
                                         round_normalized=flags == qkr.FLAG_ROUND_NORMALIZED_BF16,
                                         eager_rounding=flags == EAGER, return_ties=True)
    sq = assert_bf16_close_or_tie(q, rq, tq, what + " q")
    sk = assert_bf16_close_or_tie(k, rk, tk, what + " k")
    return q, k, sq, sk


def test_flag_value_matches_the_header():
    assert qkr.FLAG_EAGER_ROUNDING == EAGER


@pytest.mark.parametrize("pairing", [W.PAIRING_GPTJ, W.PAIRING_NEOX])
@pytest.mark.parametrize("flags", [EAGER, 1])
def test_joint_full_size(pairing, flags):
    """512 + 4096 tokens, 24 heads, D = 128, fp32 table: both rounding
    contracts within tolerance of the oracle's, except at rounding ties."""
    w = W.config3(pairing=pairing)
    q, k, sq, sk = _check(w, flags, "joint")
    # the tie admission is rare: a few in ten thousand of the elements at most
    assert sq["outside_at_ties"] + sk["outside_at_ties"] < 1e-4 * (q.numel() + k.numel())


def test_single_stream_config():
    _check(W.config1(), EAGER, "config1")


def test_eager_differs_from_default_and_single_rounding():
    """The preset changes results where the rounding points matter: the
    outputs differ from the unrounded default and from the single rounding,
    and where the preset changes an output, the change goes the oracle's
    way (the preset's value is closer to the oracle's preset value than the
    default's is)."""
    w = W.config3(seed=41, T_txt=40, img_h=8, img_w=8, H=8, D=128)
    qe, _ = run_fused(w, EAGER)
    q0, _ = run_fused(w, 0)
    q1, _ = run_fused(w, 1)
    e, z, o = (x.float().cpu().numpy().astype(np.float64) for x in (qe, q0, q1))
    assert (e != z).mean() > 0.01 and (e != o).mean() > 0.001
    re_, _ = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle,
                                 eager_rounding=True)
    re_ = re_.reshape(e.shape)
    m = e != z
    closer = np.abs(e[m] - re_[m]) <= np.abs(z[m] - re_[m])
    assert closer.mean() > 0.8, closer.mean()


def _shape_runs(w, flags):
    outs = []
    try:
        for pipe, u in [(1, 1), (1, 2), (1, 4), (3, 2), (3, 4)]:
            qkr.tune_rope(pipe, u, 0, 0)
            outs.append(run_fused(w, flags))
    finally:
        qkr.tune_rope(0, 0, 0, 0)
    return outs


@pytest.mark.parametrize("D,rot,pairing", [(128, 128, W.PAIRING_GPTJ), (128, 128, W.PAIRING_NEOX),
                                           (80, 64, W.PAIRING_NEOX), (64, 22, W.PAIRING_GPTJ),
                                           (256, 96, W.PAIRING_NEOX), (64, 20, W.PAIRING_NEOX)])
def test_every_kernel_and_layout(D, rot, pairing):
    """Item kernel at several head blocks, streaming kernel and (rot % 16 != 0
    NeoX) the exchange kernel: the same bits for the preset on every shape of
    one kernel, and the oracle's values up to rounding ties."""
    T = 45
    pos = np.random.default_rng(D * 7 + rot).integers(0, 60000, T).astype(np.int32)
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos[None],
                      inv_freq=W.inv_freq(1e4, max(rot // 2, 1), max(rot, 2)).numpy())
    w = W.random_rope_case(900 + D + rot, [T], 6, 3, D, rot, pairing, A)
    if rot % 16 and pairing == W.PAIRING_NEOX:
        _check(w, EAGER, "exchange D=%d rot=%d" % (D, rot))
        assert qkr.last_launch()["kernel_name"] == "rope_exchange"
        return
    outs = _shape_runs(w, EAGER)
    for q, k in outs[1:]:
        assert torch.equal(q.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(k.view(torch.int16), outs[0][1].view(torch.int16))
    _check(w, EAGER, "D=%d rot=%d" % (D, rot))


def test_mrope_and_set_rows_take_the_preset():
    """mrope_apply with gammas and rope_set_rows accept the preset and agree
    with fused_qk_norm_rope's rows (same rounding points), and refuse it
    without gammas."""
    w = W.config4(seed=43, T=300, Hq=4, Hkv=2)
    s = w.streams[0]
    q, k = to_dev(s.q), to_dev(s.k)
    pos, inv = to_dev(w.angle.positions), to_dev(w.angle.inv_freq)
    gq = to_dev(W.bf16_uniform((w.D,), 0.5, 1.5, torch.Generator().manual_seed(44)))
    gk = to_dev(W.bf16_uniform((w.D,), 0.5, 1.5, torch.Generator().manual_seed(45)))
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    qkr.mrope_apply(q, k, qo, ko, pos, inv, w.rot, w.angle.section_mode, w.angle.sections,
                    w.pairing, gamma_q=gq, gamma_k=gk, eps=w.eps, flags=EAGER)
    torch.cuda.synchronize()
    st = W.StreamInputs(s.q, s.k, gq.cpu(), gk.cpu())
    rq, rk, tq, tk = oracle.qk_norm_rope([st], w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps,
                                         w.angle, eager_rounding=True, return_ties=True)
    assert_bf16_close_or_tie(qo, rq, tq, "mrope eager q")
    assert_bf16_close_or_tie(ko, rk, tk, "mrope eager k")
    T = q.shape[0]
    cache = Guarded((T + 7, w.Hk, w.D))
    rid = torch.randperm(T + 7, generator=torch.Generator().manual_seed(46))[:T].to("cuda")
    qkr.rope_set_rows(k, cache.tensor, rid, pos, inv, w.rot, w.angle.section_mode,
                      w.angle.sections, w.pairing, gamma=gk, eps=w.eps, flags=EAGER)
    torch.cuda.synchronize()
    cache.check()
    assert torch.equal(cache.tensor[rid].view(torch.int16), ko.view(torch.int16))
    with pytest.raises(qkr.QkrError):
        qkr.mrope_apply(q, k, qo, ko, pos, inv, w.rot, w.angle.section_mode, w.angle.sections,
                        w.pairing, flags=EAGER)
