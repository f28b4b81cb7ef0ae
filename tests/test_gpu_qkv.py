"""GPU parity of fused_qkv_norm_rope: the joint Q/K/V form of the fused op.

Q and K must equal fused_qk_norm_rope's outputs bit for bit (and the oracle
within the bf16 tolerance); V must be the text-first concatenation of the
streams' V rows, bit for bit.  Covered: the joint configuration at full size
with V, zero-copy views into packed [T, 3, H, D] QKV buffers, every kernel
path (direct table reads, staged table, positions / streaming kernel, the
exchange kernel for rot_dim % 16 != 0, the forced item kernel) and Hv != Hk.
"""
import numpy as np
import pytest
import torch

import mrope_qk_norm_b200 as qkr
import oracle
import workloads as W
from tests._gpu_util import Guarded, assert_bf16_close, to_dev

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.contiguous().view(torch.int16)


def _angle(angle, keep):
    if angle.kind == W.ANGLE_POSITIONS:
        pos = to_dev(torch.as_tensor(np.asarray(angle.positions), dtype=torch.int32))
        inv = to_dev(torch.as_tensor(np.asarray(angle.inv_freq), dtype=torch.float32))
        keep += [pos, inv]
        return qkr.angle_positions(pos, inv, angle.section_mode, angle.sections,
                                   angle.token_offset)
    cos = to_dev(torch.as_tensor(np.asarray(angle.cos), dtype=torch.float32))
    sin = to_dev(torch.as_tensor(np.asarray(angle.sin), dtype=torch.float32))
    keep += [cos, sin]
    return qkr.angle_table(cos, sin, angle.section_mode, angle.sections, angle.token_offset)


def run_qkv(w, v_host, Hv, packed=False):
    """Joint Q/K/V launch; v_host: per-stream [T_s, Hv, D] bf16 (CPU).  With
    packed=True every stream's Q, K and V are views into one [T, 3, H, D]
    buffer (needs Hq == Hk == Hv)."""
    keep, streams = [], []
    for s, v in zip(w.streams, v_host):
        if packed:
            buf = torch.stack([s.q, s.k, v], dim=1)  # [T, 3, H, D]
            d = to_dev(buf)
            keep.append(d)
            q, k, vv = d[:, 0], d[:, 1], d[:, 2]
        else:
            q, k, vv = to_dev(s.q), to_dev(s.k), to_dev(v)
        gq, gk = to_dev(s.gamma_q), to_dev(s.gamma_k)
        keep += [q, k, vv, gq, gk]
        streams.append(qkr.stream_desc(q, k, gq, gk, vv))
    T = w.n_tokens
    qo, ko, vo = Guarded((T, w.Hq, w.D)), Guarded((T, w.Hk, w.D)), Guarded((T, Hv, w.D))
    a = _angle(w.angle, keep)
    qkr.fused_qkv_norm_rope(streams, qo.tensor, ko.tensor, vo.tensor, w.rot, w.pairing, w.eps,
                            a)
    torch.cuda.synchronize()
    for g in (qo, ko, vo):
        g.check()
    return qo.tensor, ko.tensor, vo.tensor


def run_qk(w):
    keep, streams = [], []
    for s in w.streams:
        t = (to_dev(s.q), to_dev(s.k), to_dev(s.gamma_q), to_dev(s.gamma_k))
        keep += list(t)
        streams.append(t)
    T = w.n_tokens
    qo = torch.empty(T, w.Hq, w.D, dtype=torch.bfloat16, device="cuda")
    ko = torch.empty(T, w.Hk, w.D, dtype=torch.bfloat16, device="cuda")
    qkr.fused_qk_norm_rope(streams, qo, ko, w.rot, w.pairing, w.eps, _angle(w.angle, keep))
    torch.cuda.synchronize()
    return qo, ko


def _v_inputs(w, Hv, seed):
    g = torch.Generator().manual_seed(seed)
    return [W.bf16_normal((s.q.shape[0], Hv, w.D), g) for s in w.streams]


def check(w, Hv, seed, packed=False, what=""):
    v_host = _v_inputs(w, Hv, seed)
    q, k, v = run_qkv(w, v_host, Hv, packed)
    q2, k2 = run_qk(w)
    assert torch.equal(_bits(q), _bits(q2)), what + ": Q differs from the Q/K-only op"
    assert torch.equal(_bits(k), _bits(k2)), what + ": K differs from the Q/K-only op"
    assert np.array_equal(oracle.bits(v), oracle.joint_v(v_host)), what + ": V not copied"
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle)
    assert_bf16_close(q, rq, what + " q")
    assert_bf16_close(k, rk, what + " k")
    return qkr.last_launch()


@pytest.mark.parametrize("pairing", [W.PAIRING_GPTJ, W.PAIRING_NEOX])
def test_joint_qkv_full_size(pairing):
    w = W.config3(pairing=pairing)
    rec = check(w, 24, 301, what="joint qkv")
    assert rec["launches"] == 1


def test_packed_qkv_views():
    w = W.config3(seed=303, T_txt=37, img_h=9, img_w=10, H=8, D=128)
    check(w, 8, 303, packed=True, what="packed qkv")


@pytest.mark.parametrize("D,rot,pairing,Hv", [
    (128, 128, W.PAIRING_NEOX, 3),   # positions: streaming kernel
    (80, 64, W.PAIRING_NEOX, 5),     # pass-through tail
    (64, 20, W.PAIRING_NEOX, 2),     # exchange kernel
    (64, 22, W.PAIRING_GPTJ, 7),     # vector layout with identity pairs
    (256, 256, W.PAIRING_GPTJ, 1),
])
def test_qkv_positions_geometries(D, rot, pairing, Hv):
    T = 53
    pos = np.random.default_rng(D + rot).integers(0, 30000, (1, T)).astype(np.int32)
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos,
                      inv_freq=W.inv_freq(1e4, max(rot // 2, 1), max(rot, 2)).numpy())
    w = W.random_rope_case(400 + D + rot, [T], 6, 2, D, rot, pairing, A)
    check(w, Hv, 401 + D, what="D=%d rot=%d" % (D, rot))


def test_qkv_every_kernel_path():
    """Item kernel with direct and staged table reads, streaming kernel, and
    the forced item kernel on positions: same Q/K bits, V copied."""
    w = W.config3(seed=305, T_txt=21, img_h=5, img_w=9, H=5, D=128, pairing=W.PAIRING_GPTJ)
    v_host = _v_inputs(w, 4, 305)
    ref = run_qkv(w, v_host, 4)
    vref = oracle.joint_v(v_host)
    try:
        for pipe, u in ((1, 1), (1, 2), (1, 4), (3, 1), (3, 2), (3, 4)):
            qkr.tune_rope(pipe, u, 0, 0)
            q, k, v = run_qkv(w, v_host, 4)
            assert torch.equal(_bits(q), _bits(ref[0])), (pipe, u)
            assert torch.equal(_bits(k), _bits(ref[1])), (pipe, u)
            assert np.array_equal(oracle.bits(v), vref), (pipe, u)
    finally:
        qkr.tune_rope(0, 0, 0, 0)


def test_qkv_empty_text_stream():
    w = W.config3(seed=307, T_txt=0, img_h=4, img_w=6, H=3, D=64)
    check(w, 3, 307, what="empty text stream")
