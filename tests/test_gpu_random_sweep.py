"""Seeded random sweep of fused_qk_norm_rope / mrope_apply geometries vs the oracle.

Each case draws head_dim, rot_dim, pairing, head counts, token counts (one
or two streams, including empty and ragged ones), the angle source (int32
positions or an fp32 table), the section mode (with admissible sections),
norm on/off and the rounding contract.  Every kernel the launcher can pick is
reached this way (PAIRED, VECTOR, EXCHANGE layouts; item, direct-angle and
streaming kernels).  Outputs must match the oracle within the bf16 tolerance
and stay inside their buffers.
"""
import numpy as np
import pytest
import torch

import mrope_qk_norm_b200 as qkr
import oracle
import workloads as W
from tests._gpu_util import Guarded, assert_bf16_close, to_dev

pytestmark = pytest.mark.gpu

MODES = [W.SECTIONS_NONE, W.SECTIONS_CONTIGUOUS, W.SECTIONS_INTERLEAVED,
         W.SECTIONS_INTERLEAVED_QUOTA, W.SECTIONS_IMROPE]


def _sections(rng, mode, P):
    """Admissible sections for P rotated pairs: sum in [P, 2P]; IMROPE may use a
    fourth section; the interleaved modes need non-empty t/h/w sections."""
    if mode == W.SECTIONS_NONE:
        return (0, 0, 0, 0)
    total = int(rng.integers(P, 2 * P + 1))
    if mode == W.SECTIONS_IMROPE:
        cuts = np.sort(rng.integers(0, total + 1, 3))
        s = [cuts[0], cuts[1] - cuts[0], cuts[2] - cuts[1], total - cuts[2]]
    else:
        lo = 1 if mode in (W.SECTIONS_INTERLEAVED, W.SECTIONS_INTERLEAVED_QUOTA) else 0
        if total < 3 * lo:
            total = 3 * lo
        cuts = np.sort(rng.integers(lo, total - lo + 1, 2))
        s = [cuts[0], cuts[1] - cuts[0], total - cuts[1], 0]
        if lo and min(s[:3]) < 1:
            s = [total - 2, 1, 1, 0]
    return tuple(int(v) for v in s)


def _case(seed):
    rng = np.random.default_rng(seed)
    D = int(rng.choice([8, 16, 32, 48, 64, 80, 96, 128, 192, 256]))
    rot = int(rng.choice([0, D, D, D // 2, 2 * int(rng.integers(1, D // 2 + 1))]))
    rot = min(rot - rot % 2, D)
    pairing = int(rng.choice([W.PAIRING_NEOX, W.PAIRING_GPTJ]))
    Hq, Hk = int(rng.integers(1, 9)), int(rng.integers(1, 5))
    two = bool(rng.integers(0, 2))
    Ts = [int(rng.integers(0, 40)), int(rng.integers(1, 90))] if two else [int(rng.integers(1, 130))]
    T = sum(Ts)
    P = rot // 2
    mode = int(rng.choice(MODES)) if P >= 3 else W.SECTIONS_NONE
    secs = _sections(rng, mode, P) if P > 0 else (0, 0, 0, 0)
    rows = 4 if mode == W.SECTIONS_IMROPE else (1 if mode == W.SECTIONS_NONE else 3)
    off = int(rng.integers(0, 5))
    if rng.integers(0, 2) or P == 0:
        pos = rng.integers(0, 60000, (rows, T + off)).astype(np.int32)
        A = W.AngleInputs(kind=W.ANGLE_POSITIONS, section_mode=mode, sections=secs,
                          positions=pos, inv_freq=W.inv_freq(1e4, max(P, 1), max(rot, 2)).numpy(),
                          token_offset=off)
    else:
        planes = rows if mode != W.SECTIONS_NONE else 1
        ang = rng.uniform(-60.0, 60.0, (planes, T + off, P))
        ld = P + int(rng.choice([0, 0, 1, 3]))  # sometimes a padded row pitch
        cos = np.zeros((planes, T + off, ld), np.float32)
        sin = np.zeros_like(cos)
        cos[:, :, :P] = np.cos(ang)
        sin[:, :, :P] = np.sin(ang)
        A = W.AngleInputs(kind=W.ANGLE_TABLE, section_mode=mode, sections=secs, cos=cos,
                          sin=sin, token_offset=off)
    norm = bool(rng.integers(0, 4))  # mostly normalised
    if not norm and (two or A.kind != W.ANGLE_POSITIONS):
        norm = True  # the no-norm entry point (mrope_apply) takes one stream and positions
    w = W.random_rope_case(seed, Ts, Hq, Hk, D, rot, pairing, A, norm=norm)
    flags = qkr.FLAG_ROUND_NORMALIZED_BF16 if norm and rng.integers(0, 4) == 0 else 0
    return w, flags


def _angle(angle, keep):
    if angle.kind == W.ANGLE_POSITIONS:
        pos = to_dev(torch.as_tensor(np.asarray(angle.positions), dtype=torch.int32))
        inv = to_dev(torch.as_tensor(np.asarray(angle.inv_freq), dtype=torch.float32))
        keep += [pos, inv]
        return qkr.angle_positions(pos, inv, angle.section_mode, angle.sections,
                                   angle.token_offset)
    cos = to_dev(torch.as_tensor(angle.cos))
    sin = to_dev(torch.as_tensor(angle.sin))
    keep += [cos, sin]
    return qkr.angle_table(cos, sin, angle.section_mode, angle.sections, angle.token_offset)


@pytest.mark.parametrize("seed", list(range(1000, 1096)))
def test_random_geometry(seed):
    w, flags = _case(seed)
    keep, streams = [], []
    for s in w.streams:
        t = (to_dev(s.q), to_dev(s.k), to_dev(s.gamma_q), to_dev(s.gamma_k))
        keep += list(t)
        streams.append(t)
    T = w.n_tokens
    qo, ko = Guarded((T, w.Hq, w.D)), Guarded((T, w.Hk, w.D))
    a = _angle(w.angle, keep)
    if w.norm:
        qkr.fused_qk_norm_rope(streams, qo.tensor, ko.tensor, w.rot, w.pairing, w.eps, a, flags)
    else:
        # no norm: the mrope_apply entry point (single stream, positions)
        pos = to_dev(torch.as_tensor(np.asarray(w.angle.positions), dtype=torch.int32))
        inv = to_dev(torch.as_tensor(np.asarray(w.angle.inv_freq), dtype=torch.float32))
        qkr.mrope_apply(streams[0][0], streams[0][1], qo.tensor, ko.tensor, pos, inv, w.rot,
                        w.angle.section_mode, w.angle.sections, w.pairing,
                        token_offset=w.angle.token_offset, eps=w.eps)
    torch.cuda.synchronize()
    qo.check()
    ko.check()
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle,
                                 norm=w.norm, round_normalized=bool(flags))
    what = "seed %d D=%d rot=%d pairing=%d mode=%d kind=%d %s" % (
        seed, w.D, w.rot, w.pairing, w.angle.section_mode, w.angle.kind,
        qkr.last_launch()["kernel_name"])
    assert_bf16_close(qo.tensor, rq, what + " q")
    assert_bf16_close(ko.tensor, rk, what + " k")
