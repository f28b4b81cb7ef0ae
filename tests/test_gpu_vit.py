"""GPU parity of vit_mrope_setup and the plane-reading apply half.

Configuration: 8 grids, t in {1, 2}, h and w even in [16, 64], spatial merge
2, inv_freq_t/h/w of lengths 16/24/24 (theta 1e4), (3, N, 64) fp32 planes;
then RMSNorm + NeoX RoPE of Q, K [N, 16, 80] reading the planes with
contiguous sections (16, 24, 24) on rotary dim 64 of head dim 80.
"""
import numpy as np
import pytest
import torch

import mrope_qk_norm_b200 as qkr
import oracle
import workloads as W
from tests._gpu_util import Guarded, assert_bf16_close, assert_plane_close, to_dev

pytestmark = pytest.mark.gpu


def vit_meta(grids):
    """cu_seqlens [G+1] and grids [G, 3] as one int32 upload, like the page's host side."""
    g = np.asarray(grids, dtype=np.int64).reshape(-1, 3)
    cu = np.concatenate([[0], np.cumsum(g[:, 0] * g[:, 1] * g[:, 2])])
    buf = torch.from_numpy(np.concatenate([cu, g.reshape(-1)]).astype(np.int32)).pin_memory()
    dev = buf.to("cuda", non_blocking=True)
    G = g.shape[0]
    return dev[:G + 1], dev[G + 1:].view(G, 3), int(cu[-1])


def run_setup(w: W.VitWorkload):
    cu, grids, N = vit_meta(w.grids)
    P = len(w.inv_t) + len(w.inv_h) + len(w.inv_w)
    cos = Guarded((3, N, P), dtype=torch.float32)
    sin = Guarded((3, N, P), dtype=torch.float32)
    qkr.vit_mrope_setup(to_dev(w.inv_t), to_dev(w.inv_h), to_dev(w.inv_w), cu, grids, N,
                        w.spatial_merge, cos.tensor, sin.tensor)
    torch.cuda.synchronize()
    cos.check()
    sin.check()
    return cos, sin, cu, grids, N


@pytest.mark.parametrize("m", [1, 2, 4])
def test_positions_bit_exact(m):
    w = W.config5()
    grids = [[t, h - h % (2 * m) or 2 * m, ww - ww % (2 * m) or 2 * m] for t, h, ww in w.grids]
    grids += [[3, 4 * m, 2 * m], [1, m, m]]
    cu, dgrids, N = vit_meta(grids)
    out = torch.empty(3, N, dtype=torch.int32, device="cuda")
    qkr.vit_positions(cu, dgrids, N, m, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), oracle.vit_positions(grids, m))


@pytest.mark.parametrize("m,grids", [(2, [[3, 512, 512], [1, 1024, 1024], [2, 6, 10]]),
                                     (4, [[5, 200, 300], [1, 4, 4]]),
                                     (1, [[2, 1023, 1025], [7, 3, 5]])])
def test_positions_large_grids_bit_exact(m, grids):
    """Frames and token indices on both sides of 2^20, where the kernels'
    position derivation switches from its short single-precision division
    (exact below 2^20) to integer division: every position equals the
    oracle's."""
    cu, dgrids, N = vit_meta(grids)
    out = torch.empty(3, N, dtype=torch.int32, device="cuda")
    qkr.vit_positions(cu, dgrids, N, m, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), oracle.vit_positions(grids, m))


def test_setup_config_planes():
    w = W.config5()
    cos, sin, _, _, N = run_setup(w)
    pos = oracle.vit_positions(w.grids, w.spatial_merge)
    rc, rs, written = oracle.vit_planes(pos, w.inv_t, w.inv_h, w.inv_w)
    mask = written.astype(bool)
    gc, gs = cos.tensor.cpu().numpy(), sin.tensor.cpu().numpy()
    assert_plane_close(gc, rc, mask, "cos")
    assert_plane_close(gs, rs, mask, "sin")
    # columns outside each axis's section are never written
    assert np.array_equal(cos.untouched(), ~mask)
    assert np.array_equal(sin.untouched(), ~mask)
    assert qkr.last_launch()["kernel_name"] == "vit_setup"


def test_setup_odd_lengths_and_single_grid():
    w = W.config5(seed=51, grids=[[1, 2, 2]], lens=(3, 5, 1), spatial_merge=2)
    cos, sin, _, _, _ = run_setup(w)
    pos = oracle.vit_positions(w.grids, 2)
    rc, rs, written = oracle.vit_planes(pos, w.inv_t, w.inv_h, w.inv_w)
    mask = written.astype(bool)
    assert_plane_close(cos.tensor.cpu().numpy(), rc, mask, "cos")
    assert_plane_close(sin.tensor.cpu().numpy(), rs, mask, "sin")
    assert np.array_equal(cos.untouched(), ~mask)


def test_setup_many_grids_and_long_axis():
    """More grids than a CTA stages in shared memory (600 > 512) and an axis
    longer than the staged inv_freq (600 > 512): the kernel reads that
    metadata from global memory instead, with the same results."""
    rng = np.random.default_rng(53)
    grids = [[int(rng.integers(1, 3)), 2 * int(rng.integers(1, 3)), 2 * int(rng.integers(1, 3))]
             for _ in range(600)]
    w = W.config5(seed=53, grids=grids, lens=(3, 600, 5), spatial_merge=2)
    cos, sin, _, _, _ = run_setup(w)
    pos = oracle.vit_positions(w.grids, 2)
    rc, rs, written = oracle.vit_planes(pos, w.inv_t, w.inv_h, w.inv_w)
    mask = written.astype(bool)
    assert_plane_close(cos.tensor.cpu().numpy(), rc, mask, "cos")
    assert_plane_close(sin.tensor.cpu().numpy(), rs, mask, "sin")
    assert np.array_equal(cos.untouched(), ~mask)


@pytest.mark.parametrize("lens,m", [((64, 64, 64), 1), ((4, 6, 6), 1), ((16, 24, 24), 4),
                                    ((16, 24, 24), 2), ((3, 5, 7), 2)])
def test_setup_empty_grids_and_narrow_grids(lens, m):
    """Grids with zero frames among at most 32 grids (the kernel finds a
    token's grid by shuffles over the boundaries), merge sizes 1, 2 and 4,
    and grids one merge block wide (8 consecutive tokens of a warp then span
    8 h positions; at merge size 2, two merge blocks in different block
    rows, which the kernel's two-block path handles): planes and positions
    equal the oracle's."""
    grids = [[1, 8 * m, m], [0, 4 * m, 4 * m], [2, 2 * m, 6 * m], [0, m, m], [1, 16 * m, m],
             [1, 4 * m, 4 * m]]
    w = W.config5(seed=57, grids=grids, lens=lens, spatial_merge=m)
    cos, sin, cu, dgrids, N = run_setup(w)
    pos = oracle.vit_positions(w.grids, m)
    rc, rs, written = oracle.vit_planes(pos, w.inv_t, w.inv_h, w.inv_w)
    mask = written.astype(bool)
    assert_plane_close(cos.tensor.cpu().numpy(), rc, mask, "cos")
    assert_plane_close(sin.tensor.cpu().numpy(), rs, mask, "sin")
    assert np.array_equal(cos.untouched(), ~mask)
    out = torch.empty(3, N, dtype=torch.int32, device="cuda")
    qkr.vit_positions(cu, dgrids, N, m, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), pos)


def test_setup_empty_grid_list():
    inv = torch.ones(4, dtype=torch.float32, device="cuda")
    e32 = torch.empty(0, dtype=torch.int32, device="cuda")
    cu = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(3, 0, 12, dtype=torch.float32, device="cuda")
    qkr.vit_mrope_setup(inv, inv, inv, cu, e32.view(0, 3), 0, 2, out, out)
    assert qkr.last_launch()["launches"] == 0


def _apply(w, cos, sin, N, D, rot):
    q, k = to_dev(w.q), to_dev(w.k)
    gq, gk = to_dev(w.gamma_q), to_dev(w.gamma_k)
    qo, ko = Guarded((N, q.shape[1], D)), Guarded((N, k.shape[1], D))
    secs = (len(w.inv_t), len(w.inv_h), len(w.inv_w))
    a = qkr.angle_table(cos, sin, W.SECTIONS_CONTIGUOUS, secs)
    qkr.fused_qk_norm_rope([(q, k, gq, gk)], qo.tensor, ko.tensor, rot, W.PAIRING_NEOX, w.eps, a)
    torch.cuda.synchronize()
    qo.check()
    ko.check()
    return qo.tensor, ko.tensor


@pytest.mark.parametrize("D,rot", [(80, 64), (128, 128)])
def test_setup_then_apply(D, rot):
    w = W.config5(D=D, rot=rot)
    cos, sin, _, _, N = run_setup(w)
    qo, ko = _apply(w, cos.tensor, sin.tensor, N, D, rot)
    # the oracle applies from its own planes (untouched cells are NaN there
    # and never read: every pair reads its own axis's section column)
    pos = oracle.vit_positions(w.grids, w.spatial_merge)
    rc, rs, _ = oracle.vit_planes(pos, w.inv_t, w.inv_h, w.inv_w)
    secs = (len(w.inv_t), len(w.inv_h), len(w.inv_w), 0)
    A = W.AngleInputs(kind=W.ANGLE_TABLE, section_mode=W.SECTIONS_CONTIGUOUS, sections=secs,
                      cos=rc, sin=rs)
    s = W.StreamInputs(w.q, w.k, w.gamma_q, w.gamma_k)
    rq, rk = oracle.qk_norm_rope([s], w.q.shape[1], w.k.shape[1], D, rot, W.PAIRING_NEOX, w.eps, A)
    assert not np.isnan(rq).any()
    assert_bf16_close(qo, rq, "apply q")
    assert_bf16_close(ko, rk, "apply k")
