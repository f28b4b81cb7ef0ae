"""GPU parity of rms_norm_residual against the CPU oracle.

Decode configuration R in {1, 32} x hidden 5120 plus the row sweep
R in {1 .. 16384} x hidden {2048, 4096, 8192}; the updated residual stream
is compared bit for bit, the normalised output within the bf16 tolerance.
"""
import numpy as np
import pytest
import torch

import mrope_qk_norm_b200 as qkr
import oracle
import workloads as W
from tests._gpu_util import Guarded, assert_bf16_close, to_dev

pytestmark = pytest.mark.gpu


def run_rms(w, out_is_x=False):
    x = to_dev(w.x)
    res_g = Guarded(w.residual.shape)
    res_g.tensor.copy_(to_dev(w.residual))
    out_g = None
    if out_is_x:
        out = x
    else:
        out_g = Guarded(w.x.shape)
        out = out_g.tensor
    qkr.rms_norm_residual(x, res_g.tensor, to_dev(w.gamma), out, w.eps)
    torch.cuda.synchronize()
    res_g.check()
    if out_g:
        out_g.check()
    return res_g.tensor, out


def check(w, rows=None, out_is_x=False):
    res, out = run_rms(w, out_is_x)
    info = qkr.last_launch()
    x, r = w.x, w.residual
    if rows is not None:
        idx = torch.from_numpy(np.asarray(rows, dtype=np.int64))
        x, r = x[idx], r[idx]
        res, out = res[idx.cuda()], out[idx.cuda()]
    rb, ro = oracle.rms_norm_residual(x, r, w.gamma, w.eps)
    got_bits = res.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got_bits, rb), "residual stream not bit-exact"
    assert_bf16_close(out, ro, w.name)
    return info


@pytest.mark.parametrize("R", [1, 32])
def test_decode_config(R):
    info = check(W.config2(R=R, hidden=5120))
    # a decode row of 5120 fits one CTA with every vector in flight at once
    # (640 threads x one 16-byte vector of x and of the residual)
    assert info["kernel_name"] == "rms_rows" and info["block"] == 640 and info["slots"] == 1


@pytest.mark.parametrize("hidden", [16384, 32768, 65536])
@pytest.mark.parametrize("R", [1, 8, 17, 32, 33])
def test_wide_rows_split_over_a_cluster(R, hidden):
    """Rows wider than one CTA's 1024 vectors are split over a thread-block
    cluster at decode sizes (8 CTAs up to 16 rows, 4 up to 32); beyond that,
    one CTA per row."""
    info = check(W.config2(R=R, hidden=hidden, seed=700 + R))
    if R <= 32:
        assert info["kernel_name"] == "rms_cluster" and info["cluster"] == (8 if R <= 16 else 4)
    else:
        assert info["kernel_name"] == "rms_rows"


@pytest.mark.parametrize("R,hidden", [(2, 8192), (5, 4096), (3, 65536)])
def test_every_split_and_width(R, hidden):
    """Every (CTAs per row, threads per CTA) choice: the residual stream is
    bit-identical and the output within tolerance of the oracle."""
    w = W.config2(R=R, hidden=hidden, seed=800 + R)
    try:
        for cs, thr in [(1, 0), (1, 256), (1, 1024), (2, 512), (4, 128), (8, 256), (16, 64),
                        (16, 0)]:
            if hidden // 8 // cs > 8 * (thr or 1024):
                continue
            qkr.tune_rms(cs, thr)
            info = check(w)
            assert info["cluster"] == cs
    finally:
        qkr.tune_rms(0, 0)


@pytest.mark.parametrize("hidden", [2048, 4096, 8192])
@pytest.mark.parametrize("R", [1, 2, 3, 4, 16, 64, 148, 300, 1024, 4096, 16384])
def test_row_sweep(R, hidden):
    w = W.config2(R=R, hidden=hidden, seed=100 + R)
    rows = None
    if R * hidden > 2 ** 24:  # compare a sample of rows at the largest sizes
        rows = np.unique(np.concatenate([[0, R - 1], np.random.default_rng(R).integers(0, R, 200)]))
    check(w, rows)


@pytest.mark.parametrize("hidden", [8, 24, 40, 520, 5128, 65536])
def test_odd_hidden_sizes(hidden):
    for R in (1, 5, 400):
        check(W.config2(R=R, hidden=hidden, seed=hidden + R))


def test_out_aliases_x():
    check(W.config2(R=7, hidden=4096, seed=9), out_is_x=True)


def test_strided_rows():
    w = W.config2(R=9, hidden=1024, seed=10)
    big = torch.zeros(9, 1536, dtype=torch.bfloat16, device="cuda")
    big[:, :1024] = to_dev(w.x)
    res = to_dev(w.residual).clone()
    out = torch.empty(9, 2048, dtype=torch.bfloat16, device="cuda")
    qkr.rms_norm_residual(big[:, :1024], res, to_dev(w.gamma), out[:, 8:1032], w.eps)
    torch.cuda.synchronize()
    rb, ro = oracle.rms_norm_residual(w.x, w.residual, w.gamma, w.eps)
    assert np.array_equal(res.cpu().view(torch.int16).numpy().view(np.uint16), rb)
    assert_bf16_close(out[:, 8:1032], ro, "strided")


def test_deterministic_repeat():
    w = W.config2(R=3, hidden=5120, seed=11)
    _, o1 = run_rms(w)
    _, o2 = run_rms(w)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def _decode_e4m3(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def assert_fp8_codes(got: np.ndarray, ref_vals: np.ndarray, ref_codes: np.ndarray, what=""):
    """Codes must equal the oracle's, except where the oracle's exact value
    lies within 1e-5 (relative) of the midpoint between the oracle's code and
    an adjacent one (the GPU takes the rounding decision from its fp32 value,
    which differs from the fp64 value by a few fp32 ulps); those few may take
    the neighbour."""
    bad = got != ref_codes
    if not bad.any():
        return 0
    gv = _decode_e4m3(got[bad])
    rv = _decode_e4m3(ref_codes[bad])
    v = ref_vals[bad]
    mid = 0.5 * (gv + rv)
    near = np.abs(v - mid) <= 1e-5 * np.abs(mid) + 1e-12
    # adjacent: no representable value strictly between the two codes
    adjacent = np.abs(got[bad].astype(int) - ref_codes[bad].astype(int)) == 1
    ok = near & adjacent
    assert ok.all(), "%s: %d codes differ beyond a rounding tie; first got %s ref %s value %r" % (
        what, int((~ok).sum()), hex(int(got[bad][~ok][0])), hex(int(ref_codes[bad][~ok][0])),
        float(v[~ok][0]))
    assert bad.sum() <= max(2, 1e-4 * got.size), "%s: too many tie flips" % what
    return int(bad.sum())


@pytest.mark.parametrize("R,hidden,with_res,scale", [
    (1, 5120, True, 0.05), (32, 5120, True, 0.05), (1000, 2048, True, 1.0),
    (3, 8192, False, 0.02), (257, 4096, False, 0.5), (64, 2048, True, 1e-3)])
def test_rms_norm_fp8_vs_oracle(R, hidden, with_res, scale):
    w = W.config2(R=R, hidden=hidden, seed=600 + R)
    x = to_dev(w.x)
    res = None
    if with_res:
        res_g = Guarded(w.residual.shape)
        res_g.tensor.copy_(to_dev(w.residual))
        res = res_g.tensor
    guard = 4096
    buf = torch.full((guard + R * hidden + guard,), 0xA5, dtype=torch.uint8, device="cuda")
    out8 = buf[guard:guard + R * hidden].view(R, hidden)
    sc = torch.tensor([scale], dtype=torch.float32, device="cuda")
    qkr.rms_norm_fp8(x, res, to_dev(w.gamma), out8, sc, w.eps)
    torch.cuda.synchronize()
    assert bool((buf[:guard] == 0xA5).all()) and bool((buf[guard + R * hidden:] == 0xA5).all()), \
        "write outside the FP8 output"
    info = qkr.last_launch()
    assert info["kernel_name"] in ("rms_rows", "rms_cluster")
    ref_res, ys, codes = oracle.rms_norm_fp8(w.x, w.residual if with_res else None, w.gamma,
                                             w.eps, scale)
    if with_res:
        res_g.check()
        assert np.array_equal(oracle.bits(res), ref_res), "residual stream not bit-exact"
    got = out8.cpu().numpy()
    assert_fp8_codes(got, ys, codes, "R=%d hidden=%d" % (R, hidden))


@pytest.mark.parametrize("R,hidden", [(1, 5120), (7, 8192), (3, 65536)])
def test_fp8_every_width_bit_identical(R, hidden):
    """One vector per thread (gamma and the scale loaded with the row) and
    several vectors per thread (loaded after the reduction), in one CTA or a
    cluster: the same E4M3 codes and residual stream, bit for bit."""
    w = W.config2(R=R, hidden=hidden, seed=900 + R)
    gamma = to_dev(w.gamma)
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    outs = []
    try:
        for cs, thr in [(1, 1024), (1, 256), (1, 128), (4, 512), (8, 64)]:
            nvec = hidden // 8 // cs
            if nvec > 8 * thr or (nvec + thr - 1) // thr > 8:
                continue
            qkr.tune_rms(cs, thr)
            res = to_dev(w.residual)
            out8 = torch.empty(R, hidden, dtype=torch.uint8, device="cuda")
            qkr.rms_norm_fp8(to_dev(w.x), res, gamma, out8, sc, w.eps)
            torch.cuda.synchronize()
            info = qkr.last_launch()
            outs.append((out8.cpu(), res.view(torch.int16).cpu(), info["slots"], info["cluster"]))
    finally:
        qkr.tune_rms(0, 0)
    assert len({(o[2], o[3]) for o in outs}) >= 2, outs
    for o in outs[1:]:
        assert torch.equal(o[0], outs[0][0]), (o[2], o[3])
        assert torch.equal(o[1], outs[0][1]), (o[2], o[3])
