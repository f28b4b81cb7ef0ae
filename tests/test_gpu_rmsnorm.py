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
    # a handful of rows cannot fill the GPU one CTA per row: split over a cluster
    assert info["kernel_name"] == "rms_cluster" and info["cluster"] >= 8


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
