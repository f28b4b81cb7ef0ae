"""GPU parity of rope_set_rows: rotate K rows and scatter them into cache rows.

cache[row_idx[t]] must equal mrope_apply's K output row t bit for bit (same
kernels, same arithmetic) and the oracle within the bf16 tolerance; rows no
index names keep their sentinel; an index outside the cache writes nothing
and raises bit 4 of the device status word.  Covers plain RoPE, the
interleaved config-4 sections, ggml's four-row sector rule (IMROPE), a
chunked launch with a token offset, per-head RMSNorm, and every kernel path.
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


def _case(mode, T=301, H=8, D=128, seed=500):
    return W.config4(seed=seed, T=T, Hq=H, Hkv=H, D=D, section_mode=mode)


def _positions(w):
    pos = to_dev(torch.as_tensor(np.asarray(w.angle.positions), dtype=torch.int32))
    # plain RoPE reads one position row
    return pos[:1].contiguous() if w.angle.section_mode == W.SECTIONS_NONE else pos


def _scatter(w, idx, R, norm=False, t0=0, t1=None, cache=None):
    s = w.streams[0]
    t1 = w.n_tokens if t1 is None else t1
    x = to_dev(s.k)[t0:t1]
    pos = _positions(w)
    inv = to_dev(torch.as_tensor(np.asarray(w.angle.inv_freq), dtype=torch.float32))
    if cache is None:
        cache = Guarded((R, w.Hk, w.D))
    rid = to_dev(torch.as_tensor(idx, dtype=torch.int64))[t0:t1]
    qkr.rope_set_rows(x, cache.tensor, rid, pos, inv, w.rot, w.angle.section_mode,
                      w.angle.sections, w.pairing, token_offset=t0,
                      gamma=to_dev(s.gamma_k) if norm else None, eps=w.eps)
    torch.cuda.synchronize()
    cache.check()
    return cache


def _mrope_k(w, norm=False):
    s = w.streams[0]
    q, k = to_dev(s.q), to_dev(s.k)
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    qkr.mrope_apply(q, k, qo, ko, _positions(w), to_dev(w.angle.inv_freq), w.rot,
                    w.angle.section_mode, w.angle.sections, w.pairing,
                    gamma_q=to_dev(s.gamma_q) if norm else None,
                    gamma_k=to_dev(s.gamma_k) if norm else None, eps=w.eps)
    torch.cuda.synchronize()
    return ko


@pytest.mark.parametrize("mode,norm", [(W.SECTIONS_INTERLEAVED, False),
                                       (W.SECTIONS_IMROPE, False),
                                       (W.SECTIONS_NONE, True),
                                       (W.SECTIONS_CONTIGUOUS, True)])
def test_scatter_matches_mrope_and_oracle(mode, norm):
    w = _case(mode, seed=501 + mode)
    T, R = w.n_tokens, 1000
    idx = np.random.default_rng(7 + mode).permutation(R)[:T]
    cache = _scatter(w, idx, R, norm=norm)
    got = cache.tensor
    ref_k = _mrope_k(w, norm)
    rid = torch.as_tensor(idx, dtype=torch.int64, device="cuda")
    assert torch.equal(_bits(got[rid]), _bits(ref_k)), "scatter != mrope_apply K rows"
    untouched = cache.untouched()
    named = np.zeros(R, dtype=bool)
    named[idx] = True
    assert untouched[~named].all(), "a row no index names was written"
    _, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle,
                                norm=norm)
    ref = oracle.scatter_rows(rk, idx, R)
    assert_bf16_close(got[rid], ref[idx], "scatter")


def test_chunked_scatter_equals_whole():
    w = _case(W.SECTIONS_INTERLEAVED, T=700, seed=511)
    R = 2048
    idx = np.random.default_rng(11).permutation(R)[:700]
    whole = _scatter(w, idx, R).tensor
    cache = Guarded((R, w.Hk, w.D))
    for t0, t1 in ((0, 257), (257, 700)):
        _scatter(w, idx, R, t0=t0, t1=t1, cache=cache)
    assert torch.equal(_bits(cache.tensor), _bits(whole))


def test_scatter_every_kernel_path():
    w = _case(W.SECTIONS_INTERLEAVED, T=97, seed=513)
    R = 300
    idx = np.random.default_rng(13).permutation(R)[:97]
    ref = _scatter(w, idx, R).tensor
    try:
        for pipe, u in ((1, 1), (1, 2), (1, 4), (3, 1), (3, 4)):
            qkr.tune_rope(pipe, u, 0, 0)
            got = _scatter(w, idx, R).tensor
            assert torch.equal(_bits(got), _bits(ref)), (pipe, u)
    finally:
        qkr.tune_rope(0, 0, 0, 0)
    # rot_dim % 16 != 0 (exchange kernel) against the oracle
    pos = np.random.default_rng(15).integers(0, 4000, (1, 61)).astype(np.int32)
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos,
                      inv_freq=W.inv_freq(1e4, 10, 20).numpy())
    w2 = W.random_rope_case(515, [61], 2, 3, 64, 20, W.PAIRING_NEOX, A)
    idx2 = np.random.default_rng(17).permutation(80)[:61]
    c = _scatter(w2, idx2, 80, norm=True)
    assert qkr.last_launch()["kernel_name"] == "rope_exchange"
    _, rk = oracle.qk_norm_rope(w2.streams, w2.Hq, w2.Hk, w2.D, w2.rot, w2.pairing, w2.eps,
                                w2.angle)
    rid = torch.as_tensor(idx2, dtype=torch.int64, device="cuda")
    assert_bf16_close(c.tensor[rid], rk, "exchange scatter")


def test_out_of_range_row_is_skipped_and_reported():
    """The kernel's own bounds check turns an index outside the cache into a
    skipped row plus bit 4 of the status word; every valid row still lands."""
    w = _case(W.SECTIONS_INTERLEAVED, T=40, seed=517)
    R = 64
    idx = np.random.default_rng(19).permutation(R)[:40].astype(np.int64)
    idx[5] = R        # one past the end
    idx[17] = -3      # negative
    assert qkr.device_status(reset=True) == 0
    cache = _scatter(w, idx, R)
    status = qkr.device_status(reset=True)
    assert status & 4
    ref_k = _mrope_k(w)
    good = [t for t in range(40) if 0 <= idx[t] < R]
    rid = torch.as_tensor(idx[good], dtype=torch.int64, device="cuda")
    assert torch.equal(_bits(cache.tensor[rid]), _bits(ref_k[good]))
    named = np.zeros(R, dtype=bool)
    named[idx[good]] = True
    assert cache.untouched()[~named].all()


def test_scatter_full_size():
    """The measured size: 8192 tokens x 8 K heads into a 16384-row cache, in
    the launch shape the launcher picks for it (more than 8 tokens per CTA,
    since a token has only 8 heads, and at most one wave: 14 on 148 SMs)."""
    w = _case(W.SECTIONS_INTERLEAVED, T=8192, seed=521)
    R = 16384
    idx = np.random.default_rng(21).permutation(R)[:8192]
    cache = _scatter(w, idx, R)
    rec = qkr.last_launch()
    assert rec["pipelined"] == 2 and 8 < rec["tokens_per_cta"] <= 16, rec
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert rec["grid"] <= 4 * sms, rec
    rid = torch.as_tensor(idx, dtype=torch.int64, device="cuda")
    assert torch.equal(_bits(cache.tensor[rid]), _bits(_mrope_k(w))), "scatter != mrope_apply"
    assert cache.untouched()[np.setdiff1d(np.arange(R), idx)].all()
    _, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle,
                                norm=False)
    assert_bf16_close(cache.tensor[rid], rk, "full-size scatter")


@pytest.mark.parametrize("hk", [1, 2, 3, 8])
def test_scatter_every_kernel_agrees(hk):
    """The automatic choice, the item kernel with staged angles and the
    streaming kernel give the same bits for a K-only scatter of 1..8 heads
    (3 leaves one head of the last item dead)."""
    w = _case(W.SECTIONS_INTERLEAVED, T=1000, seed=600 + hk, H=hk)
    R = 1500
    idx = np.random.default_rng(hk).permutation(R)[:1000]
    outs = []
    try:
        for pipe in (0, 1, 3):
            qkr.tune_rope(pipe, 0, 0, 0)
            outs.append((_scatter(w, idx, R).tensor.clone(), qkr.last_launch()))
    finally:
        qkr.tune_rope(0, 0, 0, 0)
    for c, rec in outs[1:]:
        assert torch.equal(_bits(c), _bits(outs[0][0])), rec
