"""GPU parity of fused_qk_norm_rope against the CPU oracle.

Covers the single-stream configuration (T=16, H=4, D=64, NeoX, positions
0..15, seed 0), the joint text/image configuration at full size (512 + 4096
tokens, 24 heads, D=128, fp32 [4608, 64] cos/sin table, both pairings), the
2^31-element storage-offset variant on either stream at full size (and row
offsets past 2^31 formed inside the kernel), strided views, the
bf16-rounded-normalised-value contract, every kernel layout, launch shape
and ragged shapes.
"""
import numpy as np
import pytest
import torch

import mrope_qk_norm_b200 as qkr
import oracle
import workloads as W
from tests._gpu_util import Guarded, assert_bf16_close, to_dev

pytestmark = pytest.mark.gpu


def _angle_desc(angle, dev_keep):
    if angle.kind == W.ANGLE_POSITIONS:
        pos = to_dev(torch.as_tensor(np.asarray(angle.positions), dtype=torch.int32))
        inv = to_dev(torch.as_tensor(np.asarray(angle.inv_freq), dtype=torch.float32))
        dev_keep += [pos, inv]
        return qkr.angle_positions(pos, inv, angle.section_mode, angle.sections, angle.token_offset)
    cos = to_dev(torch.as_tensor(np.asarray(angle.cos), dtype=torch.float32))
    sin = to_dev(torch.as_tensor(np.asarray(angle.sin), dtype=torch.float32))
    dev_keep += [cos, sin]
    return qkr.angle_table(cos, sin, angle.section_mode, angle.sections, angle.token_offset)


def run_fused(w: W.RopeWorkload, flags=0, guard=True):
    keep = []
    streams = []
    for s in w.streams:
        q, k, gq, gk = (to_dev(s.q), to_dev(s.k), to_dev(s.gamma_q), to_dev(s.gamma_k))
        keep += [q, k, gq, gk]
        streams.append((q, k, gq, gk))
    T = w.n_tokens
    qo = Guarded((T, w.Hq, w.D))
    ko = Guarded((T, w.Hk, w.D))
    a = _angle_desc(w.angle, keep)
    qkr.fused_qk_norm_rope(streams, qo.tensor, ko.tensor, w.rot, w.pairing, w.eps, a, flags)
    torch.cuda.synchronize()
    qo.check()
    ko.check()
    return qo.tensor, ko.tensor


def check_against_oracle(w, flags=0, what=""):
    q, k = run_fused(w, flags)
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle,
                                 norm=w.norm, round_normalized=bool(flags & 1))
    sq = assert_bf16_close(q, rq, what + " q")
    sk = assert_bf16_close(k, rk, what + " k")
    return q, k, sq, sk


@pytest.mark.parametrize("pairing", [W.PAIRING_NEOX, W.PAIRING_GPTJ])
def test_single_stream_config(pairing):
    w = W.config1(pairing=pairing)
    check_against_oracle(w, what="config1")
    info = qkr.last_launch()
    assert info["kernel_name"] == ("rope_paired" if pairing == W.PAIRING_NEOX else "rope_vector")
    assert info["launches"] == 1


@pytest.mark.parametrize("pairing", [W.PAIRING_GPTJ, W.PAIRING_NEOX])
def test_joint_config_full_size(pairing):
    w = W.config3(pairing=pairing)
    q, k, _, _ = check_against_oracle(w, what="joint")
    # the joint launch equals the two streams launched separately, bit for bit
    txt = W.RopeWorkload("txt", w.streams[:1], w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle)
    img_angle = W.AngleInputs(kind=W.ANGLE_TABLE, cos=w.angle.cos, sin=w.angle.sin,
                              token_offset=w.streams[0].q.shape[0])
    img = W.RopeWorkload("img", w.streams[1:], w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, img_angle)
    qt, kt = run_fused(txt)
    qi, ki = run_fused(img)
    assert torch.equal(q.view(torch.int16), torch.cat([qt, qi]).view(torch.int16))
    assert torch.equal(k.view(torch.int16), torch.cat([kt, ki]).view(torch.int16))


def test_joint_small_ragged_vs_oracle():
    # 37 text + 5x7 image tokens: several CTA tiles and a ragged last tile
    for pairing in (W.PAIRING_GPTJ, W.PAIRING_NEOX):
        w = W.config3(seed=13, T_txt=37, img_h=5, img_w=7, H=6, D=128, pairing=pairing)
        check_against_oracle(w, what="joint small")


def _offset_stream(q, k, off):
    """Copies of q and k placed `off` elements into fresh storage."""
    big_q = torch.empty(off + q.numel(), dtype=torch.bfloat16, device="cuda")
    big_q[off:].copy_(q.reshape(-1))
    big_k = torch.empty(off + k.numel(), dtype=torch.bfloat16, device="cuda")
    big_k[off:].copy_(k.reshape(-1))
    qv, kv = big_q[off:].view(q.shape), big_k[off:].view(k.shape)
    assert qv.storage_offset() == off and kv.storage_offset() == off
    return qv, kv, [big_q, big_k]


def _wide_row_stream(q, k, ts):
    """q and k as the first two column windows of one buffer whose token rows
    are `ts` elements apart, so token t of the stream sits t*ts elements into
    the storage."""
    T, H, D = q.shape
    buf = torch.empty(T, ts, dtype=torch.bfloat16, device="cuda")
    buf[:, :H * D].copy_(q.reshape(T, H * D))
    buf[:, H * D:2 * H * D].copy_(k.reshape(T, H * D))
    qv = buf[:, :H * D].view(T, H, D)
    kv = buf[:, H * D:2 * H * D].view(T, H, D)
    assert qv.stride(0) == ts and kv.stride(0) == ts
    return qv, kv, [buf]


def _run_joint_with(w, which, place):
    """The joint launch with stream `which` placed by `place(q, k)`."""
    keep, streams = [], []
    for i, s in enumerate(w.streams):
        q, k = to_dev(s.q), to_dev(s.k)
        if i == which:
            q, k, big = place(q, k)
            keep += big
        gq, gk = to_dev(s.gamma_q), to_dev(s.gamma_k)
        keep += [q, k, gq, gk]
        streams.append((q, k, gq, gk))
    T = w.n_tokens
    qo = Guarded((T, w.Hq, w.D))
    ko = Guarded((T, w.Hk, w.D))
    a = _angle_desc(w.angle, keep)
    qkr.fused_qk_norm_rope(streams, qo.tensor, ko.tensor, w.rot, w.pairing, w.eps, a)
    torch.cuda.synchronize()
    qo.check()
    ko.check()
    del keep
    return qo.tensor, ko.tensor


@pytest.mark.parametrize("which", [0, 1])
@pytest.mark.parametrize("pairing", [W.PAIRING_GPTJ, W.PAIRING_NEOX])
def test_large_storage_offset_full_size(which, pairing):
    """The joint workload at full size (512 + 4096 tokens, 24 heads, D=128)
    with one stream 2^31 elements into its storage (vllm-omni #7600, 64-bit
    row addressing): equal bit for bit to the launch without the offset and
    within tolerance of the oracle.  Needs about 8.1 GiB for the offset
    stream."""
    free, _ = torch.cuda.mem_get_info()
    if free < 12 * 2 ** 30:
        pytest.skip("needs 12 GiB of free device memory")
    w = W.config3(pairing=pairing)
    assert w.n_tokens == 4608 and w.Hq == 24 and w.D == 128
    ref_q, ref_k = run_fused(w)
    q, k = _run_joint_with(w, which, lambda q, k: _offset_stream(q, k, 2 ** 31))
    assert torch.equal(q.view(torch.int16), ref_q.view(torch.int16))
    assert torch.equal(k.view(torch.int16), ref_k.view(torch.int16))
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle)
    assert_bf16_close(q, rq, "offset q")
    assert_bf16_close(k, rk, "offset k")
    torch.cuda.empty_cache()


@pytest.mark.parametrize("which", [0, 1])
@pytest.mark.parametrize("pairing", [W.PAIRING_GPTJ, W.PAIRING_NEOX])
def test_row_offsets_past_2_31_in_kernel(which, pairing):
    """The kernel's own row addressing past 2^31 elements: the stream's token
    stride is so wide that token t*stride crosses 2^31 inside the launch
    (the storage offset above is added on the host; here the kernel forms
    the large offsets).  Full-size joint workload; about 4.4 GiB for the wide
    stream."""
    free, _ = torch.cuda.mem_get_info()
    if free < 10 * 2 ** 30:
        pytest.skip("needs 10 GiB of free device memory")
    w = W.config3(pairing=pairing)
    T_s = int(w.streams[which].q.shape[0])
    ts = -(-(2 ** 31 + 2 ** 20) // (T_s - 1))
    ts = -(-ts // 8) * 8                      # a multiple of 8 elements
    assert (T_s - 1) * ts > 2 ** 31
    ref_q, ref_k = run_fused(w)
    q, k = _run_joint_with(w, which, lambda q, k: _wide_row_stream(q, k, ts))
    assert torch.equal(q.view(torch.int16), ref_q.view(torch.int16))
    assert torch.equal(k.view(torch.int16), ref_k.view(torch.int16))
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle)
    assert_bf16_close(q, rq, "wide-row q")
    assert_bf16_close(k, rk, "wide-row k")
    torch.cuda.empty_cache()


def test_strided_chunked_qkv_views():
    # Q and K are views into a packed [T, 3, H, D] QKV buffer (zero-copy split).
    g = torch.Generator().manual_seed(21)
    T, H, D = 50, 8, 128
    qkv = W.bf16_normal((T, 3, H, D), g)
    gq = W.bf16_uniform((D,), 0.5, 1.5, g)
    gk = W.bf16_uniform((D,), 0.5, 1.5, g)
    inv = W.inv_freq(1e4, D // 2, D)
    pos = torch.arange(3, 3 + T, dtype=torch.int32).view(1, T)
    dq = to_dev(qkv)
    dgq, dgk, dpos, dinv = to_dev(gq), to_dev(gk), to_dev(pos), to_dev(inv)
    qo = torch.empty(T, H, D, dtype=torch.bfloat16, device="cuda")
    ko = torch.empty_like(qo)
    a = qkr.angle_positions(dpos, dinv)
    qkr.fused_qk_norm_rope([(dq[:, 0], dq[:, 1], dgq, dgk)], qo, ko, D, W.PAIRING_NEOX, 1e-6, a)
    torch.cuda.synchronize()
    s = W.StreamInputs(qkv[:, 0].contiguous(), qkv[:, 1].contiguous(), gq, gk)
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos, inv_freq=inv)
    rq, rk = oracle.qk_norm_rope([s], H, H, D, D, W.PAIRING_NEOX, 1e-6, A)
    assert_bf16_close(qo, rq, "strided q")
    assert_bf16_close(ko, rk, "strided k")


@pytest.mark.parametrize("D,rot,pairing,kernel", [
    (64, 64, W.PAIRING_NEOX, "rope_paired"),
    (128, 128, W.PAIRING_NEOX, "rope_paired"),
    (80, 64, W.PAIRING_NEOX, "rope_paired"),
    (128, 64, W.PAIRING_NEOX, "rope_paired"),
    (256, 256, W.PAIRING_NEOX, "rope_paired"),
    (256, 96, W.PAIRING_NEOX, "rope_exchange"),
    (96, 96, W.PAIRING_NEOX, "rope_paired"),
    (32, 16, W.PAIRING_NEOX, "rope_paired"),
    (64, 20, W.PAIRING_NEOX, "rope_exchange"),
    (24, 2, W.PAIRING_NEOX, "rope_exchange"),
    (8, 8, W.PAIRING_NEOX, "rope_exchange"),
    (256, 256, W.PAIRING_GPTJ, "rope_vector"),
    (80, 64, W.PAIRING_GPTJ, "rope_vector"),
    (64, 22, W.PAIRING_GPTJ, "rope_vector"),
    (8, 6, W.PAIRING_GPTJ, "rope_vector"),
    (128, 0, W.PAIRING_NEOX, "rope_vector"),
])
def test_geometries(D, rot, pairing, kernel):
    T = 45  # ragged against every tokens-per-CTA choice
    pos = np.random.default_rng(D * 1000 + rot).integers(0, 100000, T).astype(np.int32)
    inv = W.inv_freq(1e4, max(rot // 2, 1), max(rot, 2)).numpy()
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos[None], inv_freq=inv)
    w = W.random_rope_case(D + rot, [T], 5, 3, D, rot, pairing, A)
    check_against_oracle(w, what="D=%d rot=%d" % (D, rot))
    assert qkr.last_launch()["kernel_name"] == kernel


def test_round_normalized_contract():
    w = W.config3(seed=23, T_txt=40, img_h=8, img_w=8, H=8, D=128)
    check_against_oracle(w, flags=qkr.FLAG_ROUND_NORMALIZED_BF16, what="round-normalised")


def test_zero_positions_is_pure_norm_and_deterministic():
    g = torch.Generator().manual_seed(29)
    T, H, D = 33, 4, 128
    pos = np.zeros((1, T), dtype=np.int32)
    inv = W.inv_freq(1e4, 64, 128).numpy()
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos, inv_freq=inv)
    w = W.random_rope_case(29, [T], H, H, D, D, W.PAIRING_NEOX, A)
    q1, k1 = run_fused(w)
    q2, k2 = run_fused(w)
    assert torch.equal(q1.view(torch.int16), q2.view(torch.int16))
    w0 = W.random_rope_case(29, [T], H, H, D, 0, W.PAIRING_NEOX, A)
    q0, k0 = run_fused(w0)
    assert torch.equal(q1.view(torch.int16), q0.view(torch.int16))
    assert torch.equal(k1.view(torch.int16), k0.view(torch.int16))


def test_empty_streams():
    # an empty text stream and an empty call
    w = W.config3(seed=31, T_txt=0, img_h=4, img_w=4, H=2, D=64)
    check_against_oracle(w, what="empty text stream")
    keep = []
    a = _angle_desc(w.angle, keep)
    e = torch.empty(0, 2, 64, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(64, dtype=torch.bfloat16, device="cuda")
    qkr.fused_qk_norm_rope([(e, e, g, g)], e, e, 64, 0, 1e-6, a)
    assert qkr.last_launch()["launches"] == 0


def _shape_variants(w, flags=0):
    """Run the item kernel at every heads-per-item choice and the streaming
    kernel; return the results and launch records."""
    outs = []
    try:
        for pipe, u in [(1, 1), (1, 2), (1, 3), (1, 4), (3, 2)]:
            qkr.tune_rope(pipe, u, 0, 0)
            outs.append((run_fused(w, flags), qkr.last_launch()))
    finally:
        qkr.tune_rope(0, 0, 0, 0)
    return outs


def _shape_cases():
    cases = [("joint-gptj", W.config3(seed=61, T_txt=77, img_h=9, img_w=13, H=24, D=128,
                                      pairing=W.PAIRING_GPTJ)),
             ("joint-neox", W.config3(seed=62, T_txt=64, img_h=8, img_w=8, H=24, D=128,
                                      pairing=W.PAIRING_NEOX))]
    pos = np.random.default_rng(3).integers(0, 4096, (1, 301)).astype(np.int32)
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos,
                      inv_freq=W.inv_freq(1e4, 32, 64).numpy())
    cases.append(("vit-d80", W.random_rope_case(63, [301], 16, 16, 80, 64, W.PAIRING_NEOX, A)))
    pos = np.arange(7, dtype=np.int32)[None]
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos,
                      inv_freq=W.inv_freq(1e4, 32, 64).numpy())
    cases.append(("partial-tile", W.random_rope_case(64, [7], 3, 1, 64, 64, W.PAIRING_GPTJ, A)))
    pos = np.random.default_rng(4).integers(0, 9000, (1, 53)).astype(np.int32)
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos,
                      inv_freq=W.inv_freq(1e4, 128, 256).numpy())
    cases.append(("d256", W.random_rope_case(65, [53], 4, 2, 256, 256, W.PAIRING_NEOX, A)))
    return cases


@pytest.mark.parametrize("case,w", _shape_cases(), ids=lambda v: v if isinstance(v, str) else "")
def test_heads_per_item_and_kernels_agree(case, w):
    """Every heads-per-item choice of the item kernel and the streaming kernel
    give the same bits, for both layouts, direct and staged angles and ragged
    tiles, and match the oracle."""
    outs = _shape_variants(w)
    (q0, k0), _ = outs[0]
    for (q, k), rec in outs[1:]:
        assert torch.equal(q.view(torch.int16), q0.view(torch.int16)), (case, rec)
        assert torch.equal(k.view(torch.int16), k0.view(torch.int16)), (case, rec)
    assert outs[-1][1]["pipelined"] == 2 and outs[0][1]["pipelined"] == 0
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle)
    assert_bf16_close(q0, rq, case + " q")
    assert_bf16_close(k0, rk, case + " k")


def test_strided_heads_every_kernel_and_tile():
    # non-dense head stride, both kernels, heads per item, ring depth and tile size
    g = torch.Generator().manual_seed(66)
    T, H, D = 41, 6, 128
    qkv = W.bf16_normal((T, H, 3, D), g)
    gq = W.bf16_uniform((D,), 0.5, 1.5, g)
    gk = W.bf16_uniform((D,), 0.5, 1.5, g)
    inv = W.inv_freq(1e4, 64, 128)
    pos = torch.arange(T, dtype=torch.int32).view(1, T) * 3
    dq = to_dev(qkv)
    qv = dq[:, :, 0]  # [T, H, D] with head stride 3*D
    kv = dq[:, :, 1]
    assert qv.stride(1) == 3 * D
    a = qkr.angle_positions(to_dev(pos), to_dev(inv))
    outs = []
    try:
        for pipe, u, tt, st in [(1, 0, 0, 0), (1, 2, 1, 0), (1, 4, 3, 0), (1, 1, 5, 0),
                                (3, 2, 1, 2), (3, 4, 4, 3), (3, 1, 2, 4)]:
            qkr.tune_rope(pipe, u, tt, st)
            qo = torch.empty(T, H, D, dtype=torch.bfloat16, device="cuda")
            ko = torch.empty_like(qo)
            qkr.fused_qk_norm_rope([(qv, kv, to_dev(gq), to_dev(gk))], qo, ko, D, W.PAIRING_NEOX,
                                   1e-6, a)
            torch.cuda.synchronize()
            assert qkr.last_launch()["pipelined"] == (2 if pipe == 3 else 0)
            outs.append((qo, ko))
    finally:
        qkr.tune_rope(0, 0, 0)
    for qo, ko in outs[1:]:
        assert torch.equal(qo.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(ko.view(torch.int16), outs[0][1].view(torch.int16))
    s = W.StreamInputs(qkv[:, :, 0].contiguous(), qkv[:, :, 1].contiguous(), gq, gk)
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos, inv_freq=inv)
    rq, rk = oracle.qk_norm_rope([s], H, H, D, D, W.PAIRING_NEOX, 1e-6, A)
    assert_bf16_close(outs[0][0], rq, "strided heads q")
    assert_bf16_close(outs[0][1], rk, "strided heads k")


def _table_call(w, cos, sin, mode=W.SECTIONS_NONE, sections=None):
    """Run w with the given device tables; returns (q, k, launch record)."""
    keep = []
    streams = []
    for s in w.streams:
        t = (to_dev(s.q), to_dev(s.k), to_dev(s.gamma_q), to_dev(s.gamma_k))
        keep += list(t)
        streams.append(t)
    T = w.n_tokens
    qo = Guarded((T, w.Hq, w.D))
    ko = Guarded((T, w.Hk, w.D))
    a = qkr.angle_table(cos, sin, mode, sections)
    qkr.fused_qk_norm_rope(streams, qo.tensor, ko.tensor, w.rot, w.pairing, w.eps, a)
    torch.cuda.synchronize()
    qo.check()
    ko.check()
    return qo.tensor, ko.tensor, qkr.last_launch()


@pytest.mark.parametrize("pairing", [W.PAIRING_GPTJ, W.PAIRING_NEOX])
def test_direct_table_reads_equal_staged(pairing):
    """Per-item 16-byte table reads and per-token staging give the same bits.

    A table with row pitch 64 floats is read directly; the same values at row
    pitch 66 (rows no longer 16-byte aligned) are staged in shared memory."""
    w = W.config3(seed=71, T_txt=45, img_h=7, img_w=9, H=12, D=128, pairing=pairing)
    cos = to_dev(torch.as_tensor(np.asarray(w.angle.cos), dtype=torch.float32))[0]
    sin = to_dev(torch.as_tensor(np.asarray(w.angle.sin), dtype=torch.float32))[0]
    T, P = cos.shape
    cw = torch.zeros(T, 66, dtype=torch.float32, device="cuda")
    sw = torch.zeros_like(cw)
    cw[:, :P] = cos
    sw[:, :P] = sin
    qd, kd, ld = _table_call(w, cos, sin)
    qs, ks, ls = _table_call(w, cw[:, :P], sw[:, :P])
    assert ld["direct_angles"] == 1 and ls["direct_angles"] == 0
    assert torch.equal(qd.view(torch.int16), qs.view(torch.int16))
    assert torch.equal(kd.view(torch.int16), ks.view(torch.int16))
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle)
    assert_bf16_close(qd, rq, "direct q")
    assert_bf16_close(kd, rk, "direct k")


@pytest.mark.parametrize("sections,direct", [((16, 24, 24), 1), ((18, 22, 24), 0),
                                             ((12, 20, 32), 1), ((30, 2, 32), 0)])
def test_plane_sections_direct_and_staged(sections, direct):
    """Three planes under contiguous sections: boundaries on multiples of four
    pairs are read directly, others are staged; both match the oracle."""
    rng = np.random.default_rng(sum(sections) * 7 + sections[0])
    T, H, D, rot = 83, 5, 128, 128
    P = rot // 2
    ang = rng.uniform(-40.0, 40.0, (3, T, P))
    cos = np.cos(ang).astype(np.float32)
    sin = np.sin(ang).astype(np.float32)
    A = W.AngleInputs(kind=W.ANGLE_TABLE, cos=cos, sin=sin, section_mode=W.SECTIONS_CONTIGUOUS,
                      sections=sections)
    w = W.random_rope_case(81 + sections[0], [T], H, 3, D, rot, W.PAIRING_NEOX, A)
    q, k, rec = _table_call(w, to_dev(torch.from_numpy(cos)), to_dev(torch.from_numpy(sin)),
                            W.SECTIONS_CONTIGUOUS, sections)
    assert rec["direct_angles"] == direct
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle)
    assert_bf16_close(q, rq, "planes q")
    assert_bf16_close(k, rk, "planes k")


def test_direct_table_launch_shapes_bit_identical():
    """Every (heads per item, token split) shape of the direct-angle kernel
    computes the same bits, including ranges larger than the staged kernels
    allow, 6 heads per item and the automatic split."""
    w = W.config3(seed=73, T_txt=33, img_h=6, img_w=11, H=10, D=128, pairing=W.PAIRING_GPTJ)
    cos = to_dev(torch.as_tensor(np.asarray(w.angle.cos), dtype=torch.float32))
    sin = to_dev(torch.as_tensor(np.asarray(w.angle.sin), dtype=torch.float32))
    outs = []
    try:
        for u, tt in [(0, 0), (1, 1), (2, 3), (3, 16), (4, 64), (6, 5), (6, 64)]:
            qkr.tune_rope(1, u, tt)
            q, k, rec = _table_call(w, cos, sin)
            assert rec["direct_angles"] == 1
            if tt:
                T = w.n_tokens
                assert rec["grid"] == -(-T // tt) and rec["heads_per_item"] == u
                assert rec["tokens_per_cta"] == -(-T // rec["grid"])
            outs.append((q, k))
    finally:
        qkr.tune_rope(0, 0, 0)
    for q, k in outs[1:]:
        assert torch.equal(q.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(k.view(torch.int16), outs[0][1].view(torch.int16))


def test_one_wave_grid_covers_every_token():
    """The automatic direct-angle grid has balanced token ranges; token counts
    around multiples of the grid (and fewer tokens than CTAs) still write
    every row exactly once."""
    for T_txt, img_w in ((297, 1), (297, 37), (297, 45), (5, 1)):
        w = W.config3(seed=75 + img_w, T_txt=T_txt, img_h=8, img_w=img_w, H=4, D=64,
                      pairing=W.PAIRING_GPTJ)
        q, k, _, _ = check_against_oracle(w, what="one wave T=%d" % w.n_tokens)
        rec = qkr.last_launch()
        assert rec["direct_angles"] == 1
        assert rec["grid"] <= w.n_tokens
        assert rec["tokens_per_cta"] == -(-w.n_tokens // rec["grid"])


def _with_shape(w, pipe, u=0, tt=0, stages=0, flags=0):
    try:
        qkr.tune_rope(pipe, u, tt, stages)
        out = run_fused(w, flags)
        rec = qkr.last_launch()
    finally:
        qkr.tune_rope(0, 0, 0, 0)
    return out, rec


def _stream_cases():
    cases = []
    for D, rot, pairing in [(128, 128, W.PAIRING_GPTJ), (128, 128, W.PAIRING_NEOX),
                            (80, 64, W.PAIRING_NEOX), (256, 128, W.PAIRING_NEOX),
                            (64, 22, W.PAIRING_GPTJ), (32, 16, W.PAIRING_NEOX),
                            (128, 0, W.PAIRING_NEOX)]:
        pos = np.random.default_rng(D + 7 * rot).integers(0, 50000, (1, 61)).astype(np.int32)
        A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos,
                          inv_freq=W.inv_freq(1e4, max(rot // 2, 1), max(rot, 2)).numpy())
        cases.append(("pos D=%d rot=%d p=%d" % (D, rot, pairing),
                      W.random_rope_case(D * 3 + rot, [61], 7, 3, D, rot, pairing, A)))
    cases.append(("joint gptj table", W.config3(seed=101, T_txt=37, img_h=9, img_w=11, H=12,
                                                 D=128, pairing=W.PAIRING_GPTJ)))
    return cases


@pytest.mark.parametrize("name,w", _stream_cases(), ids=lambda v: v if isinstance(v, str) else "")
def test_streaming_kernel_equals_item_kernel(name, w):
    """The cp.async streaming kernel computes the same bits as the item kernel,
    for every layout, with positions and tables, and matches the oracle."""
    (qa, ka), ra = _with_shape(w, 3)
    (qb, kb), rb = _with_shape(w, 1)
    assert ra["pipelined"] == 2 and ra["stages"] >= 2 and rb["pipelined"] == 0
    assert torch.equal(qa.view(torch.int16), qb.view(torch.int16)), name
    assert torch.equal(ka.view(torch.int16), kb.view(torch.int16)), name
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle,
                                 norm=w.norm)
    assert_bf16_close(qa, rq, name + " q")
    assert_bf16_close(ka, rk, name + " k")


def test_streaming_kernel_shapes_and_round_flag():
    """Heads per item, ring depth and token split do not change a bit; the
    bf16-rounded-normalised contract is served too."""
    w = W.config3(seed=103, T_txt=45, img_h=7, img_w=13, H=10, D=128, pairing=W.PAIRING_NEOX)
    ref, _ = _with_shape(w, 1)
    for u, tt, st in [(1, 0, 2), (2, 1, 3), (4, 7, 4), (4, 64, 2), (2, 0, 4)]:
        out, rec = _with_shape(w, 3, u, tt, st)
        assert rec["heads_per_item"] == u and rec["stages"] == st
        assert torch.equal(out[0].view(torch.int16), ref[0].view(torch.int16)), (u, tt, st)
        assert torch.equal(out[1].view(torch.int16), ref[1].view(torch.int16)), (u, tt, st)
    flags = qkr.FLAG_ROUND_NORMALIZED_BF16
    (qa, ka), _ = _with_shape(w, 3, flags=flags)
    (qb, kb), _ = _with_shape(w, 1, flags=flags)
    assert torch.equal(qa.view(torch.int16), qb.view(torch.int16))
    assert torch.equal(ka.view(torch.int16), kb.view(torch.int16))


@pytest.mark.parametrize("pairing", [W.PAIRING_GPTJ, W.PAIRING_NEOX])
@pytest.mark.parametrize("t_txt,img_h,img_w", [(77, 30, 21), (513, 64, 64)])
def test_joint_ragged_token_counts(pairing, t_txt, img_h, img_w):
    """Joint launches whose token count is not a multiple of the tokens per
    CTA the direct-angle launcher picks (2 for GPT-J at 6 heads per item, 16
    for NeoX at 24 heads), so the balanced ranges differ by one token across
    CTAs: equal to the oracle, and every token written once."""
    w = W.config3(seed=81, T_txt=t_txt, img_h=img_h, img_w=img_w, pairing=pairing)
    check_against_oracle(w, what="ragged joint")
    rec = qkr.last_launch()
    assert rec["direct_angles"] == 1
    assert rec["grid"] * rec["tokens_per_cta"] >= w.n_tokens
    assert (rec["grid"] - 1) * rec["tokens_per_cta"] < w.n_tokens


def _item_split(hq, hk, groups=16):
    """The launcher's rule for one-vector GPT-J rows with table angles, restated:
    the largest share of lane-group row slots that carry a row, then the fewest
    passes per CTA, then the most heads per item (4 or 6), at most 3 passes."""
    best = None
    for u in (4, 6):
        gpt = -(-hq // u) + -(-hk // u)
        share = (hq + hk) / (u * gpt)
        for tt in range(1, max(1, 3 * groups // gpt) + 1):
            items = tt * gpt
            passes = -(-items // groups)
            key = (round(share * items / (passes * groups), 9), -passes, u, -tt)
            if best is None or key > best[0]:
                best = (key, u, tt)
    return best[1], best[2]


@pytest.mark.parametrize("hq,hk", [(24, 24), (32, 8), (64, 8), (6, 6), (16, 8), (12, 12),
                                   (40, 8), (5, 3), (1, 1), (1, 7), (128, 8)])
def test_item_split_head_counts(hq, hk):
    """One-vector GPT-J rows with table angles, over head counts for which the
    launcher takes 4 or 6 heads per item, full or short last items and one to
    three passes per CTA (700 joint tokens, more than one wave of resident
    CTAs): equal to the oracle, every row written once, the documented split,
    and bit-identical to a forced 4 heads x 4 tokens shape."""
    cos, sin = W.joint_table(60, 20, 32, 32, 1e4)
    A = W.AngleInputs(kind=W.ANGLE_TABLE, cos=cos.unsqueeze(0), sin=sin.unsqueeze(0))
    w = W.random_rope_case(900 + 7 * hq + hk, [60, 640], hq, hk, 128, 128, W.PAIRING_GPTJ, A)
    q, k, _, _ = check_against_oracle(w, what="split %d+%d" % (hq, hk))
    rec = qkr.last_launch()
    u, tt = _item_split(hq, hk)
    assert rec["direct_angles"] == 1 and rec["heads_per_item"] == u, (rec, u, tt)
    assert rec["grid"] == -(-w.n_tokens // tt), (rec, u, tt)
    (qf, kf), rf = _with_shape(w, 1, 4, 4)
    assert rf["heads_per_item"] == 4 and rf["tokens_per_cta"] == 4
    assert torch.equal(q.view(torch.int16), qf.view(torch.int16))
    assert torch.equal(k.view(torch.int16), kf.view(torch.int16))
    for flags in (qkr.FLAG_ROUND_NORMALIZED_BF16, qkr.FLAG_EAGER_ROUNDING):
        (qa, ka), ra = _with_shape(w, 0, flags=flags)
        (qb, kb), rb = _with_shape(w, 1, 4, 4, flags=flags)
        assert ra["heads_per_item"] == u and rb["heads_per_item"] == 4
        assert torch.equal(qa.view(torch.int16), qb.view(torch.int16)), flags
        assert torch.equal(ka.view(torch.int16), kb.view(torch.int16)), flags


@pytest.mark.parametrize("pairing", [W.PAIRING_NEOX, W.PAIRING_GPTJ])
def test_large_normed_positions_launch(pairing):
    """Positions launches with the norm from 8192 tokens take the item kernel
    (staged angles); equal to the oracle and bit-identical to the streaming
    kernel forced on the same call."""
    pos = np.random.default_rng(5).integers(0, 8192, (1, 8200)).astype(np.int32)
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos,
                      inv_freq=W.inv_freq(1e4, 64, 128).numpy())
    w = W.random_rope_case(88 + pairing, [8200], 8, 8, 128, 128, pairing, A)
    (qa, ka), ra = _with_shape(w, 0)
    assert ra["pipelined"] == 0 and ra["direct_angles"] == 0, ra
    (qb, kb), rb = _with_shape(w, 3)
    assert rb["pipelined"] == 2
    assert torch.equal(qa.view(torch.int16), qb.view(torch.int16))
    assert torch.equal(ka.view(torch.int16), kb.view(torch.int16))
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle)
    assert_bf16_close(qa, rq, "large positions q")
    assert_bf16_close(ka, rk, "large positions k")


@pytest.mark.parametrize("pairing,hq,hk,T", [(W.PAIRING_GPTJ, 16, 16, 16), (W.PAIRING_GPTJ, 16, 16, 300),
                                             (W.PAIRING_GPTJ, 16, 16, 1024), (W.PAIRING_NEOX, 16, 16, 16),
                                             (W.PAIRING_NEOX, 16, 8, 512), (W.PAIRING_NEOX, 4, 4, 16)])
def test_staged_split_small_positions_launches(pairing, hq, hk, T):
    """Positions launches below the streaming kernel's range: the staged item
    kernel takes 1, 2 or 4 tokens per CTA (about one pass of work items, fewer
    tokens than one wave allows); equal to the oracle and bit-identical to a
    forced 4 tokens per CTA."""
    pos = np.random.default_rng(T + hq).integers(0, 30000, (1, T)).astype(np.int32)
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos,
                      inv_freq=W.inv_freq(1e4, 64, 128).numpy())
    w = W.random_rope_case(700 + T + hq, [T], hq, hk, 128, 128, pairing, A)
    (qa, ka), ra = _with_shape(w, 0)
    assert ra["pipelined"] == 0 and ra["direct_angles"] == 0, ra
    assert ra["tokens_per_cta"] in (1, 2, 3, 4), ra
    if hq + hk >= 24:
        assert ra["tokens_per_cta"] < 4 or T > 1000, ra
    (qb, kb), rb = _with_shape(w, 1, 2, 4)
    assert rb["tokens_per_cta"] == 4
    assert torch.equal(qa.view(torch.int16), qb.view(torch.int16))
    assert torch.equal(ka.view(torch.int16), kb.view(torch.int16))
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle)
    assert_bf16_close(qa, rq, "staged split q")
    assert_bf16_close(ka, rk, "staged split k")


@pytest.mark.parametrize("flags", [0, qkr.FLAG_ROUND_NORMALIZED_BF16, qkr.FLAG_EAGER_ROUNDING])
@pytest.mark.parametrize("T", [16, 300, 1024])
def test_pairx_rows_equal_paired(flags, T):
    """NeoX rows of head_dim 64 rotated whole with staged angles take the
    one-vector-per-lane PAIRX mapping (8 lanes per row, the partner half by
    shuffle): bit-identical to the streaming kernel's paired layout under
    every rounding contract, and equal to the oracle."""
    pos = np.random.default_rng(T).integers(0, 40000, (1, T)).astype(np.int32)
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos,
                      inv_freq=W.inv_freq(1e4, 32, 64).numpy())
    w = W.random_rope_case(500 + T, [T], 6, 2, 64, 64, W.PAIRING_NEOX, A)
    (qa, ka), ra = _with_shape(w, 1, flags=flags)
    assert ra["kernel_name"] == "rope_paired" and ra["lanes_per_row"] == 8, ra
    assert ra["slots"] == 1 and ra["pipelined"] == 0, ra
    (qb, kb), rb = _with_shape(w, 3, flags=flags)
    assert rb["pipelined"] == 2 and rb["lanes_per_row"] == 4, rb
    assert torch.equal(qa.view(torch.int16), qb.view(torch.int16))
    assert torch.equal(ka.view(torch.int16), kb.view(torch.int16))
    if flags == 0:
        rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps,
                                     w.angle)
        assert_bf16_close(qa, rq, "pairx q")
        assert_bf16_close(ka, rk, "pairx k")


@pytest.mark.parametrize("streams_T", [[1], [5, 37], [64, 700]])
def test_pairx_joint_streams_and_edges(streams_T):
    """The one-vector-per-lane NeoX mapping on joint launches (text then
    image stream, positions over the joint tokens) and a single token: equal
    to the oracle and bit-identical to the paired streaming kernel."""
    T = sum(streams_T)
    pos = np.random.default_rng(T + 3).integers(0, 9000, (1, T)).astype(np.int32)
    A = W.AngleInputs(kind=W.ANGLE_POSITIONS, positions=pos,
                      inv_freq=W.inv_freq(1e4, 32, 64).numpy())
    w = W.random_rope_case(600 + T, streams_T, 5, 3, 64, 64, W.PAIRING_NEOX, A)
    (qa, ka), ra = _with_shape(w, 1)
    assert ra["lanes_per_row"] == 8 and ra["slots"] == 1, ra
    (qb, kb), _ = _with_shape(w, 3)
    assert torch.equal(qa.view(torch.int16), qb.view(torch.int16))
    assert torch.equal(ka.view(torch.int16), kb.view(torch.int16))
    rq, rk = oracle.qk_norm_rope(w.streams, w.Hq, w.Hk, w.D, w.rot, w.pairing, w.eps, w.angle)
    assert_bf16_close(qa, rq, "pairx joint q")
    assert_bf16_close(ka, rk, "pairx joint k")
