"""Pins of the CPU oracle to things other than itself.

Each test checks the oracle against a library routine, a closed form, an
invariant the mathematics fixes, brute force on tiny inputs, or a value worked
by hand in tests/golden/.  Together they are chosen so that a dropped term,
a wrong sign or index, or a swapped operand in the oracle fails at least one.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.float().numpy().astype(np.float64)


class _S:  # minimal stream record
    def __init__(self, q, k, gq=None, gk=None):
        D = q.shape[-1]
        self.q, self.k = q, k
        self.gamma_q = gq if gq is not None else torch.ones(D, dtype=torch.bfloat16)
        self.gamma_k = gk if gk is not None else torch.ones(D, dtype=torch.bfloat16)


def _pos_angle(pos, inv, mode=W.SECTIONS_NONE, sections=(0, 0, 0, 0), token_offset=0):
    pos = np.asarray(pos, dtype=np.int32)
    if pos.ndim == 1:
        pos = pos[None]
    return W.AngleInputs(kind=W.ANGLE_POSITIONS, section_mode=mode, sections=sections,
                         positions=pos, inv_freq=np.asarray(inv, dtype=np.float32),
                         token_offset=token_offset)


# ------------------------------------------------------------------ bf16 --

def test_bf16_round_matches_torch_rne():
    # torch's fp32 -> bf16 conversion is round-to-nearest-even: a library pin.
    g = torch.Generator().manual_seed(11)
    x = torch.randn(20000, generator=g) * torch.exp2(torch.randint(-20, 20, (20000,), generator=g).float())
    # add exact ties: bf16 value + half an ulp
    base = x[:2000].to(torch.bfloat16).float()
    ulp = torch.exp2(torch.floor(torch.log2(base.abs())) - 7)
    ties = base + 0.5 * ulp
    x = torch.cat([x, ties, torch.tensor([0.0, -0.0, 1.0, -3.0, 65504.0, 1e-38, -2e-39])])
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_round(x.double().numpy())
    assert np.array_equal(ref, got)


def test_bf16_round_hand_ties():
    # 1 + 2^-8 sits halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1).
    # 1 + 3*2^-8 sits halfway between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6.
    got = oracle.bf16_round(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8]))
    assert list(got) == [0x3F80, 0x3F82]


# ---------------------------------------------------------- section maps --

def _golden_maps():
    rows = []
    with open(os.path.join(GOLDEN, "section_maps.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            mode, secs, P, axes = line.split()
            rows.append((int(mode), tuple(int(s) for s in secs.split(",")), int(P),
                         np.array([int(c) for c in axes], dtype=np.int8)))
    return rows


@pytest.mark.parametrize("row", _golden_maps(), ids=lambda r: "mode%d-%s" % (r[0], r[1]))
def test_section_map_golden(row):
    mode, secs, P, axes = row
    assert len(axes) == P
    assert np.array_equal(oracle.section_map(mode, secs, P), axes)


def _all_sections(P, with_e=False):
    for s0 in range(P + 1):
        for s1 in range(P + 1 - s0):
            for s2 in range(P + 1 - s0 - s1):
                if with_e:
                    for s3 in range(2 * P + 1 - s0 - s1 - s2):
                        if P <= s0 + s1 + s2 + s3 <= 2 * P:
                            yield (s0, s1, s2, s3)
                elif s0 + s1 + s2 == P:
                    yield (s0, s1, s2, 0)


def test_section_contiguous_brute_force():
    # Contiguous blocks: the map is non-decreasing and each axis gets exactly
    # its section's count of pairs.
    for P in range(1, 10):
        for s in _all_sections(P):
            m = oracle.section_map(W.SECTIONS_CONTIGUOUS, s, P)
            assert np.all(np.diff(m) >= 0)
            assert [int((m == a).sum()) for a in range(3)] == list(s[:3])


def test_section_interleaved_modes_agree_on_equal_sections():
    # With equal sections the three interleaved readings coincide: axis = j mod 3.
    for s in range(1, 8):
        P = 3 * s
        want = np.arange(P) % 3
        for mode in (W.SECTIONS_INTERLEAVED, W.SECTIONS_INTERLEAVED_QUOTA, W.SECTIONS_IMROPE):
            assert np.array_equal(oracle.section_map(mode, (s, s, s, 0), P), want)


def test_section_interleaved_tail_brute_force():
    # Tail-contiguous reading: head cycles t,h,w; tail equals the contiguous map.
    for P in range(1, 10):
        for s in _all_sections(P):
            m = oracle.section_map(W.SECTIONS_INTERLEAVED, s, P)
            c = oracle.section_map(W.SECTIONS_CONTIGUOUS, s, P)
            k = 3 * min(s[:3])
            assert np.array_equal(m[:k], np.arange(k) % 3)
            assert np.array_equal(m[k:], c[k:])


def test_section_quota_brute_force():
    # Quota reading: every axis receives exactly its section's count of pairs,
    # the head cycles t,h,w, and the tail is non-decreasing (t, then h, then w).
    for P in range(1, 10):
        for s in _all_sections(P):
            m = oracle.section_map(W.SECTIONS_INTERLEAVED_QUOTA, s, P)
            k = 3 * min(s[:3])
            assert [int((m == a).sum()) for a in range(3)] == list(s[:3])
            assert np.array_equal(m[:k], np.arange(k) % 3)
            assert np.all(np.diff(m[k:]) >= 0)


def test_section_imrope_by_dealing():
    # The sector rule is round-robin dealing: deal round k gives slot 3k to t
    # while k < s0, slot 3k+1 to h while k < s1, slot 3k+2 to w while k < s2;
    # a slot whose axis has run out goes to the fourth row.  Brute force for
    # every section set admitted by the P <= sum <= 2P window.
    for P in range(1, 9):
        for s in _all_sections(P, with_e=True):
            total = sum(s)
            dealt = []
            for k in range(total):  # enough rounds to cover every sector
                for r in range(3):
                    dealt.append(r if k < s[r] else 3)
            want = np.array([dealt[j % total] for j in range(P)], dtype=np.int8)
            assert np.array_equal(oracle.section_map(W.SECTIONS_IMROPE, s, P), want), s


# ---------------------------------------------------------------- RMSNorm --

def test_rmsnorm_hand_worked():
    with open(os.path.join(GOLDEN, "rmsnorm_worked.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            D, xs, gs, ys = [p.split() for p in line.split("|")]
            D = int(D[0])
            x = _bf16([float(v) for v in xs]).reshape(1, 1, D)
            g = _bf16([float(v) for v in gs])
            s = _S(x, x, g, g)
            q, _ = oracle.qk_norm_rope([s], 1, 1, D, 0, W.PAIRING_NEOX, 0.0,
                                       _pos_angle([0], [1.0]))
            np.testing.assert_allclose(q.reshape(-1), [float(v) for v in ys], rtol=1e-14)


@pytest.mark.parametrize("c", [0.25, -0.25, 1.0, -1.0, 7.0, -7.0])
def test_rmsnorm_constant_row(c):
    # RMS of a constant row is |c|: the output is gamma * sign(c) up to eps.
    D = 64
    g = W.bf16_uniform((D,), 0.5, 1.5, torch.Generator().manual_seed(1))
    x = _bf16(np.full((1, 1, D), c))
    q, _ = oracle.qk_norm_rope([_S(x, x, g, g)], 1, 1, D, 0, 0, 1e-6, _pos_angle([0], [0.0]))
    np.testing.assert_allclose(q.reshape(-1), np.sign(c) * _f64(g), rtol=2e-5)


def test_rmsnorm_scale_invariant_and_gamma_linear():
    g0 = torch.Generator().manual_seed(2)
    D = 96
    x = W.bf16_normal((3, 2, D), g0)
    gam = W.bf16_uniform((D,), 0.5, 1.5, g0)
    ones = torch.ones(D, dtype=torch.bfloat16)
    a = oracle.qk_norm_rope([_S(x, x, gam, gam)], 2, 2, D, 0, 0, 0.0, _pos_angle([0, 0, 0], [1.0]))[0]
    # scaling by a power of two is exact in bf16 and must not change the output
    x4 = (x.float() * 4).to(torch.bfloat16)
    b = oracle.qk_norm_rope([_S(x4, x4, gam, gam)], 2, 2, D, 0, 0, 0.0, _pos_angle([0, 0, 0], [1.0]))[0]
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)
    # gamma multiplies elementwise
    u = oracle.qk_norm_rope([_S(x, x, ones, ones)], 2, 2, D, 0, 0, 0.0, _pos_angle([0, 0, 0], [1.0]))[0]
    np.testing.assert_allclose(a, u * _f64(gam), rtol=1e-13)
    # unit RMS after normalisation with unit gamma
    np.testing.assert_allclose(np.sqrt((u ** 2).mean(-1)), 1.0, rtol=1e-12)


def test_rmsnorm_eps_and_zero_row():
    D = 8
    z = torch.zeros(1, 1, D, dtype=torch.bfloat16)
    q, _ = oracle.qk_norm_rope([_S(z, z)], 1, 1, D, 0, 0, 1e-6, _pos_angle([0], [0.0]))
    assert np.all(q == 0)
    # a constant row at the scale of sqrt(eps): |y| = c / sqrt(c^2 + eps)
    c = 2.0 ** -10
    x = _bf16(np.full((1, 1, D), c))
    q, _ = oracle.qk_norm_rope([_S(x, x)], 1, 1, D, 0, 0, 1e-6, _pos_angle([0], [0.0]))
    np.testing.assert_allclose(q.reshape(-1), c / np.sqrt(c * c + 1e-6), rtol=1e-12)


# ------------------------------------------------------------- rotation --

def _complex_rope(x: np.ndarray, pos: np.ndarray, inv: np.ndarray, pairing: int, rot: int):
    """RoPE as complex multiplication: pair (a, b) is a + i b, times exp(i theta)."""
    P = rot // 2
    if pairing == W.PAIRING_NEOX:
        ia, ib = np.arange(P), np.arange(P) + P
    else:
        ia, ib = 2 * np.arange(P), 2 * np.arange(P) + 1
    theta = (pos.astype(np.float32)[:, None] * inv[None, :P].astype(np.float32)).astype(np.float64)
    z = (x[..., ia] + 1j * x[..., ib]) * np.exp(1j * theta)[:, None, :]
    y = x.copy()
    y[..., ia] = z.real
    y[..., ib] = z.imag
    return y


@pytest.mark.parametrize("pairing", [W.PAIRING_NEOX, W.PAIRING_GPTJ])
@pytest.mark.parametrize("D,rot", [(64, 64), (80, 64), (32, 20), (16, 2)])
def test_rotation_is_complex_multiplication(pairing, D, rot):
    g = torch.Generator().manual_seed(3)
    T, H = 7, 3
    x = W.bf16_normal((T, H, D), g)
    pos = np.array([0, 1, 2, 5, 100, 8191, -7], dtype=np.int32)
    inv = W.inv_freq(10000.0, rot // 2 if rot else 1, max(rot, 2)).numpy()
    q, k = oracle.qk_norm_rope([_S(x, x)], H, H, D, rot, pairing, 0.0, _pos_angle(pos, inv),
                               norm=False)
    want = _complex_rope(_f64(x), pos, inv, pairing, rot)
    np.testing.assert_allclose(q, want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(k, want, rtol=1e-12, atol=1e-12)


def test_rotation_quarter_turn():
    # theta = fp32(pi/2) at position 1: (a, b) -> (-b, a) up to cos(fp32(pi/2)) ~ -4.4e-8.
    D = 4
    x = _bf16([[[1.5, -2.0, 0.75, 3.0]]])
    inv = np.array([np.float32(np.pi / 2), np.float32(np.pi / 2)], dtype=np.float32)
    q, _ = oracle.qk_norm_rope([_S(x, x)], 1, 1, D, 4, W.PAIRING_NEOX, 0.0, _pos_angle([1], inv),
                               norm=False)
    # NeoX pairs: (x0, x2) and (x1, x3)
    np.testing.assert_allclose(q.reshape(-1), [-0.75, -3.0, 1.5, -2.0], atol=1e-6)
    q, _ = oracle.qk_norm_rope([_S(x, x)], 1, 1, D, 4, W.PAIRING_GPTJ, 0.0, _pos_angle([1], inv),
                               norm=False)
    # GPT-J pairs: (x0, x1) and (x2, x3)
    np.testing.assert_allclose(q.reshape(-1), [2.0, 1.5, -3.0, 0.75], atol=1e-6)


def test_rotation_zero_position_is_identity_and_norm_preserving():
    g = torch.Generator().manual_seed(4)
    T, H, D = 5, 2, 64
    x = W.bf16_normal((T, H, D), g)
    gam = W.bf16_uniform((D,), 0.5, 1.5, g)
    inv = W.inv_freq(10000.0, 32, 64).numpy()
    zero = oracle.qk_norm_rope([_S(x, x, gam, gam)], H, H, D, 64, 0, 1e-6, _pos_angle(np.zeros(T), inv))[0]
    unrot = oracle.qk_norm_rope([_S(x, x, gam, gam)], H, H, D, 0, 0, 1e-6, _pos_angle(np.zeros(T), inv))[0]
    assert np.array_equal(zero, unrot)
    pos = np.array([3, 77, 1000, 4095, 8191])
    rot = oracle.qk_norm_rope([_S(x, x, gam, gam)], H, H, D, 64, 0, 1e-6, _pos_angle(pos, inv))[0]
    np.testing.assert_allclose(rot[..., :32] ** 2 + rot[..., 32:] ** 2,
                               unrot[..., :32] ** 2 + unrot[..., 32:] ** 2, rtol=1e-12)


def test_rotation_relative_position():
    # <R(p) q, R(p') k> depends only on p - p'.
    g = torch.Generator().manual_seed(5)
    D = 64
    q = W.bf16_normal((1, 1, D), g)
    k = W.bf16_normal((1, 1, D), g)
    inv = W.inv_freq(10000.0, 32, 64).numpy()
    for pairing in (0, 1):
        dots = []
        for p, pp in [(10, 3), (107, 100), (1007, 1000), (7, 0)]:
            a = oracle.qk_norm_rope([_S(q, q)], 1, 1, D, D, pairing, 0.0, _pos_angle([p], inv), norm=False)[0]
            b = oracle.qk_norm_rope([_S(k, k)], 1, 1, D, D, pairing, 0.0, _pos_angle([pp], inv), norm=False)[0]
            dots.append(float((a * b).sum()))
        # fp32 angles: theta(p) - theta(p') carries fp32 rounding of each product
        np.testing.assert_allclose(dots, dots[-1], rtol=2e-4, atol=2e-4)


def test_gptj_equals_neox_on_deinterleaved_input():
    g = torch.Generator().manual_seed(6)
    T, H, D = 4, 2, 32
    x = W.bf16_normal((T, H, D), g)
    gam = W.bf16_uniform((D,), 0.5, 1.5, g)
    P = D // 2
    perm = np.empty(D, dtype=np.int64)  # neox layout index -> gptj layout index
    perm[:P] = 2 * np.arange(P)
    perm[P:] = 2 * np.arange(P) + 1
    inv = W.inv_freq(10000.0, P, D).numpy()
    pos = np.array([1, 9, 200, 4000])
    gj = oracle.qk_norm_rope([_S(x, x, gam, gam)], H, H, D, D, W.PAIRING_GPTJ, 1e-6, _pos_angle(pos, inv))[0]
    xn = x[..., perm].contiguous()
    nx = oracle.qk_norm_rope([_S(xn, xn, gam[perm].contiguous(), gam[perm].contiguous())], H, H, D, D,
                             W.PAIRING_NEOX, 1e-6, _pos_angle(pos, inv))[0]
    np.testing.assert_array_equal(gj[..., perm], nx)


def test_table_source_equals_positions_source():
    # A cos/sin table built by a library routine (numpy) from the same fp32
    # angles must give the same rotation as in-place angles.
    g = torch.Generator().manual_seed(7)
    T, H, D = 6, 2, 32
    x = W.bf16_normal((T, H, D), g)
    inv = W.inv_freq(10000.0, 16, 32).numpy()
    pos = np.array([0, 1, 2, 3, 50, 60], dtype=np.int32)
    ang = (pos.astype(np.float32)[:, None] * inv[None]).astype(np.float64)
    A = W.AngleInputs(kind=W.ANGLE_TABLE, cos=np.cos(ang).astype(np.float32)[None],
                      sin=np.sin(ang).astype(np.float32)[None])
    a = oracle.qk_norm_rope([_S(x, x)], H, H, D, D, 0, 1e-6, A)[0]
    b = oracle.qk_norm_rope([_S(x, x)], H, H, D, D, 0, 1e-6, _pos_angle(pos, inv))[0]
    np.testing.assert_allclose(a, b, rtol=0, atol=2e-7 * 8)


# --------------------------------------------------- mRoPE and chunking --

def test_mrope_equal_rows_collapse_to_plain_rope():
    g = torch.Generator().manual_seed(8)
    T, Hq, Hk, D = 9, 4, 2, 128
    q, k = W.bf16_normal((T, Hq, D), g), W.bf16_normal((T, Hk, D), g)
    inv = W.inv_freq(5e6, 64, 128).numpy()
    p = np.random.default_rng(0).integers(0, 8192, T).astype(np.int32)
    plain = oracle.qk_norm_rope([_S(q, k)], Hq, Hk, D, D, 0, 0.0, _pos_angle(p, inv), norm=False)
    for mode, rows in [(1, 3), (2, 3), (3, 3), (4, 4)]:
        same = np.stack([p] * rows)
        got = oracle.qk_norm_rope([_S(q, k)], Hq, Hk, D, D, 0, 0.0,
                                  _pos_angle(same, inv, mode, (24, 20, 20, 0)), norm=False)
        assert np.array_equal(got[0], plain[0]) and np.array_equal(got[1], plain[1])
        distinct = np.stack([p] + [np.roll(p, i + 1) + 7 for i in range(rows - 1)])
        diff = oracle.qk_norm_rope([_S(q, k)], Hq, Hk, D, D, 0, 0.0,
                                   _pos_angle(distinct, inv, mode, (24, 20, 20, 0)), norm=False)
        assert not np.allclose(diff[0], plain[0], atol=1e-3)


def test_mrope_pair_reads_its_axis_row():
    # Pair j must take its angle from row axis(j): zero every row but one and
    # check that exactly the pairs mapped to that row rotate.
    T, D = 1, 128
    x = _bf16(np.ones((T, 1, D)))
    inv = np.full(64, 0.5, dtype=np.float32)
    for mode in (1, 2, 3, 4):
        rows = 4 if mode == 4 else 3
        amap = oracle.section_map(mode, (24, 20, 20, 0), 64)
        for r in range(rows):
            pos = np.zeros((rows, T), dtype=np.int32)
            pos[r] = 3
            y = oracle.qk_norm_rope([_S(x, x)], 1, 1, D, D, 0, 0.0,
                                    _pos_angle(pos, inv, mode, (24, 20, 20, 0)), norm=False)[0]
            moved = ~np.isclose(y[0, 0, :64], 1.0)
            assert np.array_equal(moved, amap == r), (mode, r)


def test_chunked_equals_unchunked():
    g = torch.Generator().manual_seed(9)
    T, Hq, Hk, D = 300, 2, 1, 64
    q, k = W.bf16_normal((T, Hq, D), g), W.bf16_normal((T, Hk, D), g)
    inv = W.inv_freq(5e6, 32, 64).numpy()
    pos = np.random.default_rng(1).integers(0, 8192, (3, T)).astype(np.int32)
    full = oracle.qk_norm_rope([_S(q, k)], Hq, Hk, D, D, 0, 0.0,
                               _pos_angle(pos, inv, 2, (12, 10, 10, 0)), norm=False)
    parts = []
    for t0, t1 in [(0, 2), (2, 245), (245, 300)]:
        parts.append(oracle.qk_norm_rope([_S(q[t0:t1], k[t0:t1])], Hq, Hk, D, D, 0, 0.0,
                                         _pos_angle(pos, inv, 2, (12, 10, 10, 0), token_offset=t0),
                                         norm=False))
    assert np.array_equal(np.concatenate([p[0] for p in parts]), full[0])
    assert np.array_equal(np.concatenate([p[1] for p in parts]), full[1])


def test_joint_equals_per_stream_concat():
    w = W.config3(T_txt=5, img_h=3, img_w=4, H=2, D=32)
    joint = oracle.qk_norm_rope(w.streams, 2, 2, 32, 32, w.pairing, w.eps, w.angle)
    a = oracle.qk_norm_rope(w.streams[:1], 2, 2, 32, 32, w.pairing, w.eps, w.angle)
    off = W.AngleInputs(kind=W.ANGLE_TABLE, cos=w.angle.cos, sin=w.angle.sin, token_offset=5)
    b = oracle.qk_norm_rope(w.streams[1:], 2, 2, 32, 32, w.pairing, w.eps, off)
    assert np.array_equal(joint[0], np.concatenate([a[0], b[0]]))
    assert np.array_equal(joint[1], np.concatenate([a[1], b[1]]))
    # text first: the first five joint tokens are the text stream's
    assert np.array_equal(joint[0][:5], a[0])


def test_round_normalized_contract():
    # With the bf16-rounded normalised value and an identity rotation the
    # output is exactly the bf16 rounding (torch RNE, a library pin) of the
    # unrounded normalised value, which is within half a bf16 ulp of it.
    g = torch.Generator().manual_seed(10)
    T, H, D = 3, 2, 64
    x = W.bf16_normal((T, H, D), g)
    gam = W.bf16_uniform((D,), 0.5, 1.5, g)
    inv = W.inv_freq(1e4, 32, 64).numpy()
    A = _pos_angle(np.zeros(T), inv)
    exact = oracle.qk_norm_rope([_S(x, x, gam, gam)], H, H, D, D, 0, 1e-6, A)[0]
    rnd = oracle.qk_norm_rope([_S(x, x, gam, gam)], H, H, D, D, 0, 1e-6, A, round_normalized=True)[0]
    lib = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16).double().numpy()
    # fp64 -> fp32 -> bf16 can differ from direct rounding only at exact ties,
    # which random normal inputs do not produce.
    assert np.array_equal(rnd, lib)


def _eager_case():
    x = _bf16([1, 1, 7, 1, 1, 1, 1, 1]).reshape(1, 1, 8)
    g = _bf16([1.5, 0.75, 1, 1, 1, 1, 1, 1])
    return _S(x, x, g, g)


@pytest.mark.parametrize("contract", ["eager", "round_normalized", "none"])
def test_rounding_contracts_hand_worked(contract):
    """The three rounding contracts on the hand-worked row of
    tests/golden/eager_rounding.txt, at position 0 (identity rotation)."""
    rows = {}
    with open(os.path.join(GOLDEN, "eager_rounding.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, ys = [p.strip() for p in line.split("|")]
            rows[name] = [float(v) for v in ys.split()]
    q, _ = oracle.qk_norm_rope([_eager_case()], 1, 1, 8, 8, W.PAIRING_GPTJ, 0.0,
                               _pos_angle([0], np.zeros(4)),
                               round_normalized=contract == "round_normalized",
                               eager_rounding=contract == "eager")
    np.testing.assert_allclose(q.reshape(-1), rows[contract], rtol=1e-15, atol=0)
    if contract != "none":
        assert rows["eager"][:2] != rows["round_normalized"][:2]  # the example separates them


def test_eager_rounding_happens_before_the_rotation():
    """With a table angle (cos, sin) = (fp32 0.6, fp32 0.8) on every pair, the
    eager output is the textbook rotation of the hand-worked rounded values
    (rounding first, then the exact rotation, no rounding after it)."""
    c, s = float(np.float32(0.6)), float(np.float32(0.8))
    cos = np.full((1, 4), c, dtype=np.float32)
    sin = np.full((1, 4), s, dtype=np.float32)
    A = W.AngleInputs(kind=W.ANGLE_TABLE, cos=cos, sin=sin)
    q, _ = oracle.qk_norm_rope([_eager_case()], 1, 1, 8, 8, W.PAIRING_GPTJ, 0.0, A,
                               eager_rounding=True)
    y = [0.5703125, 0.28515625, 2.640625] + [0.37890625] * 5
    want = []
    for j in range(4):
        a, b = y[2 * j], y[2 * j + 1]
        want += [a * c - b * s, b * c + a * s]
    np.testing.assert_allclose(q.reshape(-1), want, rtol=1e-15, atol=1e-15)


def test_eager_rounding_is_two_roundings_of_torch():
    """On random rows the eager contract equals torch's bf16 rounding (RNE, a
    library pin) applied to x r and then to the rounded value times gamma,
    with r from the unrounded contract's own output (y = x r gamma)."""
    g = torch.Generator().manual_seed(12)
    T, H, D = 4, 3, 64
    x = W.bf16_normal((T, H, D), g)
    gam = W.bf16_uniform((D,), 0.5, 1.5, g)
    A = _pos_angle(np.zeros(T), W.inv_freq(1e4, 32, 64).numpy())
    exact = oracle.qk_norm_rope([_S(x, x, gam, gam)], H, H, D, D, 0, 1e-6, A)[0]
    eager = oracle.qk_norm_rope([_S(x, x, gam, gam)], H, H, D, D, 0, 1e-6, A,
                                eager_rounding=True)[0]
    xr = exact / _f64(gam)                       # x r per element
    n = torch.from_numpy(xr).to(torch.bfloat16).double()
    want = (n * torch.from_numpy(_f64(gam))).to(torch.bfloat16).double().numpy()
    assert np.array_equal(eager, want)
    assert not np.array_equal(eager, exact)


def test_tie_masks():
    """The near-tie masks: empty without intermediate rounding, shared by both
    members of every rotation pair, and about 2e-3 of the elements (values
    within 1e-3 quanta of a midpoint) on random rows."""
    g = torch.Generator().manual_seed(13)
    T, H, D = 64, 8, 128
    x = W.bf16_normal((T, H, D), g)
    gam = W.bf16_uniform((D,), 0.5, 1.5, g)
    A = _pos_angle(np.arange(T), W.inv_freq(1e4, 64, 128).numpy())
    _, _, tq0, _ = oracle.qk_norm_rope([_S(x, x, gam, gam)], H, H, D, D, 0, 1e-6, A,
                                       return_ties=True)
    assert not tq0.any()
    for kw in ({"eager_rounding": True}, {"round_normalized": True}):
        _, _, tq, tk = oracle.qk_norm_rope([_S(x, x, gam, gam)], H, H, D, D, 0, 1e-6, A,
                                           return_ties=True, **kw)
        assert np.array_equal(tq[..., :64], tq[..., 64:])     # NeoX pairs (j, j + 64)
        frac = tq.mean()
        assert 5e-4 < frac < 1.2e-2, frac


# ------------------------------------------------------------ ViT setup --

def _unravel_positions(grids, m):
    # np.unravel_index over the radices (t, h/m, w/m, m, m) of the
    # merge-block token order: a library routine, not the oracle's loops.
    out = []
    for t, h, w in grids:
        idx = np.arange(t * h * w)
        tt, bh, bw, mh, mw = np.unravel_index(idx, (t, h // m, w // m, m, m))
        out.append(np.stack([tt, bh * m + mh, bw * m + mw]))
    return np.concatenate(out, axis=1).astype(np.int32)


@pytest.mark.parametrize("m", [1, 2, 4])
def test_vit_positions_unravel_and_bijection(m):
    grids = [[1, 4, 8], [2, 8, 4], [3, 4, 4], [1, 12, 16]]
    pos = oracle.vit_positions(grids, m)
    assert np.array_equal(pos, _unravel_positions(grids, m))
    start = 0
    for t, h, w in grids:
        seg = pos[:, start:start + t * h * w]
        assert tuple(seg[:, 0]) == (0, 0, 0)
        assert tuple(seg[:, -1]) == (t - 1, h - 1, w - 1)
        trip = set(map(tuple, seg.T.tolist()))
        assert trip == {(a, b, c) for a in range(t) for b in range(h) for c in range(w)}
        start += t * h * w
    if m == 1:  # no merging: plain raster order
        r = np.concatenate([np.indices((t, h, w)).reshape(3, -1) for t, h, w in grids], axis=1)
        assert np.array_equal(pos, r)


def test_vit_positions_merge2_small_hand_case():
    # One frame, h = w = 4, m = 2: the first merge block covers rows 0-1 and
    # columns 0-1 in row-major order, then the block to its right.
    pos = oracle.vit_positions([[1, 4, 4]], 2)
    assert pos[1, :8].tolist() == [0, 0, 1, 1, 0, 0, 1, 1]
    assert pos[2, :8].tolist() == [0, 1, 0, 1, 2, 3, 2, 3]


def test_vit_positions_rejects_unmergeable_grid():
    with pytest.raises(ValueError):
        oracle.vit_positions([[1, 3, 4]], 2)


def test_vit_planes_layout_and_values():
    pos = np.array([[0, 1, 2], [0, 1, 5], [0, 3, 1]], dtype=np.int32)
    inv_t = np.array([1.0, 0.5], dtype=np.float32)
    inv_h = np.array([1.0, 0.25, 0.125], dtype=np.float32)
    inv_w = np.array([1.0], dtype=np.float32)
    cos, sin, wr = oracle.vit_planes(pos, inv_t, inv_h, inv_w)
    P = 6
    assert cos.shape == (3, 3, P)
    # written cells: plane t cols [0,2), plane h cols [2,5), plane w col [5,6)
    want = np.zeros((3, 3, P), dtype=bool)
    want[0, :, 0:2] = True
    want[1, :, 2:5] = True
    want[2, :, 5:6] = True
    assert np.array_equal(wr.astype(bool), want)
    assert np.all(np.isnan(cos[~want]))
    # position 0 -> (1, 0) exactly
    assert np.all(cos[:, 0][want[:, 0]] == 1.0) and np.all(sin[:, 0][want[:, 0]] == 0.0)
    # textbook constants: cos(1), sin(1), cos(2), sin(0.75)
    assert cos[0, 1, 0] == np.float32(0.5403023058681398)
    assert sin[0, 1, 0] == np.float32(0.8414709848078965)
    assert cos[0, 2, 0] == np.float32(-0.4161468365471424)
    assert sin[1, 1, 3] == np.float32(np.sin(0.25))  # h pos 1 * 0.25
    assert sin[2, 1, 5] == np.float32(0.1411200080598672)  # w pos 3 * 1 -> sin(3)
    np.testing.assert_allclose(cos[want] ** 2 + sin[want] ** 2, 1.0, rtol=1e-6)


# ---------------------------------------------------- RMSNorm + residual --

def test_rms_norm_residual_pins():
    w = W.config2(R=4, hidden=256)
    res_bits, out = oracle.rms_norm_residual(w.x, w.residual, w.gamma, w.eps)
    # the new residual is bf16(x + residual): torch's fp32 add + RNE is a library pin
    lib = (w.x.float() + w.residual.float()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(res_bits, lib)
    s = oracle.bf16_bits_to_f64(res_bits)
    u = out / _f64(w.gamma)[None]
    np.testing.assert_allclose(np.sqrt((u ** 2).mean(-1)),
                               np.sqrt((s ** 2).mean(-1) / ((s ** 2).mean(-1) + w.eps)), rtol=1e-12)
    # out / gamma is proportional to the summed residual row
    ratio = u / np.where(s == 0, np.nan, s)
    assert np.nanmax(np.abs(ratio - np.nanmean(ratio, axis=1, keepdims=True))) < 1e-12


def test_rms_norm_residual_constant_row():
    D = 64
    x = torch.full((1, D), 0.75, dtype=torch.bfloat16)
    r = torch.full((1, D), 0.25, dtype=torch.bfloat16)
    g = W.bf16_uniform((D,), 0.5, 1.5, torch.Generator().manual_seed(3))
    res_bits, out = oracle.rms_norm_residual(x, r, g, 1e-6)
    assert np.all(res_bits == 0x3F80)  # 1.0
    np.testing.assert_allclose(out.reshape(-1), _f64(g), rtol=1e-6)


# ------------------------------------------------------------- workloads --

def test_workload_shapes_match_configs():
    w1 = W.config1()
    assert tuple(w1.streams[0].q.shape) == (16, 4, 64) and w1.angle.positions.tolist() == [list(range(16))]
    w3 = W.config3()
    assert [tuple(s.q.shape) for s in w3.streams] == [(512, 24, 128), (4096, 24, 128)]
    assert tuple(w3.angle.cos.shape) == (1, 4608, 64)
    w4 = W.config4()
    assert tuple(w4.streams[0].q.shape) == (8192, 16, 128) and tuple(w4.streams[0].k.shape) == (8192, 8, 128)
    assert tuple(w4.angle.positions.shape) == (3, 8192)
    assert int(w4.angle.positions.min()) >= 0 and int(w4.angle.positions.max()) < 8192
    w5 = W.config5()
    assert len(w5.grids) == 8
    for t, h, w in w5.grids:
        assert t in (1, 2) and h % 2 == 0 and w % 2 == 0 and 16 <= h <= 64 and 16 <= w <= 64
    assert [len(w5.inv_t), len(w5.inv_h), len(w5.inv_w)] == [16, 24, 24]
    g = W.config2(R=32, hidden=5120).gamma.float()
    assert float(g.min()) >= 0.5 and float(g.max()) <= 1.5


def test_joint_v_is_text_first_row_copy():
    """V of the joint Q/K/V op: row n of the joint output is row n of the text
    stream for n < T0, else row n - T0 of the image stream, bit for bit
    (checked row by row, including an empty text stream)."""
    g = torch.Generator().manual_seed(5)
    for T0, T1 in ((3, 5), (0, 4), (6, 0)):
        a = W.bf16_normal((T0, 2, 8), g)
        b = W.bf16_normal((T1, 2, 8), g)
        j = oracle.joint_v([a, b])
        assert j.shape == (T0 + T1, 2, 8) and j.dtype == np.uint16
        for n in range(T0 + T1):
            src = a[n] if n < T0 else b[n - T0]
            assert np.array_equal(j[n], src.view(torch.int16).numpy().view(np.uint16))


def test_scatter_rows_places_each_row_once():
    """rope_set_rows's destination: brute-force row placement on a tiny case,
    including unnamed rows (fill) and a reversed index order."""
    rows = np.arange(4 * 2 * 3, dtype=np.float64).reshape(4, 2, 3)
    idx = [6, 0, 3, 1]
    out = oracle.scatter_rows(rows, idx, 8, fill=-1.0)
    for t, r in enumerate(idx):
        assert np.array_equal(out[r], rows[t])
    for r in set(range(8)) - set(idx):
        assert (out[r] == -1.0).all()
    rev = oracle.scatter_rows(rows, [3, 2, 1, 0], 4)
    assert np.array_equal(rev, rows[::-1])


def _e4m3_decode(code: int) -> float:
    """The E4M3 ("FN") format written out: sign, 4-bit exponent (bias 7),
    3-bit mantissa, exponent 0 = subnormal m * 2^-9."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 7
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1 + m / 8) * 2.0 ** (e - 7)


def test_fp8_e4m3_hand_values():
    cases = [(1.0, 0x38), (3.5, 0x46), (-3.5, 0xC6), (448.0, 0x7E), (-448.0, 0xFE),
             (2.0 ** -9, 0x01), (7 * 2.0 ** -9, 0x07), (2.0 ** -6, 0x08),
             (2.0 ** -10, 0x00),              # tie between 0 and the smallest subnormal: even
             (3 * 2.0 ** -10, 0x02),          # tie between 1 and 2 subnormal steps: even
             (1.0625, 0x38), (1.1875, 0x3A),  # ties between mantissas 0/1 and 1/2
             (464.0, 0x7E), (470.0, 0x7E), (500.0, 0x7E), (-1e9, 0xFE),  # saturation
             (0.0, 0x00), (-0.0, 0x80)]
    for v, code in cases:
        assert int(oracle.fp8_e4m3([v])[0]) == code, (v, hex(code))


def test_fp8_e4m3_round_trip_and_torch():
    """Every finite code decodes (format definition above; torch's own
    float8_e4m3fn agrees) and re-encodes to itself; random values in range
    encode as torch's round-to-nearest-even cast does."""
    codes = [c for c in range(256) if (c & 0x7F) != 0x7F]
    vals = np.array([_e4m3_decode(c) for c in codes])
    t = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(vals, t)
    enc = oracle.fp8_e4m3(vals)
    assert np.array_equal(enc[vals != 0], np.array(codes, dtype=np.uint8)[vals != 0])
    rng = np.random.default_rng(3)
    r = np.concatenate([rng.uniform(-448, 448, 4000), rng.normal(0, 0.05, 4000),
                        rng.normal(0, 2 ** -8, 2000)])
    want = torch.from_numpy(r).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.fp8_e4m3(r), want)


def test_rms_norm_fp8_matches_rms_norm_and_encoder():
    """The FP8 RMSNorm is the bf16-path RMSNorm divided by the scale and
    encoded: same residual bits, y/scale equals out/scale, codes equal the
    encoder's; without a residual s = x."""
    w = W.config2(R=3, hidden=64, seed=41)
    res_o, y_o = oracle.rms_norm_residual(w.x, w.residual, w.gamma, w.eps)
    res_f, ys, codes = oracle.rms_norm_fp8(w.x, w.residual, w.gamma, w.eps, 0.05)
    assert np.array_equal(res_o, res_f)
    assert np.allclose(ys, y_o / 0.05, rtol=1e-15, atol=0)
    assert np.array_equal(codes, oracle.fp8_e4m3(ys))
    zero = torch.zeros_like(w.residual)
    _, y_z = oracle.rms_norm_residual(w.x, zero, w.gamma, w.eps)
    none, ys_n, _ = oracle.rms_norm_fp8(w.x, None, w.gamma, w.eps, 2.0)
    assert none is None
    assert np.allclose(ys_n, y_z / 2.0, rtol=1e-15, atol=0)
