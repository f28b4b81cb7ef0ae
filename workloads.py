"""Seeded synthetic inputs for the normalise-then-rotate path.

This module is the only code shared by the CPU oracle (``oracle/``) and the
CUDA path (``mrope_qk_norm_b200``).  It draws random numbers and lays out the
five workloads (sizes, distributions, position layouts); it performs none of
the method's arithmetic (no normalisation, no rotation, no section rule, no
grid-to-position mapping).

Two inputs are deterministic rather than random and are built here because
the pages treat them as caller-supplied inputs, not as steps of the op:

* ``inv_freq`` -- the per-pair inverse frequencies ``theta**(-2j/dim)``.
  The ViT setup page (vLLM ``mrope_vit_setup``, ``VitMropeSetup.forward``
  docstring) takes them as per-axis caller buffers of length ``dim // 2``.
* the joint text/image ``[cos | sin]`` table of the Ovis-Image workload.  The
  vllm-omni page ("Fuse text/image QK RMSNorm + cat + RoPE into one Triton
  launch", Purpose) says the model's position embedder produces it once per
  forward and the fused op only reads it.

All generation uses the torch CPU generator, so values do not depend on the
GPU.  Random tensors are returned as CPU torch tensors (bf16 / int32 / fp32).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

# Numeric codes shared with include/qkr.h and the oracle (plain integers).
PAIRING_NEOX = 0
PAIRING_GPTJ = 1

SECTIONS_NONE = 0          # plain 1-D RoPE: every pair reads row 0
SECTIONS_CONTIGUOUS = 1    # t block, then h block, then w block
SECTIONS_INTERLEAVED = 2   # pair i -> axis i mod 3 while i < 3*min, else contiguous
SECTIONS_INTERLEAVED_QUOTA = 3  # same head; tail pairs go to axes with quota left
SECTIONS_IMROPE = 4        # sector rule with a fourth ("e") position row

ANGLE_POSITIONS = 0
ANGLE_TABLE = 1


def _gen(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(int(seed))


def bf16_normal(shape, g: torch.Generator) -> torch.Tensor:
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def bf16_uniform(shape, lo: float, hi: float, g: torch.Generator) -> torch.Tensor:
    u = torch.rand(shape, generator=g, dtype=torch.float32)
    return (lo + (hi - lo) * u).to(torch.bfloat16)


def inv_freq(theta: float, n_pairs: int, dim: int) -> torch.Tensor:
    """fp32 ``theta ** (-2 j / dim)`` for ``j < n_pairs``, evaluated in fp64."""
    j = np.arange(n_pairs, dtype=np.float64)
    return torch.from_numpy((theta ** (-2.0 * j / dim)).astype(np.float32))


# --------------------------------------------------------------------------
# Workload containers
# --------------------------------------------------------------------------

@dataclass
class StreamInputs:
    q: torch.Tensor        # [T, Hq, D] bf16
    k: torch.Tensor        # [T, Hk, D] bf16
    gamma_q: torch.Tensor  # [D] bf16
    gamma_k: torch.Tensor  # [D] bf16


@dataclass
class AngleInputs:
    kind: int
    section_mode: int = SECTIONS_NONE
    sections: tuple = (0, 0, 0, 0)
    positions: torch.Tensor | None = None   # [rows, T_total] int32
    inv_freq: torch.Tensor | None = None    # [P] fp32
    cos: torch.Tensor | None = None         # [planes, N, ld] fp32
    sin: torch.Tensor | None = None
    token_offset: int = 0


@dataclass
class RopeWorkload:
    name: str
    streams: list
    Hq: int
    Hk: int
    D: int
    rot: int
    pairing: int
    eps: float
    angle: AngleInputs
    norm: bool = True
    extra: dict = field(default_factory=dict)

    @property
    def n_tokens(self) -> int:
        return sum(int(s.q.shape[0]) for s in self.streams)


@dataclass
class RmsWorkload:
    name: str
    x: torch.Tensor         # [R, hidden] bf16
    residual: torch.Tensor  # [R, hidden] bf16
    gamma: torch.Tensor     # [hidden] bf16
    eps: float


@dataclass
class VitWorkload:
    name: str
    grids: list             # [[t, h, w], ...]
    spatial_merge: int
    inv_t: torch.Tensor
    inv_h: torch.Tensor
    inv_w: torch.Tensor
    q: torch.Tensor         # [N, H, D] bf16 for the apply half
    k: torch.Tensor
    gamma_q: torch.Tensor
    gamma_k: torch.Tensor
    rot: int
    eps: float

    @property
    def n_tokens(self) -> int:
        return sum(t * h * w for t, h, w in self.grids)


# --------------------------------------------------------------------------
# Config 1: single-stream QK RMSNorm + NeoX RoPE, T=16, H=4, D=64, seed 0
# --------------------------------------------------------------------------

def config1(seed: int = 0, T: int = 16, H: int = 4, D: int = 64,
            theta: float = 10000.0, pairing: int = PAIRING_NEOX) -> RopeWorkload:
    g = _gen(seed)
    q = bf16_normal((T, H, D), g)
    k = bf16_normal((T, H, D), g)
    gq = bf16_uniform((D,), 0.5, 1.5, g)
    gk = bf16_uniform((D,), 0.5, 1.5, g)
    pos = torch.arange(T, dtype=torch.int32).reshape(1, T)
    angle = AngleInputs(kind=ANGLE_POSITIONS, section_mode=SECTIONS_NONE,
                        positions=pos, inv_freq=inv_freq(theta, D // 2, D))
    return RopeWorkload("single-stream qk-norm+rope T=%d H=%d D=%d" % (T, H, D),
                        [StreamInputs(q, k, gq, gk)], H, H, D, D, pairing, 1e-6, angle)


# --------------------------------------------------------------------------
# Config 2: hidden-size RMSNorm + residual
# --------------------------------------------------------------------------

def config2(R: int = 1, hidden: int = 5120, seed: int = 2) -> RmsWorkload:
    g = _gen(seed)
    x = bf16_normal((R, hidden), g)
    res = bf16_normal((R, hidden), g)
    gamma = bf16_uniform((hidden,), 0.5, 1.5, g)
    return RmsWorkload("rmsnorm+residual R=%d hidden=%d" % (R, hidden), x, res, gamma, 1e-6)


# --------------------------------------------------------------------------
# Config 3: joint text/image QK RMSNorm + cat + RoPE from a [cos|sin] table
# --------------------------------------------------------------------------

def joint_table(T_txt: int, img_h: int, img_w: int, n_pairs_per_axis: int,
                theta: float) -> tuple[torch.Tensor, torch.Tensor]:
    """fp32 cos/sin table [T_txt + img_h*img_w, 2*n_pairs_per_axis].

    Columns [0, n) carry the h axis, [n, 2n) the w axis, both with
    ``inv_freq_j = theta**(-2j/(2n))``.  Text token i has position i on both
    axes; image token (r, c), row-major over the grid, has h=r and w=c.
    The angle is the fp32 product ``fp32(pos) * inv_freq`` and cos/sin are
    evaluated in fp64 and rounded to fp32.
    """
    n = n_pairs_per_axis
    inv = inv_freq(theta, n, 2 * n).numpy()
    txt = np.arange(T_txt, dtype=np.int64)
    rr, cc = np.meshgrid(np.arange(img_h), np.arange(img_w), indexing="ij")
    pos_h = np.concatenate([txt, rr.reshape(-1)]).astype(np.float32)
    pos_w = np.concatenate([txt, cc.reshape(-1)]).astype(np.float32)
    ang = np.concatenate([pos_h[:, None] * inv[None, :], pos_w[:, None] * inv[None, :]],
                         axis=1).astype(np.float32)
    cos = np.cos(ang.astype(np.float64)).astype(np.float32)
    sin = np.sin(ang.astype(np.float64)).astype(np.float32)
    return torch.from_numpy(cos), torch.from_numpy(sin)


def config3(seed: int = 3, T_txt: int = 512, img_h: int = 64, img_w: int = 64,
            H: int = 24, D: int = 128, theta: float = 10000.0,
            pairing: int = PAIRING_GPTJ) -> RopeWorkload:
    g = _gen(seed)
    T_img = img_h * img_w
    txt = StreamInputs(bf16_normal((T_txt, H, D), g), bf16_normal((T_txt, H, D), g),
                       bf16_uniform((D,), 0.5, 1.5, g), bf16_uniform((D,), 0.5, 1.5, g))
    img = StreamInputs(bf16_normal((T_img, H, D), g), bf16_normal((T_img, H, D), g),
                       bf16_uniform((D,), 0.5, 1.5, g), bf16_uniform((D,), 0.5, 1.5, g))
    cos, sin = joint_table(T_txt, img_h, img_w, D // 4, theta)
    angle = AngleInputs(kind=ANGLE_TABLE, section_mode=SECTIONS_NONE,
                        cos=cos.unsqueeze(0), sin=sin.unsqueeze(0))
    return RopeWorkload("joint txt/img qk-norm+cat+rope T_txt=%d T_img=%d H=%d D=%d"
                        % (T_txt, T_img, H, D), [txt, img], H, H, D, D, pairing, 1e-6, angle)


# --------------------------------------------------------------------------
# Config 4: interleaved multi-section mRoPE on Q/K (no norm), GQA
# --------------------------------------------------------------------------

def config4(seed: int = 4, T: int = 8192, Hq: int = 16, Hkv: int = 8, D: int = 128,
            sections=(24, 20, 20), theta: float = 5e6,
            section_mode: int = SECTIONS_INTERLEAVED, pos_max: int = 8192) -> RopeWorkload:
    g = _gen(seed)
    q = bf16_normal((T, Hq, D), g)
    k = bf16_normal((T, Hkv, D), g)
    rows = 4 if section_mode == SECTIONS_IMROPE else 3
    pos = torch.randint(0, pos_max, (rows, T), generator=g, dtype=torch.int32)
    secs = tuple(sections) + (0,) * (4 - len(sections))
    angle = AngleInputs(kind=ANGLE_POSITIONS, section_mode=section_mode, sections=secs,
                        positions=pos, inv_freq=inv_freq(theta, D // 2, D))
    ones = torch.ones(D, dtype=torch.bfloat16)
    return RopeWorkload("interleaved mrope T=%d Hq=%d Hkv=%d D=%d" % (T, Hq, Hkv, D),
                        [StreamInputs(q, k, ones, ones)], Hq, Hkv, D, D, PAIRING_NEOX,
                        1e-6, angle, norm=False, extra={"chunk_split": 2457})


# --------------------------------------------------------------------------
# Config 5: ViT mRoPE setup + apply
# --------------------------------------------------------------------------

def config5(seed: int = 5, n_grids: int = 8, H: int = 16, D: int = 80, rot: int = 64,
            theta: float = 10000.0, lens=(16, 24, 24), spatial_merge: int = 2,
            grids: list | None = None) -> VitWorkload:
    g = _gen(seed)
    if grids is None:
        t = torch.randint(1, 3, (n_grids,), generator=g)
        h = 2 * torch.randint(8, 33, (n_grids,), generator=g)
        w = 2 * torch.randint(8, 33, (n_grids,), generator=g)
        grids = [[int(a), int(b), int(c)] for a, b, c in zip(t, h, w)]
    N = sum(a * b * c for a, b, c in grids)
    inv = [inv_freq(theta, n, 2 * n) for n in lens]
    q = bf16_normal((N, H, D), g)
    k = bf16_normal((N, H, D), g)
    gq = bf16_uniform((D,), 0.5, 1.5, g)
    gk = bf16_uniform((D,), 0.5, 1.5, g)
    return VitWorkload("vit mrope setup+apply G=%d N=%d H=%d D=%d" % (len(grids), N, H, D),
                       grids, spatial_merge, inv[0], inv[1], inv[2], q, k, gq, gk, rot, 1e-6)


def random_positions(rows: int, T: int, lo: int, hi: int, seed: int) -> torch.Tensor:
    g = _gen(seed)
    return torch.randint(lo, hi, (rows, T), generator=g, dtype=torch.int32)


def random_rope_case(seed: int, streams_T: list, Hq: int, Hk: int, D: int, rot: int,
                     pairing: int, angle: AngleInputs, norm: bool = True,
                     eps: float = 1e-6, scale: float = 1.0) -> RopeWorkload:
    """Generic small case used by parity and edge-case tests."""
    g = _gen(seed)
    streams = []
    for T in streams_T:
        q = bf16_normal((T, Hq, D), g)
        k = bf16_normal((T, Hk, D), g)
        if scale != 1.0:
            q = (q.float() * scale).to(torch.bfloat16)
            k = (k.float() * scale).to(torch.bfloat16)
        streams.append(StreamInputs(q, k, bf16_uniform((D,), 0.5, 1.5, g),
                                    bf16_uniform((D,), 0.5, 1.5, g)))
    return RopeWorkload("random case seed=%d" % seed, streams, Hq, Hk, D, rot, pairing,
                        eps, angle, norm=norm)
