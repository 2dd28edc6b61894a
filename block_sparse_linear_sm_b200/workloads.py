"""Seeded synthetic workloads for the sparse+linear attention layer.

This module only draws random numbers and rounds them to bf16. It holds none of
the layer's arithmetic, so both the CUDA path and the float64 oracle can take
their inputs from it without sharing any of the method.

Five workloads are defined, each named by what it is:

* ``tiny``       - B=1, H=2, N=1024, d=64; Q, K, V i.i.d. N(0, 1); k_h = k_l = 25 %.
* ``wan1.3b``    - B=1, H=12, d=128, 32760 tokens on a 21x30x52 (t, h, w) grid
                   padded to 32768; Q, K from 64 random Fourier features of the
                   grid position times a random 64x128 matrix plus 0.5 N(0, 1)
                   noise; V ~ N(0, 1); k_h = 5 %, k_l = 10 %.
* ``salad``      - the ``wan1.3b`` Q, K, V with k_h = 10 %, k_l = 0 and a
                   per-head sigmoid gate w_g ~ N(0, 1/d).
* ``nsa_causal`` - B=1, N=65536, 64 query heads over 4 KV heads, d=128; fixed
                   top-16 blocks per query block plus a 512-token causal window;
                   Q, V ~ N(0, 1), K ~ N(0, 1) plus a per-(KV head, block) mean
                   shift with standard deviation 0.5.
* ``wan14b``     - B=1, H=40, d=128, 75600 tokens on a 21x45x80 grid padded to
                   75648; same generator as ``wan1.3b``; k_h = 5 %, k_l = 10 %.

The video shapes follow the Wan2.1 models that the SLA page evaluates on; the
Fourier-feature tokens stand in for real DiT activations (no weights or videos
are used). Percentages become counts as k_h = ceil(p_h * nkb),
k_l = floor(p_l * nkb).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict
from typing import Optional

import numpy as np

MODE_THREEWAY = 0
MODE_TOPN_WINDOW = 1


@dataclass
class LayerConfig:
    """Shape and routing parameters of one attention layer (mirrors ``sla_config``)."""

    name: str
    B: int
    H: int
    H_kv: int
    N: int
    N_valid: int
    d: int
    block: int = 64
    mode: int = MODE_THREEWAY
    k_h: int = 0
    k_l: int = 0
    top_n: int = 0
    window: int = 0
    causal: int = 0
    has_proj: int = 1
    proj_per_head: int = 0        # 1: one W_p per query head ([H, d, d])
    has_gate: int = 0
    smooth_k: int = 0             # 1: linear branch on K minus the head's mean valid key
    linear_all: int = 0           # 1: linear branch over all valid key blocks
    cos_filter: int = 0           # 1: key blocks with CosSim < cos_theta score -inf
    scale: float = 0.0            # 0 -> 1/sqrt(d)
    cos_theta: float = 0.0
    nsa_branches: int = 0         # top-n mode: NSA's compressed, selected and window branches
    cmp_block: int = 32           # NSA compressed blocks: tokens per block ...
    cmp_stride: int = 16          # ... and stride
    generator: str = "iid"        # iid | fourier | block_shift
    grid: Optional[tuple] = None  # (t, h, w) for the Fourier generator
    seed: int = 0
    qkv_seed: Optional[int] = None  # Q/K/V stream seed when it differs from ``seed``

    @property
    def nqb(self) -> int:
        return self.N // self.block

    @property
    def nkb(self) -> int:
        return self.N // self.block

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale > 0 else 1.0 / math.sqrt(self.d)

    def replace(self, **kw) -> "LayerConfig":
        d = asdict(self)
        d.update(kw)
        return LayerConfig(**d)

    def dense_flops(self) -> float:
        """Dense-equivalent FLOP of the layer: 4 N_v^2 d H (causal: 4 d H N_v(N_v+1)/2)."""
        n = float(self.N_valid)
        if self.causal:
            return 4.0 * self.d * self.H * self.B * n * (n + 1) / 2.0
        return 4.0 * n * n * self.d * self.H * self.B


def _counts(p_h: float, p_l: float, nkb: int) -> tuple[int, int]:
    return int(math.ceil(p_h * nkb - 1e-9)), int(math.floor(p_l * nkb + 1e-9))


def _preset(name: str) -> LayerConfig:
    if name == "tiny":
        k_h, k_l = _counts(0.25, 0.25, 16)
        return LayerConfig(name, 1, 2, 2, 1024, 1024, 64, k_h=k_h, k_l=k_l,
                           has_proj=1, has_gate=0, generator="iid", seed=1001)
    if name == "wan1.3b":
        k_h, k_l = _counts(0.05, 0.10, 512)
        return LayerConfig(name, 1, 12, 12, 32768, 32760, 128, k_h=k_h, k_l=k_l,
                           has_proj=1, has_gate=0, generator="fourier",
                           grid=(21, 30, 52), seed=1002)
    if name == "salad":
        k_h, k_l = _counts(0.10, 0.0, 512)
        return LayerConfig(name, 1, 12, 12, 32768, 32760, 128, k_h=k_h, k_l=k_l,
                           has_proj=1, has_gate=1, generator="fourier",
                           grid=(21, 30, 52), seed=1003, qkv_seed=1002)
    if name == "nsa_causal":
        return LayerConfig(name, 1, 64, 4, 65536, 65536, 128, mode=MODE_TOPN_WINDOW,
                           top_n=16, window=512, causal=1, has_proj=0, has_gate=0,
                           generator="block_shift", seed=1004)
    if name == "nsa_branches":
        # NSA's three parallel branches on the NSA-shaped layer: compressed blocks of 32
        # tokens at stride 16, the top-16 selected blocks and the 512-token window, gated
        return _preset("nsa_causal").replace(name=name, nsa_branches=1, cmp_block=32, cmp_stride=16,
                                             has_gate=1)
    if name == "wan1.3b_opensource":
        # the SLA critique page's reading of the open-source code: smooth-K and the
        # linear branch over all tokens, on the Wan2.1-1.3B layer's inputs
        return _preset("wan1.3b").replace(name=name, smooth_k=1, linear_all=1)
    if name == "wan1.3b_cosfilter":
        # SpargeAttn's key-block similarity filter on the Wan2.1-1.3B layer: key blocks
        # whose tokens are least alike (CosSim < 0.1) drop out of the critical set
        return _preset("wan1.3b").replace(name=name, cos_filter=1, cos_theta=0.1)
    if name == "wan14b":
        k_h, k_l = _counts(0.05, 0.10, 1182)
        return LayerConfig(name, 1, 40, 40, 75648, 75600, 128, k_h=k_h, k_l=k_l,
                           has_proj=1, has_gate=0, generator="fourier",
                           grid=(21, 45, 80), seed=1005)
    raise KeyError(name)


PRESETS = ("tiny", "wan1.3b", "salad", "nsa_causal", "wan14b", "wan1.3b_opensource", "wan1.3b_cosfilter",
           "nsa_branches")


def preset(name: str) -> LayerConfig:
    return _preset(name)


# ---------------------------------------------------------------------------
# bf16 rounding (round to nearest even) on raw bits
# ---------------------------------------------------------------------------

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32/float64 values to bf16 (nearest even); returns uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact float64 values of bf16 bit patterns."""
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# generators
# ---------------------------------------------------------------------------

@dataclass
class LayerInputs:
    """bf16 bit patterns (uint16) of every input of one layer."""

    cfg: LayerConfig
    q: np.ndarray                  # [B, H, N, d]
    k: np.ndarray                  # [B, H_kv, N, d]
    v: np.ndarray                  # [B, H_kv, N, d]
    w_p: Optional[np.ndarray]      # [d, d], [H, d, d] (per-head projection) or None
    w_g: Optional[np.ndarray]      # [H, d] or None
    extra: dict = field(default_factory=dict)

    def f64(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        return None if a is None else bf16_bits_to_f64(a)


def _grid_coords(grid, n_valid):
    t, h, w = grid
    assert t * h * w == n_valid, (grid, n_valid)
    tt, hh, ww = np.meshgrid(np.arange(t), np.arange(h), np.arange(w), indexing="ij")
    return np.stack([tt.ravel(), hh.ravel(), ww.ravel()], axis=1).astype(np.float64)


def _fourier_head(rng: np.random.Generator, coords: np.ndarray, d: int, n_feat: int = 64):
    omega = rng.normal(0.0, 0.25, size=(n_feat, 3))
    beta = rng.uniform(0.0, 2.0 * np.pi, size=(n_feat,))
    feats = math.sqrt(2.0 / n_feat) * np.cos(coords @ omega.T + beta)      # [Nv, 64]
    a = rng.standard_normal((n_feat, d))
    base = feats @ a                                                          # [Nv, d]
    return base


def generate(cfg: LayerConfig, v_shift: float = 0.0) -> LayerInputs:
    """Draw the seeded inputs of ``cfg``; ``v_shift`` adds a constant to every valid V entry."""
    B, H, Hkv, N, Nv, d = cfg.B, cfg.H, cfg.H_kv, cfg.N, cfg.N_valid, cfg.d
    q = np.zeros((B, H, N, d), np.uint16)
    k = np.zeros((B, Hkv, N, d), np.uint16)
    v = np.zeros((B, Hkv, N, d), np.uint16)
    qkv_seed = cfg.qkv_seed if cfg.qkv_seed is not None else cfg.seed
    root = np.random.SeedSequence(qkv_seed)
    s_q, s_kv, s_w = root.spawn(3)
    q_streams = s_q.spawn(B * H)
    kv_streams = s_kv.spawn(B * Hkv)
    if cfg.generator == "fourier":
        coords = _grid_coords(cfg.grid, Nv)
    for b in range(B):
        for hk in range(Hkv):
            rng = np.random.Generator(np.random.PCG64(kv_streams[b * Hkv + hk]))
            vv = rng.standard_normal((Nv, d), dtype=np.float32) + np.float32(v_shift)
            v[b, hk, :Nv] = to_bf16_bits(vv)
            if cfg.generator == "fourier":
                # Q and K of a head share the Fourier basis and the 64 x d matrix;
                # the Q stream of the head draws it, K reuses it below.
                continue
            kk = rng.standard_normal((Nv, d), dtype=np.float32)
            if cfg.generator == "block_shift":
                nb = (Nv + cfg.block - 1) // cfg.block
                mu = rng.normal(0.0, 0.5, size=(nb, d)).astype(np.float32)
                kk += np.repeat(mu, cfg.block, axis=0)[:Nv]
            k[b, hk, :Nv] = to_bf16_bits(kk)
        for h in range(H):
            rng = np.random.Generator(np.random.PCG64(q_streams[b * H + h]))
            if cfg.generator == "fourier":
                assert H == Hkv
                base = _fourier_head(rng, coords, d)
                qq = base + 0.5 * rng.standard_normal((Nv, d))
                kk = base + 0.5 * rng.standard_normal((Nv, d))
                q[b, h, :Nv] = to_bf16_bits(qq)
                k[b, h, :Nv] = to_bf16_bits(kk)
            else:
                q[b, h, :Nv] = to_bf16_bits(rng.standard_normal((Nv, d), dtype=np.float32))
    wrng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(cfg.seed).spawn(4)[3]))
    wp_shape = (H, d, d) if cfg.proj_per_head else (d, d)
    w_p = to_bf16_bits(wrng.normal(0.0, 1.0 / math.sqrt(d), size=wp_shape)) if cfg.has_proj else None
    # gate vectors: one per head, or one per head and NSA branch (compressed, selected, window)
    wg_shape = (H, 3, d) if getattr(cfg, "nsa_branches", 0) else (H, d)
    w_g = to_bf16_bits(wrng.normal(0.0, 1.0 / math.sqrt(d), size=wg_shape)) if cfg.has_gate else None
    return LayerInputs(cfg, q, k, v, w_p, w_g)


def small_config(name="small", **kw) -> LayerConfig:
    """A small i.i.d. layer for tests; any field can be overridden."""
    base = dict(name=name, B=1, H=2, H_kv=2, N=512, N_valid=512, d=64, k_h=2, k_l=2,
                has_proj=1, has_gate=0, generator="iid", seed=7)
    base.update(kw)
    return LayerConfig(**base)
