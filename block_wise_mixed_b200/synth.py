"""Seeded synthetic workloads for the block-wise mixed-precision linear layer.

This module only draws inputs: weights, activations, channel orders and the
per-block bit map.  It holds none of the quantization arithmetic, so both the
CUDA path and the CPU oracle can be fed from it.

The shapes are those of the Llama-2/3 layers that the ScaleBITS summary
("Experimental setup", "Key results") evaluates on; the pages' weights and
datasets are not used -- every value here is drawn from a seeded
``numpy.random.Generator(PCG64(seed))``:

* ``W``  = bf16(N(0, 0.02)) with 4 outlier input columns scaled by 10;
* ``x``  = bf16(N(0, 1)) with 3 outlier channels scaled by 20;
* channel orders: random, or a saliency sort (descending) that clusters large
  weights into the top-left blocks, the role bi-directional reordering plays in
  the ScaleBITS abstract and "Approach" section; ``None`` (identity) for the
  q/k projections, which the "Limitations" section excludes from reordering;
* bit map: drawn around the target average from the allowed set, nudged until
  the total matches ``round(avg * T)`` within 1, then assigned in descending
  order of block saliency, so high bit widths cluster where the salient
  weights are -- a stand-in for the budgeted bit-allocation search, which needs
  calibration data.

Seeds: ``seed = 1_000_000*cfg + 1_000*proj + replica``; x uses ``seed + 500``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

ALL_BITS = (0, 1, 2, 3, 4, 5, 6, 8)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def seed_of(cfg: int, proj: int = 0, replica: int = 0) -> int:
    return 1_000_000 * cfg + 1_000 * proj + replica


def make_weight(rng: np.random.Generator, N: int, K: int, std: float = 0.02,
                n_outlier_cols: int = 4, outlier_scale: float = 10.0) -> np.ndarray:
    w = rng.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(std)
    if n_outlier_cols:
        cols = rng.choice(K, size=min(n_outlier_cols, K), replace=False)
        w[:, cols] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(w)


def make_activation(rng: np.random.Generator, M: int, K: int,
                    n_outlier_ch: int = 3, outlier_scale: float = 20.0):
    x = rng.standard_normal((M, K), dtype=np.float32)
    ch = rng.choice(K, size=min(n_outlier_ch, K), replace=False)
    x[:, ch] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(x), ch


def saliency_perms(W_bits: np.ndarray, act_ch: np.ndarray):
    """Descending (stable) sort of rows and columns by a saliency score."""
    W = np.abs(bf16_bits_to_f32(W_bits)).astype(np.float64)
    a = np.ones(W.shape[1], np.float64)
    a[act_ch] = 20.0
    col_score = a * np.sqrt((W * W).sum(axis=0))
    row_score = (W * a[None, :]).sum(axis=1)
    row_perm = np.argsort(-row_score, kind="stable").astype(np.int32)
    col_perm = np.argsort(-col_score, kind="stable").astype(np.int32)
    return row_perm, col_perm


def make_bits(rng: np.random.Generator, NB: int, KB: int, avg: float,
              allowed=ALL_BITS, block_score: np.ndarray | None = None) -> np.ndarray:
    """Per-block bit map (uint8, NB*KB, row-major) with mean close to avg."""
    T = NB * KB
    allowed = np.array(sorted(allowed), dtype=np.int64)
    p = np.exp(-0.5 * (allowed - avg) ** 2)
    p /= p.sum()
    idx = rng.choice(len(allowed), size=T, p=p)
    target = int(round(avg * T))
    for _ in range(100 * T + 1000):
        total = int(allowed[idx].sum())
        if abs(total - target) <= 1:
            break
        t = int(rng.integers(T))
        if total < target and idx[t] < len(allowed) - 1:
            idx[t] += 1
        elif total > target and idx[t] > 0:
            idx[t] -= 1
    bits = np.sort(allowed[idx])[::-1]
    if block_score is None:
        order = rng.permutation(T)
    else:
        order = np.argsort(-np.asarray(block_score).reshape(-1), kind="stable")
    out = np.zeros(T, np.uint8)
    out[order] = bits.astype(np.uint8)
    return out


def block_saliency(W_bits, act_ch, row_perm, col_perm) -> np.ndarray:
    """Sum over each 64x128 block of a_j*|W'_ij| (W' = reordered W)."""
    W = np.abs(bf16_bits_to_f32(W_bits)).astype(np.float64)
    N, K = W.shape
    a = np.ones(K, np.float64)
    a[act_ch] = 20.0
    Wa = W * a[None, :]
    if row_perm is not None:
        Wa = Wa[row_perm]
    if col_perm is not None:
        Wa = Wa[:, col_perm]
    return Wa.reshape(N // 64, 64, K // 128, 128).sum(axis=(1, 3))


@dataclass
class Layer:
    name: str
    N: int
    K: int
    W: np.ndarray                  # uint16 bf16 bits, N x K, original order
    bits: np.ndarray               # uint8 [NB*KB]
    row_perm: np.ndarray | None    # int32 [N] or None (identity)
    col_perm: np.ndarray | None    # int32 [K] or None
    act_ch: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))

    @property
    def avg_bits(self) -> float:
        return float(self.bits.mean())

    @property
    def f0(self) -> float:
        return float((self.bits == 0).mean())


def make_layer(name: str, N: int, K: int, avg: float, seed: int,
               perms: str = "saliency", allowed=ALL_BITS) -> Layer:
    """One seeded layer.  perms: 'saliency', 'random' or 'identity'."""
    rng = np.random.Generator(np.random.PCG64(seed))
    W = make_weight(rng, N, K)
    xrng = np.random.Generator(np.random.PCG64(seed + 500))
    _, act_ch = make_activation(xrng, 1, K)
    if perms == "random":
        rp = rng.permutation(N).astype(np.int32)
        cp = rng.permutation(K).astype(np.int32)
    elif perms == "saliency":
        rp, cp = saliency_perms(W, act_ch)
    elif perms == "identity":
        rp, cp = None, None
    else:
        raise ValueError(perms)
    score = block_saliency(W, act_ch, rp, cp)
    bits = make_bits(rng, N // 64, K // 128, avg, allowed, score)
    return Layer(name, N, K, W, bits, rp, cp, act_ch)


def make_x(seed: int, M: int, K: int) -> np.ndarray:
    """Activations for a layer made with the same seed (bf16 bits, M x K)."""
    rng = np.random.Generator(np.random.PCG64(seed + 500))
    x, _ = make_activation(rng, M, K)
    return x


# ---------------------------------------------------------------------------
# The five workloads (shapes of the pages' Llama-2/3 evaluations)
# ---------------------------------------------------------------------------

LLAMA3_8B = [("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096),
             ("o", 4096, 4096), ("gate", 14336, 4096), ("up", 14336, 4096),
             ("down", 4096, 14336)]
LLAMA3_70B = [("q", 8192, 8192), ("k", 1024, 8192), ("v", 1024, 8192),
              ("o", 8192, 8192), ("gate", 28672, 8192), ("up", 28672, 8192),
              ("down", 8192, 28672)]

CONFIGS = {
    1: dict(desc="single linear 256x512, M=1, bits {0,1,2,3,4,8} avg 2.5, random perms",
            layers=[("lin", 256, 512)], M=[1], avg=2.5, allowed=(0, 1, 2, 3, 4, 8),
            perms="random"),
    2: dict(desc="Llama-2-7B attention projection 4096x4096, M=1, avg 2.1 bits",
            layers=[("attn", 4096, 4096)], M=[1], avg=2.1, allowed=ALL_BITS,
            perms="saliency"),
    3: dict(desc="Llama-3-8B MLP gate/up 14336x4096, down 4096x14336, M in {1,8,16,32}, avg 3.0",
            layers=[("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336)],
            M=[1, 8, 16, 32], avg=3.0, allowed=ALL_BITS, perms="saliency"),
    4: dict(desc="Llama-3-70B decoder layer, 7 projections, M in {1,4,16}, avg 2.1, identity order for q/k",
            layers=LLAMA3_70B, M=[1, 4, 16], avg=2.1, allowed=ALL_BITS,
            perms="saliency", identity=("q", "k")),
    5: dict(desc="Llama-3-8B layer prefill, 7 projections, M in {512,2048}, avg 4.0",
            layers=LLAMA3_8B, M=[512, 2048], avg=4.0, allowed=ALL_BITS,
            perms="saliency"),
}


def config_layer(cfg: int, proj: int, replica: int = 0, scale_rows: int | None = None) -> Layer:
    """Layer `proj` of workload `cfg`.  scale_rows (optional) trims N for tests."""
    c = CONFIGS[cfg]
    name, N, K = c["layers"][proj]
    if scale_rows is not None:
        N = min(N, scale_rows)
    perms = c["perms"]
    if name in c.get("identity", ()):
        perms = "identity"
    return make_layer(name, N, K, c["avg"], seed_of(cfg, proj, replica), perms,
                      c["allowed"])
