"""Seeded synthetic inputs for the hybrid dense / 2:4 weight product.

This module only draws random numbers: it holds none of the method's
arithmetic (no selection, no packing, no products).  Both the CUDA library's
tests and the CPU oracle's tests take their inputs from here, so the two sides
see the same bits.

Recipe (shapes and distributions of the workloads the pages run the method
on: Llama-class decode projections):
  * weights: fp32 N(0, std) from a seeded CPU ``torch.Generator``, rounded to
    bf16 (round-to-nearest-even); optional outliers: each entry with
    probability 0.01 is replaced by bf16(20 * w_fp32);
  * activations X[batch][k]: N(0, 1) rounded to bf16;
  * low-rank factors U[n][r], V[k][r]: N(0, std) rounded to bf16;
  * tile maps (1 = 2:4 tile, 0 = dense tile): an exact count of 2:4 tiles
    placed by a seeded shuffle, or independent Bernoulli(p) per tile.
All seeds derive from a base seed and a name through CRC-32, so every tensor
is reproducible on any machine.
"""
import zlib

import numpy as np
import torch

BASE_SEED = 20260101


def seed_of(*parts) -> int:
    """Stable 63-bit seed for a tensor named by ``parts``."""
    name = "/".join(str(p) for p in parts)
    return (BASE_SEED * 1000003 + zlib.crc32(name.encode())) & 0x7FFFFFFFFFFFFFFF


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a bf16 CPU tensor, as a numpy array."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray) -> torch.Tensor:
    """bf16 CPU tensor from uint16 bit patterns."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def normal_bf16(shape, std: float, seed: int) -> torch.Tensor:
    """fp32 N(0, std) rounded to bf16."""
    g = _gen(seed)
    w = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        w.mul_(std)
    return w.to(torch.bfloat16)


def weight(n: int, k: int, std: float, seed: int, outliers: float = 0.0,
           outlier_scale: float = 20.0) -> torch.Tensor:
    """bf16 [n][k] weight; with ``outliers`` > 0, that fraction of entries
    (Bernoulli per entry) is scaled by ``outlier_scale`` before rounding."""
    g = _gen(seed)
    w = torch.randn(n, k, generator=g, dtype=torch.float32)
    w.mul_(std)
    if outliers > 0.0:
        pick = torch.rand(n, k, generator=g) < outliers
        w = torch.where(pick, w * outlier_scale, w)
    return w.to(torch.bfloat16)


def activations(batch: int, k: int, seed: int) -> torch.Tensor:
    """bf16 X[batch][k] ~ N(0, 1)."""
    return normal_bf16((batch, k), 1.0, seed)


def lowrank(n: int, k: int, rank: int, std: float, seed: int):
    """bf16 U[n][rank], V[k][rank] ~ N(0, std)."""
    return normal_bf16((n, rank), std, seed), normal_bf16((k, rank), std, seed + 1)


def tile_map_exact(num_tiles: int, num_sparse: int, seed: int) -> np.ndarray:
    """Exactly ``num_sparse`` 2:4 tiles, positions from a seeded shuffle."""
    g = _gen(seed)
    perm = torch.randperm(num_tiles, generator=g).numpy()
    m = np.zeros(num_tiles, np.uint8)
    m[perm[:num_sparse]] = 1
    return m


def tile_map_fraction(num_tiles: int, frac: float, seed: int) -> np.ndarray:
    """round(frac * num_tiles) 2:4 tiles by seeded shuffle."""
    return tile_map_exact(num_tiles, int(round(frac * num_tiles)), seed)


def tile_map_bernoulli(num_tiles: int, p: float, seed: int) -> np.ndarray:
    """Each tile 2:4 with probability p, independently."""
    g = _gen(seed)
    return (torch.rand(num_tiles, generator=g) < p).numpy().astype(np.uint8)


def uniform(lo: float, hi: float, count: int, seed: int) -> np.ndarray:
    """``count`` draws from Uniform[lo, hi) (fp64)."""
    g = _gen(seed)
    return (lo + (hi - lo) * torch.rand(count, generator=g, dtype=torch.float64)).numpy()


# ---------------------------------------------------------------------------
# Named workloads.  Shapes are out x in (n x k); tiles b1 x b2 with b1 along n.
# ---------------------------------------------------------------------------

LLAMA8B_LAYER = [  # (role, n, k)
    ("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
    ("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336),
]
LLAMA70B_FFN = [("gate", 28672, 8192), ("up", 28672, 8192), ("down", 8192, 28672)]

WORKLOADS = {
    "tiny_256": dict(
        desc="one 256x256 bf16 weight N(0,0.02); 64x64 tiles, 8 of 16 2:4 by seeded "
             "shuffle; x batch 1 N(0,1)",
        matrices=[("w", 256, 256)], std=0.02, b1=64, b2=64, batch=[1]),
    "attn_4096": dict(
        desc="one 4096x4096 bf16 weight N(0,0.02); 128x128 tiles, each 2:4 with "
             "probability 0.5; x batch 1",
        matrices=[("q", 4096, 4096)], std=0.02, b1=128, b2=128, batch=[1]),
    "ffn_sweep": dict(
        desc="14336x4096 and 4096x14336 bf16 N(0,0.02) with 1% x20 outliers; "
             "128x128 tiles; 2:4-tile fraction {0,.25,.5,.75,1}; batch {1,4,8,16}",
        matrices=[("up", 14336, 4096), ("down", 4096, 14336)], std=0.02,
        outliers=0.01, b1=128, b2=128, fracs=[0.0, 0.25, 0.5, 0.75, 1.0],
        batch=[1, 4, 8, 16]),
    "llama8b_chain": dict(
        desc="32 Llama-3.1-8B-shaped layers (q,k,v,o,gate,up,down) bf16 N(0,0.02); "
             "128x64 tiles; per-layer 2:4-tile fraction ~ U[0.2,1.0]; batch 1, "
             "independent x per matrix",
        layers=32, matrices=LLAMA8B_LAYER, std=0.02, b1=128, b2=64, batch=[1]),
    "llama70b_ffn_lr": dict(
        desc="8 Llama-3.3-70B-shaped FFN layers (gate/up 28672x8192, down 8192x28672) "
             "bf16 N(0,0.015), all 2:4, 128x128 tiles, plus rank-128 U,V N(0,0.01); "
             "batch {1,8,16}",
        layers=8, matrices=LLAMA70B_FFN, std=0.015, b1=128, b2=128, rank=128,
        lr_std=0.01, batch=[1, 8, 16]),
}


def attn_map(num_tiles: int, seed_name="attn_4096") -> np.ndarray:
    return tile_map_bernoulli(num_tiles, 0.5, seed_of(seed_name, "map"))


def chain_fraction(layer: int) -> float:
    """Per-layer 2:4-tile fraction of the 32-layer chain, ~ U[0.2, 1.0]."""
    return float(uniform(0.2, 1.0, 32, seed_of("llama8b_chain", "fracs"))[layer])
