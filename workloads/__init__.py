"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the sparse method (no pruning, packing or
GEMM): it only draws random numbers, rounds them to bf16 bit patterns and
names the workload shapes.  Both the CPU oracle and the CUDA library receive
the very same bytes from here.

Workloads (shapes and distributions of the pages' settings):
  tiny       W 64x128 ~N(0,1), X 128x32 ~N(0,1), 2:4, identity permutation.
  rl_mlp     three linear layers 17->256->256->6 of an off-policy RL agent,
             K padded with zero columns to a multiple of 8 (17 -> 24),
             W ~U(-1/sqrt(K), 1/sqrt(K)) on the unpadded K, batch T = 256,
             X ~N(0,1); each of the patterns 2:4, 1:4 and 1:8.
  llama7b    LLaMA-7B linear shapes 4096x4096, 11008x4096, 4096x11008 at 2:4,
             W ~N(0,0.02), X K x 2048 tokens ~N(0,1), and a seeded random
             column permutation as the index map (learned-permutation stand-in).
  patch      W 4096x4096 ~N(0,0.02) in 128x128 tiles, each tile 2:4 with
             probability p in {0.25, 0.5, 0.75} (seeded Bernoulli), else dense;
             X 4096 x 4096 tokens ~N(0,1).
  vit        ViT-B MLP shapes 3072x768 and 768x3072 at 1:8, X of
             197 tokens x 256 images = 50432 columns.
  decode     13824x5120 at 2:4 with a decode batch of 16 tokens.

Seeds: base seed s (0 by default); W draws from s, X from s+1, the index map
from s+2, the tile map from s+3; layer l of a multi-layer workload adds 10*l.
Numbers are drawn in float32 with numpy's PCG64 and rounded to bf16 with
round-to-nearest-even.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np


# --------------------------------------------------------------------------
# bf16 bit patterns
# --------------------------------------------------------------------------
def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal_bf16(shape, std: float, seed: int) -> np.ndarray:
    return bf16_bits(_rng(seed).standard_normal(shape, dtype=np.float32) * np.float32(std))


def uniform_bf16(shape, lo: float, hi: float, seed: int) -> np.ndarray:
    return bf16_bits(_rng(seed).uniform(lo, hi, size=shape).astype(np.float32))


def integer_bf16(shape, lo: int, hi: int, seed: int) -> np.ndarray:
    """Small integers (exact in bf16) drawn uniformly from [lo, hi]."""
    return bf16_bits(_rng(seed).integers(lo, hi + 1, size=shape).astype(np.float32))


def integer_i8(shape, lo: int, hi: int, seed: int) -> np.ndarray:
    """int8 values drawn uniformly from [lo, hi] (-128 <= lo <= hi <= 127)."""
    return _rng(seed).integers(lo, hi + 1, size=shape).astype(np.int8)


def normal_i8(shape, std: float, seed: int) -> np.ndarray:
    """int8 values: a normal draw scaled by std, rounded to nearest and clipped to [-128, 127]."""
    x = np.rint(_rng(seed).standard_normal(shape, dtype=np.float32) * np.float32(std))
    return np.clip(x, -128, 127).astype(np.int8)


def normal_f32(shape, std: float, seed: int) -> np.ndarray:
    return _rng(seed).standard_normal(shape, dtype=np.float32) * np.float32(std)


def integer_f32(shape, lo: int, hi: int, seed: int) -> np.ndarray:
    """Small integers as float32 (exact in TF32 too) drawn uniformly from [lo, hi]."""
    return _rng(seed).integers(lo, hi + 1, size=shape).astype(np.float32)


def permutation(K: int, seed: int) -> np.ndarray:
    return _rng(seed).permutation(K).astype(np.int32)


def tile_map(rows: int, cols: int, p: float, seed: int) -> np.ndarray:
    """uint8 rows x cols map, 1 (2:4 tile) with probability p, else 0 (dense tile)."""
    return (_rng(seed).random((rows, cols)) < p).astype(np.uint8)


# --------------------------------------------------------------------------
# Workload descriptions
# --------------------------------------------------------------------------
@dataclass
class Layer:
    name: str
    R: int
    K: int
    T: int
    n: int
    m: int
    w_dist: Tuple[str, float, float]       # ("normal", mean, std) or ("uniform", lo, hi)
    x_std: float = 1.0
    seed: int = 0
    permuted: bool = False
    k_valid: Optional[int] = None          # K before zero padding (None: K)
    tile_p: Optional[float] = None         # PATCH tile probability (None: not hybrid)
    tile: int = 128

    @property
    def useful_flops(self) -> int:
        """2 * T * (stored survivors R*K*N/M): the structural non-zeros."""
        if self.tile_p is not None:
            raise ValueError("hybrid flops depend on the drawn tile map; use hybrid_useful_flops")
        return 2 * self.T * self.R * (self.K // self.m * self.n)


@dataclass
class LayerData:
    layer: Layer
    W: np.ndarray                      # R x K uint16 (bf16 bits)
    X: np.ndarray                      # K x T uint16
    idx: Optional[np.ndarray] = None   # K int32
    tmap: Optional[np.ndarray] = None  # ceil(R/tile) x ceil(K/tile) uint8


def make_layer(L: Layer) -> LayerData:
    s = L.seed
    kv = L.k_valid or L.K
    if L.w_dist[0] == "normal":
        W = normal_bf16((L.R, kv), L.w_dist[2], s)
    elif L.w_dist[0] == "uniform":
        W = uniform_bf16((L.R, kv), L.w_dist[1], L.w_dist[2], s)
    elif L.w_dist[0] == "integer":
        W = integer_bf16((L.R, kv), int(L.w_dist[1]), int(L.w_dist[2]), s)
    else:
        raise ValueError(L.w_dist)
    X = normal_bf16((kv, L.T), L.x_std, s + 1)
    if kv != L.K:  # zero padding of the reduction axis
        W = np.concatenate([W, np.zeros((L.R, L.K - kv), np.uint16)], axis=1)
        X = np.concatenate([X, np.zeros((L.K - kv, L.T), np.uint16)], axis=0)
    idx = permutation(L.K, s + 2) if L.permuted else None
    tm = None
    if L.tile_p is not None:
        tm = tile_map(-(-L.R // L.tile), -(-L.K // L.tile), L.tile_p, s + 3)
    return LayerData(L, np.ascontiguousarray(W), np.ascontiguousarray(X), idx, tm)


def hybrid_useful_flops(d: LayerData) -> int:
    """2*T*(dense-tile elements + half of the 2:4-tile elements)."""
    L = d.layer
    total = 0
    for i in range(d.tmap.shape[0]):
        rows = min(L.tile, L.R - i * L.tile)
        for j in range(d.tmap.shape[1]):
            cols = min(L.tile, L.K - j * L.tile)
            total += rows * (cols // 2 if d.tmap[i, j] else cols)
    return 2 * L.T * total


def workload(name: str, seed: int = 0) -> List[Layer]:
    """Layer list of a named workload."""
    if name == "tiny":
        return [Layer("tiny_64x128x32", 64, 128, 32, 2, 4, ("normal", 0.0, 1.0), seed=seed)]
    if name.startswith("rl_mlp"):
        # rl_mlp_2of4 / rl_mlp_1of4 / rl_mlp_1of8
        pat = {"rl_mlp_2of4": (2, 4), "rl_mlp_1of4": (1, 4), "rl_mlp_1of8": (1, 8)}[name]
        dims = [(256, 24, 17), (256, 256, 256), (6, 256, 256)]
        return [Layer(f"{name}_l{i}_{R}x{kv}", R, K, 256, pat[0], pat[1],
                      ("uniform", -1.0 / np.sqrt(kv), 1.0 / np.sqrt(kv)),
                      seed=seed + 10 * i, k_valid=kv if kv != K else None)
                for i, (R, K, kv) in enumerate(dims)]
    if name == "llama7b":
        dims = [(4096, 4096), (11008, 4096), (4096, 11008)]
        return [Layer(f"llama7b_{R}x{K}", R, K, 2048, 2, 4, ("normal", 0.0, 0.02),
                      seed=seed + 10 * i, permuted=True) for i, (R, K) in enumerate(dims)]
    if name.startswith("patch"):
        p = {"patch_p25": 0.25, "patch_p50": 0.5, "patch_p75": 0.75}[name]
        return [Layer(f"{name}_4096x4096x4096", 4096, 4096, 4096, 2, 4, ("normal", 0.0, 0.02),
                      seed=seed, tile_p=p)]
    if name == "vit":
        return [Layer(f"vit_{R}x{K}_1of8", R, K, 197 * 256, 1, 8, ("normal", 0.0, 0.02),
                      seed=seed + 10 * i) for i, (R, K) in enumerate([(3072, 768), (768, 3072)])]
    if name == "decode":
        return [Layer("decode_13824x5120x16", 13824, 5120, 16, 2, 4, ("normal", 0.0, 0.02), seed=seed)]
    raise KeyError(name)


ALL_WORKLOADS = ["tiny", "rl_mlp_2of4", "rl_mlp_1of4", "rl_mlp_1of8", "llama7b",
                 "patch_p25", "patch_p50", "patch_p75", "vit", "decode"]
