"""Seeded synthetic inputs shared by the oracle's tests, the GPU parity tests and the benchmark.

This module only draws random numbers and fixes shapes. It holds none of the method's
arithmetic (no quantisation, normalisation, gating or recurrence), so that the oracle and the
CUDA path can both consume its arrays without sharing any computation.

Workload shapes follow the model table of the MatMul-free LM pages (hysenlabs.com,
"HGRNBitBlock structure" and "three pretrained models" sections): 370M is 24 layers of hidden
1024, 1.3B is 24 layers of hidden 2048 (gate_proj 2048->11264, down_proj 5632->2048), 2.7B is
32 layers of hidden 2560; the vocabulary is 32000.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

VOCAB = 32000


@dataclass(frozen=True)
class BlockShape:
    """Sizes of one HGRNBit block: hidden d, MLP inner I (gate_proj emits 2*I), layer count."""

    name: str
    d: int
    inner: int
    n_layers: int

    @property
    def proj_shapes(self) -> dict[str, tuple[int, int]]:
        """(out_features N, in_features K) of every ternary projection in a block."""
        d, i = self.d, self.inner
        return {
            "i": (d, d), "f": (d, d), "g": (d, d), "o": (d, d),
            "gate": (2 * i, d), "down": (d, i),
        }


TINY = BlockShape("tiny", 256, 704, 1)
M370 = BlockShape("370M", 1024, 2816, 24)
B13 = BlockShape("1.3B", 2048, 5632, 24)
B27 = BlockShape("2.7B", 2560, 7040, 32)
SHAPES = {s.name: s for s in (TINY, M370, B13, B27)}


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def weight(seed: int, n: int, k: int, std: float = 0.02) -> np.ndarray:
    """Latent full-precision weight [n, k] ~ N(0, std^2), float32 (PyTorch Linear layout)."""
    return (rng(seed).standard_normal((n, k), dtype=np.float32) * np.float32(std))


def norm_weight(seed: int, k: int, random: bool = False) -> np.ndarray:
    """RMSNorm gain [k]: ones (the usual init) or N(1, 0.1^2) to exercise the gain path."""
    if not random:
        return np.ones(k, dtype=np.float32)
    return (1.0 + 0.1 * rng(seed).standard_normal(k)).astype(np.float32)


def activations(seed: int, shape: tuple[int, ...], std: float = 1.0) -> np.ndarray:
    """Activations ~ N(0, std^2), float32."""
    return (rng(seed).standard_normal(shape, dtype=np.float32) * np.float32(std))


def token_ids(seed: int, shape: tuple[int, ...], vocab: int = VOCAB) -> np.ndarray:
    """Token ids uniform in [0, vocab), int32."""
    return rng(seed).integers(0, vocab, size=shape, dtype=np.int64).astype(np.int32)


def scan_inputs(seed: int, b: int, t: int, d: int, long_memory: bool) -> tuple[np.ndarray, np.ndarray]:
    """Gate pre-activations for the recurrence sweep: zf ~ N(4,1) (long memory) or N(0,1);
    zi ~ N(0,1). float32 [b, t, d] each."""
    r = rng(seed)
    zf = r.standard_normal((b, t, d), dtype=np.float32) + np.float32(4.0 if long_memory else 0.0)
    zi = r.standard_normal((b, t, d), dtype=np.float32)
    return zf, zi


def block_params(seed: int, shape: BlockShape, random_norms: bool = False) -> dict[str, np.ndarray]:
    """Latent weights and norm gains of one block, keyed by projection name.

    Keys: 'W_<p>' [N,K] for p in i,f,g,o,gate,down; 'nw_<p>' [K]; 'gnorm_w' [d].
    """
    out: dict[str, np.ndarray] = {}
    for j, (p, (n, k)) in enumerate(shape.proj_shapes.items()):
        out[f"W_{p}"] = weight(seed * 1000 + j, n, k)
        out[f"nw_{p}"] = norm_weight(seed * 1000 + 100 + j, k, random_norms)
    out["gnorm_w"] = norm_weight(seed * 1000 + 200, shape.d, random_norms)
    return out


def embedding(seed: int, vocab: int, d: int) -> np.ndarray:
    """Token embedding table [vocab, d] ~ N(0, 0.02^2), float32."""
    return weight(seed, vocab, d, std=0.02)
