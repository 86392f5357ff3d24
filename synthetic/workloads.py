"""Seeded generators for the five synthetic workloads of the W4 + gated-EC layer.

Every array comes from numpy's PCG64 generator, sampled in fp32 and, where the
layer takes bf16, rounded to bf16 with round-to-nearest-even.  The shapes and
distributions follow the workload descriptions of the SPEAR hot path (the W4
per-channel linear with a per-token-gated low-rank error compensator):

  tiny       M=4,          N=K=512,                 r=16
  decode-qo  M in {1,4,16}, N=K=4096,               r=64, 1% outlier channels x20
  decode-mlp M in {1,8,32,64}, N=22016, K=4096,     r=64, gate bias -2 (easy tokens)
  prefill    M=2048, N=4096, K=14336,               r=128, Laplace(0,1) + 0.5% outliers x30
  sweep-1b   hidden 2048 / MLP 8192, 16 layers, EC r=32 on layers {0,1,7,15}

Readings of points the descriptions leave open are stated next to the code that
takes them.  Nothing here computes any part of the layer.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

CONFIG_NAMES = ["tiny", "decode-qo", "decode-mlp", "prefill", "sweep-1b"]

# Token counts per workload; the smaller batches use a prefix of the largest one.
CONFIG_M = {
    0: [4],
    1: [1, 4, 16],
    2: [1, 8, 32, 64],
    3: [2048],
    4: [1, 16, 256, 4096],
}

# ~1B-class model used by the sensitive-layer sweep: (name, N, K) per linear.
SWEEP_LINEARS = [("qkv", 6144, 2048), ("o", 2048, 2048), ("up_gate", 16384, 2048), ("down", 2048, 8192)]
SWEEP_LAYERS = 16
SWEEP_EC_LAYERS = (0, 1, 7, 15)
SWEEP_RANK = 32


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even) and return the 16-bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    nan = np.isnan(a)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Layer:
    """One linear layer's inputs.

    x_bits  uint16 [M_max, K]  bf16 activations (smaller M use the first rows)
    W       float32 [N, K]     master weights, quantised by the packer
    A_bits  uint16 [K, r]      bf16 EC down-projection, or None (no compensator)
    B_bits  uint16 [r, N]      bf16 EC up-projection, or None
    wg_bits uint16 [K]         bf16 gate weights, or None
    b_g     float              gate bias (fp32)
    """

    name: str
    N: int
    K: int
    rank: int
    x_bits: np.ndarray
    W: np.ndarray
    A_bits: Optional[np.ndarray]
    B_bits: Optional[np.ndarray]
    wg_bits: Optional[np.ndarray]
    b_g: float
    outlier_channels: np.ndarray

    def x(self, M: int) -> np.ndarray:
        return np.ascontiguousarray(self.x_bits[:M])


def _activations(rng: np.random.Generator, M: int, K: int, dist: str,
                 outlier_frac: float, outlier_scale: float):
    # Outlier channels: round(frac*K) channels picked by a seeded permutation, the
    # same channels for every token.
    n_out = int(round(outlier_frac * K))
    channels = np.sort(rng.permutation(K)[:n_out]) if n_out else np.zeros(0, np.int64)
    if dist == "normal":
        x = rng.standard_normal((M, K), dtype=np.float32)
    elif dist == "laplace":  # Laplace(0, b=1): variance 2
        x = rng.laplace(0.0, 1.0, size=(M, K)).astype(np.float32)
    else:
        raise ValueError(dist)
    if n_out:
        x[:, channels] *= np.float32(outlier_scale)
    return x, channels


def make_layer(name: str, seed, M: int, N: int, K: int, rank: int, *,
               x_dist: str = "normal", outlier_frac: float = 0.0, outlier_scale: float = 1.0,
               w_std: float = 0.02, ec_std: float = 0.01, wg_std: Optional[float] = 0.05,
               b_g: float = 0.0) -> Layer:
    """Draw one layer.  The draw order is fixed: channels, x, W, A, B, w_g."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x, channels = _activations(rng, M, K, x_dist, outlier_frac, outlier_scale)
    W = (rng.standard_normal((N, K), dtype=np.float32) * np.float32(w_std)).astype(np.float32)
    if rank > 0:
        A = rng.standard_normal((K, rank), dtype=np.float32) * np.float32(ec_std)
        B = rng.standard_normal((rank, N), dtype=np.float32) * np.float32(ec_std)
        if wg_std is None:
            # Reading of "b_g ~ N(-2,1), so ~85% of tokens get g<0.3": the per-token gate
            # pre-activation is N(-2, 1), i.e. w_g has std 1/sqrt(sum_k Var x_k).
            var = (K - len(channels)) * _var(x_dist) + len(channels) * _var(x_dist) * outlier_scale ** 2
            wg_std = 1.0 / np.sqrt(var)
        wg = rng.standard_normal(K, dtype=np.float32) * np.float32(wg_std)
        A_bits, B_bits, wg_bits = bf16_bits_from_f32(A), bf16_bits_from_f32(B), bf16_bits_from_f32(wg)
    else:
        A_bits = B_bits = wg_bits = None
    return Layer(name=name, N=N, K=K, rank=rank, x_bits=bf16_bits_from_f32(x), W=W,
                 A_bits=A_bits, B_bits=B_bits, wg_bits=wg_bits, b_g=float(b_g),
                 outlier_channels=channels)


def _var(dist: str) -> float:
    return 2.0 if dist == "laplace" else 1.0


def config_layers(idx: int, M: Optional[int] = None, layers=None):
    """Return the list of Layers of workload `idx` with M_max (or `M`) tokens.

    Seeds: 1000 + workload index; the sweep uses SeedSequence([1004, layer, linear]).
    """
    Mx = M if M is not None else max(CONFIG_M[idx])
    if idx == 0:
        return [make_layer("tiny", 1000, Mx, 512, 512, 16)]
    if idx == 1:
        return [make_layer("decode-qo", 1001, Mx, 4096, 4096, 64,
                           outlier_frac=0.01, outlier_scale=20.0)]
    if idx == 2:
        return [make_layer("decode-mlp", 1002, Mx, 22016, 4096, 64,
                           outlier_frac=0.01, outlier_scale=20.0, wg_std=None, b_g=-2.0)]
    if idx == 3:
        # EC factor and gate distributions are not given for this workload: the
        # tiny workload's (A, B ~ N(0, 0.01), w_g ~ N(0, 0.05), b_g = 0) are used.
        return [make_layer("prefill", 1003, Mx, 4096, 14336, 128, x_dist="laplace",
                           outlier_frac=0.005, outlier_scale=30.0, w_std=0.015)]
    if idx == 4:
        out = []
        for layer in (range(SWEEP_LAYERS) if layers is None else layers):
            for li, (lname, N, K) in enumerate(SWEEP_LINEARS):
                rank = SWEEP_RANK if layer in SWEEP_EC_LAYERS else 0
                seed = np.random.SeedSequence([1004, layer, li])
                out.append(make_layer(f"L{layer}.{lname}", seed, Mx, N, K, rank,
                                      outlier_frac=0.01, outlier_scale=20.0))
        return out
    raise ValueError(idx)
