"""Seeded synthetic inputs for the ConvRot W4A8 codebook linear layer.

This module is the one piece shared by the CUDA path's tests/benchmark and
the CPU oracle's tests: it only draws numbers.  It holds none of the method's
arithmetic (no decode, rotation, quantisation or contraction); dtype casts
to bf16 and fp8 are done by torch's own CPU conversions.

Recipe (shapes and distributions of the workloads the layer is tuned for,
"qwen3.8 shapes" on the ai-toolkit convrot_w4a8_quant.py page; no dataset
or trained checkpoint is involved):

* activations x [M, K] bf16: N(0, 1) drawn in fp64; ceil(0.01 K) channels
  chosen by the seed (fixed across tokens) are multiplied by 20; rounded
  to bf16 (nearest even).  The "gelu" variant (down-projection input) is
  GELU(z) = z * Phi(z) with the exact erf, in fp64, then rounded to bf16.
* packed codes qdata [N, K/2]: codes are i.i.d. uniform on 0..15 and two
  codes share a byte, so the packed bytes are i.i.d. uniform on 0..255;
  they are drawn as bytes directly.
* group scales srel [N, K/16]: U[32, 128] rounded to fp8 e4m3fn; stored as
  the fp8 byte.
* per-channel scales s_channel [N]: fp32 U[1e-4, 5e-4].
* codebook[16]: the page's FIXED_CODEBOOK rounded to fp32.
* rotated fp weights w_rot [N, K] fp32 (input of the offline quantiser):
  the page motivates the codebook by ConvRot making rotated groups
  Gaussian, so w = sigma_n * a_g * z with z ~ N(0, 1), a row scale sigma_n
  log-uniform on [0.005, 0.05] and a per-16-group factor a_g = exp(N(0,
  0.25^2)) so that group scales differ; drawn in fp64, rounded to fp32.
* uniform draws u [N, K] fp32 in [0, 1) for the stochastic code assignment.

Every tensor has its own counter-derived stream (seed, tag), so the weights
of a layer do not depend on M and vice versa.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np

# 16 Lloyd-Max levels for a group-normalised Gaussian (ai-toolkit
# convrot_w4a8_quant.py, FIXED_CODEBOOK).  Data, passed to both sides as an
# input.
FIXED_CODEBOOK = (
    -0.980602, -0.794529, -0.638165, -0.500986, -0.377321, -0.263187, -0.155210, -0.050720,
    0.052541, 0.156985, 0.265284, 0.379533, 0.502636, 0.638953, 0.794876, 0.980671,
)

_TAG_X, _TAG_OUTLIER, _TAG_Q, _TAG_S, _TAG_C, _TAG_BIAS = 1, 2, 3, 4, 5, 6
_TAG_W, _TAG_WROW, _TAG_WGROUP, _TAG_U = 7, 8, 9, 10


def _rng(seed: int, tag: int, extra: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), tag, int(extra)])))


def _to_bf16_bits(v64: np.ndarray) -> np.ndarray:
    import torch
    t = torch.from_numpy(np.ascontiguousarray(v64, dtype=np.float64)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def _to_fp8_bytes(v64: np.ndarray) -> np.ndarray:
    import torch
    t = torch.from_numpy(np.ascontiguousarray(v64, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy().copy()


def codebook() -> np.ndarray:
    return np.asarray(FIXED_CODEBOOK, dtype=np.float32)


@dataclass
class Layer:
    """Packed W4A8 storage of one linear (out N, in K)."""
    qdata: np.ndarray      # uint8 [N, K/2]  packed codes (even column = low nibble)
    srel: np.ndarray       # uint8 [N, K/16] fp8 e4m3fn group scale bytes
    s_channel: np.ndarray  # fp32  [N]
    codebook: np.ndarray   # fp32  [16]
    bias: Optional[np.ndarray] = None  # fp32 [N] or None

    @property
    def N(self) -> int:
        return self.qdata.shape[0]

    @property
    def K(self) -> int:
        return self.qdata.shape[1] * 2


def layer(N: int, K: int, seed: int, with_bias: bool = False) -> Layer:
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    q = _rng(seed, _TAG_Q).integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = _to_fp8_bytes(_rng(seed, _TAG_S).uniform(32.0, 128.0, size=(N, K // 16)))
    c = _rng(seed, _TAG_C).uniform(1e-4, 5e-4, size=(N,)).astype(np.float32)
    b = None
    if with_bias:
        b = _rng(seed, _TAG_BIAS).normal(0.0, 0.1, size=(N,)).astype(np.float32)
    return Layer(q, s, c, codebook(), b)


def rotated_weights(N: int, K: int, seed: int) -> np.ndarray:
    """fp32 [N, K] rotated weights for the offline quantiser (see the recipe)."""
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    sigma = np.exp(_rng(seed, _TAG_WROW).uniform(math.log(0.005), math.log(0.05), size=(N, 1, 1)))
    a = np.exp(_rng(seed, _TAG_WGROUP).normal(0.0, 0.25, size=(N, K // 16, 1)))
    z = _rng(seed, _TAG_W).standard_normal(size=(N, K // 16, 16))
    return (sigma * a * z).reshape(N, K).astype(np.float32)


def uniforms(N: int, K: int, seed: int) -> np.ndarray:
    """fp32 [N, K] uniform draws in [0, 1)."""
    return _rng(seed, _TAG_U).random(size=(N, K), dtype=np.float32)


def outlier_channels(K: int, seed: int) -> np.ndarray:
    count = int(math.ceil(0.01 * K))
    return np.sort(_rng(seed, _TAG_OUTLIER).choice(K, size=count, replace=False))


def activations(M: int, K: int, seed: int, dist: str = "outliers", row0: int = 0) -> np.ndarray:
    """bf16 bit patterns [M, K].  Rows are drawn per row index (row0 + i), so
    any row range of a large batch can be regenerated on its own."""
    out = np.empty((M, K), dtype=np.uint16)
    if M == 0:
        return out
    if dist == "outliers":
        ch = outlier_channels(K, seed)
    elif dist != "gelu":
        raise ValueError(dist)
    # One generator per block of 256 rows keeps row sampling cheap.
    blk = 256
    r = row0
    while r < row0 + M:
        b0 = (r // blk) * blk
        g = _rng(seed, _TAG_X, b0 // blk)
        z = g.standard_normal(size=(blk, K))
        lo = r - b0
        hi = min(blk, row0 + M - b0)
        z = z[lo:hi]
        if dist == "outliers":
            z[:, ch] *= 20.0
        else:
            from scipy.special import erf
            z = z * 0.5 * (1.0 + erf(z / math.sqrt(2.0)))
        out[r - row0: r - row0 + (hi - lo)] = _to_bf16_bits(z)
        r = b0 + hi
    return out


@dataclass(frozen=True)
class Case:
    name: str
    M: int
    N: int
    K: int
    seed: int
    dist: str = "outliers"


# The layer shapes the benchmark and the full-size parity tests run.
CASES = {
    "c1_decode_m1_1k": Case("c1_decode_m1_1k", 1, 1024, 1024, 0),
    "c2_decode_m8_4k": Case("c2_decode_m8_4k", 8, 4096, 4096, 1),
    "c3_prefill_2k_4k": Case("c3_prefill_2k_4k", 2048, 4096, 4096, 2),
    "c4_mlp_up": Case("c4_mlp_up", 4096, 12288, 4096, 3),
    "c4_mlp_down": Case("c4_mlp_down", 4096, 4096, 12288, 3, "gelu"),
    "c5_m1_8k": Case("c5_m1_8k", 1, 8192, 8192, 4),
    "c5_m2_8k": Case("c5_m2_8k", 2, 8192, 8192, 4),
    "c5_m4_8k": Case("c5_m4_8k", 4, 8192, 8192, 4),
    "c5_m8_8k": Case("c5_m8_8k", 8, 8192, 8192, 4),
    "c5_m16384_8k": Case("c5_m16384_8k", 16384, 8192, 8192, 4),
}
