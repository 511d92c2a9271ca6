"""Seeded synthetic inputs for the rotated W4A4 linear layer.

This module is shared by the CUDA path's harness (tests, bench) and by the CPU
oracle's callers.  It holds no arithmetic of the quantization method: it only
draws activations, weights and calibration tokens with the shapes and value
distributions of the five DiT-shaped linear layers below, and stores them as
BF16 bit patterns (uint16), the format both sides read.

Workloads (diffusion-transformer linears named on the pages: PixArt, FLUX.1-dev,
Wan 2.1):

=====  ==========================  =====  =====  =====  =====  ==========  =====
name   layer                       M      K      N      block  act / wgt    rank
=====  ==========================  =====  =====  =====  =====  ==========  =====
c1     tiny PixArt-width linear    256    1152   1152   128    INT4/INT4    0
c2     PixArt-like MLP fc1         4096   1152   4608   128    INT4/INT4    32
c3     FLUX.1-dev-like joint QKV   4608   3072   9216   128    LM16/LM16    0
c4     FLUX.1-dev-like MLP down    4608   12288  3072   256    NVFP4/NVFP4  0
c5     Wan-2.1-1.3B-like MLP, CFG  65520  1536   8960   128    LM16/LM4     0
=====  ==========================  =====  =====  =====  =====  ==========  =====

Activation recipes (a fixed set of outlier channels is a property of the layer,
so it is drawn from the layer seed; tokens are drawn from the token seed):

* c1, c2, c5: x ~ N(0,1), 4 outlier channels scaled x30, each token scaled by
  exp(0.5 * N(0,1)) (LogNormal(0, 0.5)).  c5 multiplies the second guidance
  branch (tokens 32760..65519) by 2.
* c3: x ~ N(0,1), 8 outlier channels x50, the 512 text tokens (4096..4607) x3.
* c4: x = GELU(z) with z ~ N(0,1) (exact erf form), 16 outlier channels x20.

Weights: W ~ N(0, 0.02) (standard deviation 0.02), N x K row-major.
Calibration tokens (c2's PCA basis): 512 tokens of the c1/c2 activation recipe
drawn with token seed 1.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "PCA_WORKLOADS", "workload", "bf16_bits", "bf16_to_f32", "activations", "weights",
    "calibration_tokens",
]

INT4, LM16, NVFP4, LM4 = 1, 2, 3, 4
FORMAT_NAMES = {INT4: "int4", LM16: "lm16", NVFP4: "nvfp4", LM4: "lm4"}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    block: int
    a_fmt: int
    w_fmt: int
    rank: int
    recipe: str
    description: str
    rotation: str = "rpbh"   # "pca": the full PCA rotation (rank = BF16 coordinates kept)


WORKLOADS = {
    "c1": Workload("c1", 256, 1152, 1152, 128, INT4, INT4, 0, "pixart",
                   "tiny PixArt-width linear, INT4 W4A4"),
    "c2": Workload("c2", 4096, 1152, 4608, 128, INT4, INT4, 32, "pixart",
                   "PixArt-like MLP fc1, INT4 W4A4 + rank-32 PCA branch"),
    "c3": Workload("c3", 4608, 3072, 9216, 128, LM16, LM16, 0, "flux_qkv",
                   "FLUX.1-dev-like joint-attention QKV, 16-level Lloyd-Max codes"),
    "c4": Workload("c4", 4608, 12288, 3072, 256, NVFP4, NVFP4, 0, "flux_gelu",
                   "FLUX.1-dev-like MLP down-projection, NVFP4"),
    "c5": Workload("c5", 65520, 1536, 8960, 128, LM16, LM4, 0, "wan_cfg",
                   "Wan-2.1-1.3B-like video MLP with CFG, W2A4"),
}

# The PixArt-like fc1 layer again, with the full PCA rotation in place of RPBH
# plus the rank-32 branch: y = x V, the first 32 coordinates in BF16.
PCA_WORKLOADS = {
    "c2p": Workload("c2p", 4096, 1152, 4608, 128, INT4, INT4, 32, "pixart",
                    "PixArt-like MLP fc1, INT4 W4A4 after the full PCA rotation, 32 coordinates in BF16", "pca"),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name] if name in WORKLOADS else PCA_WORKLOADS[name]

LAYER_SEED = 0
TOKEN_SEED = 0
WEIGHT_SEED = 0
CALIB_SEED = 1
CALIB_TOKENS = 512


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to BF16 (round to nearest, ties to even); return the
    16-bit patterns as uint16.  Inputs here are finite."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns (uint16) to float32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _outlier_channels(K: int, count: int, layer_seed: int) -> np.ndarray:
    rng = np.random.default_rng((layer_seed, 7, K, count))
    return np.sort(rng.choice(K, size=count, replace=False))


def _gelu(z: np.ndarray) -> np.ndarray:
    from scipy.special import erf
    return (0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))).astype(np.float32)


def activations(w: Workload, M: int | None = None, token_seed: int = TOKEN_SEED,
                layer_seed: int = LAYER_SEED, row0: int = 0) -> np.ndarray:
    """Activation rows ``row0 .. row0+M-1`` of workload ``w`` as BF16 bits (M x K).

    The rows are drawn for the full token range of the workload and sliced, so a
    short prefix is the same data the full-size run sees (only the first
    ``row0+M`` tokens are drawn)."""
    M = w.M if M is None else M
    K = w.K
    n = row0 + M
    rng = np.random.default_rng((token_seed, 11, K))
    if w.recipe in ("pixart", "wan_cfg"):
        x = rng.standard_normal((n, K), dtype=np.float32)
        x[:, _outlier_channels(K, 4, layer_seed)] *= np.float32(30.0)
        tok = np.exp(0.5 * rng.standard_normal(n)).astype(np.float32)
        x *= tok[:, None]
        if w.recipe == "wan_cfg":
            branch = np.where(np.arange(n) >= w.M // 2, 2.0, 1.0).astype(np.float32)
            x *= branch[:, None]
    elif w.recipe == "flux_qkv":
        x = rng.standard_normal((n, K), dtype=np.float32)
        x[:, _outlier_channels(K, 8, layer_seed)] *= np.float32(50.0)
        text = np.where(np.arange(n) >= 4096, 3.0, 1.0).astype(np.float32)
        x *= text[:, None]
    elif w.recipe == "flux_gelu":
        x = _gelu(rng.standard_normal((n, K), dtype=np.float32))
        x[:, _outlier_channels(K, 16, layer_seed)] *= np.float32(20.0)
    else:
        raise ValueError(w.recipe)
    return bf16_bits(x[row0:])


def weights(w: Workload, N: int | None = None, seed: int = WEIGHT_SEED) -> np.ndarray:
    """Weight rows (N x K) ~ N(0, 0.02) as BF16 bits."""
    N = w.N if N is None else N
    rng = np.random.default_rng((seed, 13, w.K, w.N))
    W = rng.standard_normal((N, w.K), dtype=np.float32) * np.float32(0.02)
    return bf16_bits(W)


def calibration_tokens(w: Workload, n: int = CALIB_TOKENS) -> np.ndarray:
    """Calibration tokens for the PCA branch: the layer's activation recipe drawn
    with token seed 1 (same outlier channels as the layer)."""
    return activations(w, M=n, token_seed=CALIB_SEED)
