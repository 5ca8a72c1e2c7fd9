"""Seeded synthetic inputs for the nested r-bit GEMM workloads.

This module only *generates inputs*: parent codes, per-group scales and
activations of the shapes and value distributions of the benchmark layers.
It holds none of the method's arithmetic (no slicing, no bit-plane packing,
no dequantization, no matmul), so both the CPU oracle and the CUDA path can
be fed from it without sharing any computation.

Recipe (MatGPTQ page, abstract: an 8-bit parent from which r-bit children
are read; the layer shapes are Llama-3.1-8B / Qwen3-8B / 70B-class linear
layers):

* W ~ N(0, 0.02^2) in fp32; exactly floor(0.01 * N * K) entries, chosen
  without replacement, are multiplied by 10 (weight outliers).
* Per 128-wide group along K: s_g = fp32(max |W_g|) / 127.5 (fp32).
* Parent codes q = clamp(rint(W / s_g) + 128, 0, 255) as uint8, computed in
  fp32 with round-half-to-even; a group with s_g == 0 gets codes 128.
* X ~ N(0, 1) rounded to bf16 (round-to-nearest-even).  The Qwen3 chain
  additionally scales K/64 distinct channels (columns of X) by 20.
* Seeds: numpy default_rng(seed); X uses seed + 500.
"""
from __future__ import annotations

import dataclasses
import numpy as np

GROUP = 128


@dataclasses.dataclass(frozen=True)
class Layer:
    name: str
    N: int
    K: int


LLAMA8B = (
    Layer("q_proj", 4096, 4096), Layer("k_proj", 1024, 4096),
    Layer("v_proj", 1024, 4096), Layer("o_proj", 4096, 4096),
    Layer("gate_proj", 14336, 4096), Layer("up_proj", 14336, 4096),
    Layer("down_proj", 4096, 14336),
)
QWEN3_8B = (
    Layer("q_proj", 4096, 4096), Layer("k_proj", 1024, 4096),
    Layer("v_proj", 1024, 4096), Layer("o_proj", 4096, 4096),
    Layer("gate_proj", 12288, 4096), Layer("up_proj", 12288, 4096),
    Layer("down_proj", 4096, 12288),
)
LLAMA70B = (
    Layer("q_proj", 8192, 8192), Layer("k_proj", 1024, 8192),
    Layer("v_proj", 1024, 8192), Layer("o_proj", 8192, 8192),
    Layer("gate_proj", 28672, 8192), Layer("up_proj", 28672, 8192),
    Layer("down_proj", 8192, 28672),
)
# Qwen3 chain: attention projections at r=4, FFN projections at r=3.
QWEN3_R = {"q_proj": 4, "k_proj": 4, "v_proj": 4, "o_proj": 4,
           "gate_proj": 3, "up_proj": 3, "down_proj": 3}

CONFIGS = {
    0: dict(name="single 512x512 layer", layers=(Layer("layer", 512, 512),),
            M=(1,), r=(8, 6, 4, 3, 2)),
    1: dict(name="Llama-3.1-8B linears, decode M=1", layers=LLAMA8B,
            M=(1,), r=(4, 3, 2)),
    2: dict(name="Llama-3.1-8B linears, batch sweep", layers=LLAMA8B,
            M=(1, 2, 4, 8, 16, 32, 64), r=(8, 4, 3, 2)),
    3: dict(name="Qwen3-8B decoder chain, mixed r", layers=QWEN3_8B,
            M=(16, 64, 128), r=None),
    4: dict(name="70B-class linears, batch sweep", layers=LLAMA70B,
            M=(1, 8, 32, 128, 256), r=(8, 6, 4, 3, 2)),
}


def layer_seed(config: int, layer_index: int) -> int:
    return 1000 * config + layer_index


def gen_weights(N: int, K: int, seed: int, outlier_frac: float = 0.01):
    """Return (codes uint8 [N, K], scales fp32 [N, K/128], W fp32 [N, K])."""
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    n_out = int(np.floor(outlier_frac * N * K))
    if n_out:
        idx = rng.choice(N * K, size=n_out, replace=False)
        W.reshape(-1)[idx] *= np.float32(10.0)
    G = K // GROUP
    Wg = W.reshape(N, G, GROUP)
    absW = np.abs(Wg)
    s = absW.max(axis=2)
    del absW
    s /= np.float32(127.5)
    # q = rint(W / s) + 128 in fp32; W / s is formed as an exact fp32 division
    t = np.empty_like(Wg)
    np.divide(Wg, s[:, :, None], out=t, where=s[:, :, None] != 0)
    t[np.broadcast_to(s[:, :, None] == 0, t.shape)] = 0.0
    np.rint(t, out=t)
    t += np.float32(128.0)
    np.clip(t, 0, 255, out=t)
    codes = t.astype(np.uint8).reshape(N, K)
    return codes, s, W


def gen_weights_asym(N: int, K: int, seed: int, outlier_frac: float = 0.01):
    """Asymmetric codes: (codes uint8 [N, K], scales fp32 [N, K/128], zero
    points fp32 [N, K/128], W fp32 [N, K]).

    W as gen_weights plus a per-(row, group) offset ~ N(0, 0.02^2), so that
    groups are not centred; per group s = (max W - min W) / 255 and
    z = -min W / s (real, in code units); q = clamp(rint(W / s + z - 0.5),
    0, 255), so that the midpoint level s (q + 0.5 - z) is nearest to W.  A
    constant group gets s = 0, z = 128, codes 128.
    """
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    rng = np.random.default_rng(seed + 7919)
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    n_out = int(np.floor(outlier_frac * N * K))
    if n_out:
        idx = rng.choice(N * K, size=n_out, replace=False)
        W.reshape(-1)[idx] *= np.float32(10.0)
    G = K // GROUP
    Wg = W.reshape(N, G, GROUP)
    Wg += (rng.standard_normal((N, G, 1), dtype=np.float32) * np.float32(0.02))
    lo, hi = Wg.min(axis=2), Wg.max(axis=2)
    s = ((hi - lo) / np.float32(255.0)).astype(np.float32)
    z = np.full((N, G), 128.0, np.float32)
    nz = s != 0
    z[nz] = (-lo[nz] / s[nz]).astype(np.float32)
    t = np.zeros_like(Wg)
    np.divide(Wg, s[:, :, None], out=t, where=nz[:, :, None])
    t += z[:, :, None] - np.float32(0.5)
    np.rint(t, out=t)
    t[np.broadcast_to(~nz[:, :, None], t.shape)] = 128.0
    np.clip(t, 0, 255, out=t)
    return t.astype(np.uint8).reshape(N, K), s, z, W


def gen_x(M: int, K: int, seed: int, outlier_channels: bool = False):
    """Return X as (bf16 bit patterns uint16 [M, K], exact fp32 values [M, K]).

    X ~ N(0, 1) rounded once to bf16 (round-to-nearest-even, done by torch's
    CPU cast).  With ``outlier_channels`` K/64 distinct columns, drawn
    uniformly with the seed, are multiplied by 20 before the rounding.
    """
    import torch
    rng = np.random.default_rng(seed + 500)
    x = rng.standard_normal((M, K), dtype=np.float32)
    if outlier_channels:
        ch = rng.choice(K, size=K // 64, replace=False)
        x[:, ch] *= np.float32(20.0)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16).copy()
    return bits, xb.to(torch.float32).numpy()


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact: shift into the high half)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def adversarial_codes(kind: str, N: int, K: int, seed: int = 0) -> np.ndarray:
    """Hand-picked parent-code patterns that stress packing and decoding."""
    if kind == "zeros":
        return np.zeros((N, K), np.uint8)
    if kind == "ones":
        return np.full((N, K), 255, np.uint8)
    if kind == "alternating":
        c = np.zeros((N, K), np.uint8)
        c[:, 0::2] = 0xAA
        c[:, 1::2] = 0x55
        c[1::2] ^= 0xFF
        return c
    if kind == "single_bit":
        # row n, column k carries exactly the bit (k + n) % 8
        n = np.arange(N)[:, None]
        k = np.arange(K)[None, :]
        return (np.uint8(1) << ((k + n) % 8).astype(np.uint8)).astype(np.uint8)
    if kind == "all_codes":
        return (np.arange(N * K) % 256).astype(np.uint8).reshape(N, K)
    if kind == "random":
        return np.random.default_rng(seed).integers(0, 256, (N, K), dtype=np.uint8)
    raise ValueError(kind)


def gen_scales(N: int, K: int, seed: int, zero_groups: int = 0) -> np.ndarray:
    """Positive fp32 scales of the size the recipe produces (~1e-4..2e-2)."""
    rng = np.random.default_rng(seed + 77)
    s = (rng.uniform(0.2, 2.0, (N, K // GROUP)) * 1e-3).astype(np.float32)
    if zero_groups:
        idx = rng.choice(s.size, size=min(zero_groups, s.size), replace=False)
        s.reshape(-1)[idx] = 0.0
    return s


def gen_hessian(K: int, seed: int, corr: float = 0.9, samples: int | None = None) -> np.ndarray:
    """A layer's Hessian proxy H = X^T X / n (fp64, K x K) from synthetic
    calibration inputs: n = samples (default K + 1024) rows whose K columns
    follow an AR(1) process with coefficient `corr` (neighbouring input
    channels correlated, as activations are), unit variance.  Inputs only:
    the quantizer's own arithmetic starts from H."""
    n = samples if samples is not None else K + 1024
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((n, K), dtype=np.float32)
    X = np.empty_like(z)
    X[:, 0] = z[:, 0]
    c, d = np.float32(corr), np.float32(np.sqrt(1.0 - corr * corr))
    for k in range(1, K):
        X[:, k] = c * X[:, k - 1] + d * z[:, k]
    X64 = X.astype(np.float64)
    return X64.T @ X64 / n


def gen_float_weights(N: int, K: int, seed: int) -> np.ndarray:
    """Float weights to quantize (fp32, N x K): N(0, 0.02^2) with the same
    outlier recipe as gen_weights (1 % of entries x10)."""
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    n_out = int(0.01 * N * K)
    idx = rng.choice(N * K, size=n_out, replace=False)
    W.reshape(-1)[idx] *= np.float32(10.0)
    return W
