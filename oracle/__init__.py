"""CPU oracle for the nested r-bit GEMM -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product library (``nested_bit_weight_b200``)
never imports it and shares no code with it; the two meet only through the
seeded generators in ``workloads.py``.

Each function states the passage it follows.  The method's definitions come
from the MatGPTQ pages (abstract of "MatGPTQ: Efficient and Accurate
Inference over Nested Quantized Models": r-bit models are read from the
parent by reading fewer bits, exactly r bits; author-page abstract of
"MatGPTQ: Accurate and Efficient Post-Training Matryoshka Quantization": the
most significant bits are sliced).  The dequantization formula and the
tolerance are the hot-path statement this library is built to:

    q_r = q >> (8 - r),   w = s_g * (2^(8-r) * q_r + 2^(7-r) - 128),
    |Y - Y_ref| <= 8e-3 * |Y_ref| + 1e-3 * rms(Y_ref)  per element.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the plain-C oracle with gcc (-O2, OpenMP, no SIMD intrinsics)."""
    if force or not os.path.exists(_LIB) or \
            os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.oracle_pack.argtypes = [P, I64, I64, P]
        lib.oracle_unpack.argtypes = [P, I64, I64, I, P]
        lib.oracle_gemm_f64.argtypes = [P, P, P, I64, I64, I64, I, P]
        lib.oracle_gemm_f64_at.argtypes = [P, P, P, I64, I, I64, P, P, P]
        lib.oracle_gemm_asym_f64.argtypes = [P, P, P, P, I64, I64, I64, I, P]
        lib.oracle_gemm_asym_f64_at.argtypes = [P, P, P, P, I64, I, I64, P, P, P]
        lib.oracle_threads.restype = I
        for f in (lib.oracle_pack, lib.oracle_unpack, lib.oracle_gemm_f64,
                  lib.oracle_gemm_f64_at, lib.oracle_gemm_asym_f64, lib.oracle_gemm_asym_f64_at):
            f.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def threads() -> int:
    return int(_load().oracle_threads())


# ---------------------------------------------------------------- definitions

def slice_codes(codes: np.ndarray, r: int) -> np.ndarray:
    """Top r bits of each 8-bit parent code (MSB slicing, integer floor)."""
    if not 1 <= r <= 8:
        raise ValueError("r must be in 1..8")
    return (codes.astype(np.uint8) >> np.uint8(8 - r)).astype(np.uint8)


def level(q_r: np.ndarray, r: int) -> np.ndarray:
    """v_r = 2^(8-r) q_r + 2^(7-r) - 128, exact in fp64."""
    return (2.0 ** (8 - r)) * q_r.astype(np.float64) + 2.0 ** (7 - r) - 128.0


def scales_f16(s: np.ndarray) -> np.ndarray:
    """The stored scale: fp32 s rounded to fp16 (round-to-nearest-even)."""
    with np.errstate(over="ignore"):
        return np.asarray(s, np.float32).astype(np.float16)


def dequant(codes: np.ndarray, s: np.ndarray, r: int) -> np.ndarray:
    """W_r[n, k] = s16[n, k // 128] * v_r(q_r[n, k]) in fp64."""
    s16 = scales_f16(s).astype(np.float64)
    v = level(slice_codes(codes, r), r)
    return v * np.repeat(s16, 128, axis=1)


# Asymmetric variant ("MatGPTQ: Efficient and Accurate Inference over Nested
# Quantized Models", captions of Tables 4-7, "asymmetric MatGPTQ"; no formula
# on the pages): a per-group zero point z, real, in units of the 8-bit code,
# stored as fp16 and shared by every r; the level is measured from it.

def level_asym(q_r: np.ndarray, r: int, z: np.ndarray) -> np.ndarray:
    """u_r = 2^(8-r) q_r + 2^(7-r) - z, in fp64 (z = 128: the symmetric level)."""
    return (2.0 ** (8 - r)) * q_r.astype(np.float64) + 2.0 ** (7 - r) - np.asarray(z, np.float64)


def zeros_f16(z: np.ndarray) -> np.ndarray:
    """The stored zero point: fp32 z rounded to fp16 (round-to-nearest-even)."""
    with np.errstate(over="ignore"):
        return np.asarray(z, np.float32).astype(np.float16)


def dequant_asym(codes: np.ndarray, s: np.ndarray, z: np.ndarray, r: int) -> np.ndarray:
    """W_r[n, k] = s16[n, k // 128] * u_r(q_r[n, k], z16[n, k // 128]) in fp64."""
    s16 = np.repeat(scales_f16(s).astype(np.float64), 128, axis=1)
    z16 = np.repeat(zeros_f16(z).astype(np.float64), 128, axis=1)
    return s16 * level_asym(slice_codes(codes, r), r, z16)


# ------------------------------------------------------------- plain-C kernels

def rows128(N: int) -> int:
    """Rows of the stored planes and scales: N padded to a multiple of 128."""
    return (N + 127) // 128 * 128


def pack(codes: np.ndarray) -> np.ndarray:
    """8 MSB-first bit planes in the tiled layout, uint32 [8, rows128(N) * K/32]."""
    codes = np.ascontiguousarray(codes, np.uint8)
    N, K = codes.shape
    out = np.empty((8, rows128(N) * (K // 32)), np.uint32)
    _load().oracle_pack(_ptr(codes), N, K, _ptr(out))
    return out


def unpack(planes: np.ndarray, r: int, N: int, K: int) -> np.ndarray:
    """r-bit codes read from the first r planes, uint8 [N, K]."""
    planes = np.ascontiguousarray(planes, np.uint32)
    if planes.size < r * rows128(N) * (K // 32):
        raise ValueError("plane buffer too small")
    out = np.empty((N, K), np.uint8)
    _load().oracle_unpack(_ptr(planes), N, K, r, _ptr(out))
    return out


def scales_stored(s: np.ndarray) -> np.ndarray:
    """The stored scales: fp16 (RNE) in the tiled order of the planes, the
    128 rows of block (t, g) contiguous at ((t * G + g) * 128); padding rows 0."""
    s16 = scales_f16(s)
    N, G = s16.shape
    Np = rows128(N)
    full = np.zeros((Np, G), np.float16)
    full[:N] = s16
    out = np.empty(Np * G, np.float16)
    for t in range(Np // 128):
        for g in range(G):
            out[(t * G + g) * 128:(t * G + g + 1) * 128] = full[t * 128:(t + 1) * 128, g]
    return out


def gemm(X: np.ndarray, codes: np.ndarray, s: np.ndarray, r: int) -> np.ndarray:
    """Y = X . W_r^T with fp64 accumulation in ascending k; Y is [M, N] fp64.

    X holds bf16 values (any float dtype holding them exactly); s is the fp32
    scale, rounded to its stored fp16 value here.
    """
    X = np.ascontiguousarray(X, np.float64)
    codes = np.ascontiguousarray(codes, np.uint8)
    s16 = np.ascontiguousarray(scales_f16(s).astype(np.float64))
    M, K = X.shape
    N = codes.shape[0]
    Y = np.empty((M, N), np.float64)
    _load().oracle_gemm_f64(_ptr(X), _ptr(codes), _ptr(s16), M, N, K, r, _ptr(Y))
    return Y


def zeros_stored(z: np.ndarray) -> np.ndarray:
    """The stored zero points: fp16 (RNE) in the same tiled order as the scales."""
    return scales_stored(np.asarray(zeros_f16(z), np.float32))


def gemm_asym(X: np.ndarray, codes: np.ndarray, s: np.ndarray, z: np.ndarray, r: int) -> np.ndarray:
    """Y = X . W_r^T for the asymmetric variant (fp64, ascending k)."""
    X = np.ascontiguousarray(X, np.float64)
    codes = np.ascontiguousarray(codes, np.uint8)
    s16 = np.ascontiguousarray(scales_f16(s).astype(np.float64))
    z16 = np.ascontiguousarray(zeros_f16(z).astype(np.float64))
    M, K = X.shape
    N = codes.shape[0]
    Y = np.empty((M, N), np.float64)
    _load().oracle_gemm_asym_f64(_ptr(X), _ptr(codes), _ptr(s16), _ptr(z16), M, N, K, r, _ptr(Y))
    return Y


def gemm_asym_at(X, codes, s, z, r, ms, ns) -> np.ndarray:
    """The asymmetric Y[ms[i], ns[i]] for a list of output positions."""
    X = np.ascontiguousarray(X, np.float64)
    codes = np.ascontiguousarray(codes, np.uint8)
    s16 = np.ascontiguousarray(scales_f16(s).astype(np.float64))
    z16 = np.ascontiguousarray(zeros_f16(z).astype(np.float64))
    ms = np.ascontiguousarray(ms, np.int64)
    ns = np.ascontiguousarray(ns, np.int64)
    out = np.empty(ms.shape[0], np.float64)
    _load().oracle_gemm_asym_f64_at(_ptr(X), _ptr(codes), _ptr(s16), _ptr(z16), X.shape[1], r,
                                    ms.shape[0], _ptr(ms), _ptr(ns), _ptr(out))
    return out


def gemm_at(X, codes, s, r, ms, ns) -> np.ndarray:
    """Y[ms[i], ns[i]] for a list of output positions (same definition)."""
    X = np.ascontiguousarray(X, np.float64)
    codes = np.ascontiguousarray(codes, np.uint8)
    s16 = np.ascontiguousarray(scales_f16(s).astype(np.float64))
    ms = np.ascontiguousarray(ms, np.int64)
    ns = np.ascontiguousarray(ns, np.int64)
    out = np.empty(ms.shape[0], np.float64)
    _load().oracle_gemm_f64_at(_ptr(X), _ptr(codes), _ptr(s16), X.shape[1], r,
                               ms.shape[0], _ptr(ms), _ptr(ns), _ptr(out))
    return out


# ------------------------------------------------------------------ tolerance

REL_TOL = 8e-3
RMS_TOL = 1e-3


def tolerance(Yref: np.ndarray, rms: float | None = None) -> np.ndarray:
    """Per-element bound 8e-3 |Y_ref| + 1e-3 rms(Y_ref) (rms over all of Y)."""
    Yref = np.asarray(Yref, np.float64)
    if rms is None:
        rms = float(np.sqrt(np.mean(Yref * Yref))) if Yref.size else 0.0
    return REL_TOL * np.abs(Yref) + RMS_TOL * rms


def violation_ratio(Y, Yref, rms: float | None = None) -> float:
    """max |Y - Y_ref| / bound; <= 1 means every element passes."""
    Y = np.asarray(Y, np.float64)
    Yref = np.asarray(Yref, np.float64)
    if Yref.size == 0:
        return 0.0
    tol = tolerance(Yref, rms)
    err = np.abs(Y - Yref)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(tol > 0, err / tol, np.where(err > 0, np.inf, 0.0))
    return float(ratio.max())


# ------------------------------------------------ per-layer bit-width search

def bitwidth_search_exhaustive(errors, nbytes, budget):
    """Every assignment of one candidate per layer (MatGPTQ author page,
    abstract: budget-aware search for heterogeneous per-layer bit-widths):
    returns (least summed error within the budget, its bytes, every optimal
    assignment at that error and byte count), or None if nothing fits.  The
    summed error is accumulated in layer order; assignments are compared by
    (error, bytes).  Small instances only."""
    import itertools
    L = len(errors)
    best = None
    for pick in itertools.product(*[range(len(row)) for row in errors]):
        b = sum(nbytes[l][pick[l]] for l in range(L))
        if b > budget:
            continue
        e = 0.0
        for l in range(L):
            e += errors[l][pick[l]]
        key = (e, b)
        if best is None or key < best[0]:
            best = (key, [pick])
        elif key == best[0]:
            best[1].append(pick)
    if best is None:
        return None
    return best[0][0], best[0][1], best[1]


# ------------------------------------------- one-shot multi-precision quantizer
# "MatGPTQ: Efficient and Accurate Inference over Nested Quantized Models"
# (abstract: a multi-precision objective with bit-slicing and cross-bit error
# compensation; Tables 6-7: the lambda weighting of the bit widths) on top of
# GPTQ's column loop.  The pages give prose only; the readings taken:
#   * U = the upper Cholesky factor of (H + damp * mean(diag H) * I)^-1;
#   * per 128-column group, when its first column is reached, the scale of a
#     row is s = alpha * max|w| / 127.5 over the group's current weights,
#     alpha searched over a small grid for the least lambda-weighted error of
#     the group (the scale search);
#   * each weight's 8-bit code minimises sum_r lambda_r (w - s v_r(q_r))^2 over
#     the nested levels of every r (ties: the smallest code);
#   * the error carried to the later columns is the lambda-weighted mean of
#     the slice errors: w_k+1.. -= e / U[k, k] * U[k, k+1..].

def matgptq_prepare(H: np.ndarray, damp: float = 0.01) -> np.ndarray:
    """U upper triangular with U^T U = (H + damp * mean(diag H) * I)^-1."""
    H = np.asarray(H, np.float64)
    K = H.shape[0]
    Hd = H + damp * float(np.mean(np.diag(H))) * np.eye(K)
    return np.linalg.cholesky(np.linalg.inv(Hd)).T


def _level_all(r: int) -> np.ndarray:
    """The r-bit level of every 8-bit code 0..255 (v_r of its top r bits)."""
    return level(np.arange(256) >> (8 - r), r)


def matgptq_best_code(w: float, s: float, rs, lams) -> int:
    """argmin over q in 0..255 of sum_r lambda_r (w - s v_r(q >> (8-r)))^2."""
    cost = np.zeros(256)
    for r, lam in zip(rs, lams):
        d = w - s * _level_all(r)
        cost += lam * d * d
    return int(np.argmin(cost))


def matgptq_quantize(W, U, rs=(3, 4, 8), lams=(1.0, 1.0, 1.0),
                     alphas=(1.0, 0.95, 0.9, 0.85, 0.8)):
    """codes uint8 [N, K], scales fp64 [N, K/128] by the column loop above."""
    W = np.array(W, np.float64, copy=True)
    U = np.asarray(U, np.float64)
    N, K = W.shape
    G = K // 128
    lsum = float(sum(lams))
    codes = np.zeros((N, K), np.uint8)
    scales = np.zeros((N, G), np.float64)
    for g in range(G):
        cols = range(128 * g, 128 * g + 128)
        for n in range(N):
            base = float(np.max(np.abs(W[n, 128 * g:128 * g + 128]))) / 127.5
            best_a, best_t = None, None
            for a in alphas:
                s = base * a
                t = 0.0
                for k in cols:
                    q = matgptq_best_code(W[n, k], s, rs, lams)
                    for r, lam in zip(rs, lams):
                        d = W[n, k] - s * float(level(np.array(q >> (8 - r)), r))
                        t += lam * d * d
                if best_t is None or t < best_t:
                    best_a, best_t = a, t
            scales[n, g] = base * best_a
        for k in cols:
            for n in range(N):
                s = scales[n, g]
                q = matgptq_best_code(W[n, k], s, rs, lams)
                codes[n, k] = q
                e = 0.0
                for r, lam in zip(rs, lams):
                    e += lam * (W[n, k] - s * float(level(np.array(q >> (8 - r)), r)))
                e /= lsum
                W[n, k + 1:] -= (e / U[k, k]) * U[k, k + 1:]
    return codes, scales


# ----------------------------- one-shot quantizer, asymmetric variant (R16)
# The same column loop with the asymmetric levels u_r = 2^(8-r) q_r +
# 2^(7-r) - z ("MatGPTQ: Efficient and Accurate Inference over Nested
# Quantized Models", captions of Tables 5-7: the evaluated models are
# asymmetric MatGPTQ).  Readings: per group and alpha, the grid spans
# alpha times the group's current range and is centred on it,
# s = alpha (hi - lo) / 255 and z = 128 - (hi + lo) / (2 s), z taken as
# stored (fp32, then fp16, RNE); s stays fp64 as in the symmetric loop.  A
# group whose range is zero, or whose z is not a finite fp16, takes the
# symmetric grid (s = alpha max|w| / 127.5, z = 128).

def matgptq_asym_grid(lo: float, hi: float, alpha: float):
    """(s, z16) of one group for one multiplier (fp64; z16 the stored value)."""
    if hi > lo:
        s = alpha * (hi - lo) / 255.0
        z = float(zeros_f16(np.array(128.0 - (hi + lo) / (2.0 * s))))
        if np.isfinite(z):
            return s, z
    return alpha * max(abs(lo), abs(hi)) / 127.5, 128.0


def _level_all_asym(r: int, z: float) -> np.ndarray:
    """The asymmetric r-bit level of every 8-bit code 0..255."""
    return level_asym(np.arange(256) >> (8 - r), r, z)


def matgptq_best_code_asym(w: float, s: float, z: float, rs, lams) -> int:
    """argmin over q of sum_r lambda_r (w - s u_r(q >> (8-r), z))^2."""
    cost = np.zeros(256)
    for r, lam in zip(rs, lams):
        d = w - s * _level_all_asym(r, z)
        cost += lam * d * d
    return int(np.argmin(cost))


def matgptq_quantize_asym(W, U, rs=(3, 4, 8), lams=(1.0, 1.0, 1.0),
                          alphas=(1.0, 0.95, 0.9, 0.85, 0.8)):
    """codes uint8 [N, K], scales fp64 [N, K/128], zero points [N, K/128]
    (the stored fp16 values, as fp64) by the column loop with asymmetric
    levels."""
    W = np.array(W, np.float64, copy=True)
    U = np.asarray(U, np.float64)
    N, K = W.shape
    G = K // 128
    lsum = float(sum(lams))
    codes = np.zeros((N, K), np.uint8)
    scales = np.zeros((N, G), np.float64)
    zeros = np.zeros((N, G), np.float64)

    def slice_err(w, s, z, q):
        out = []
        for r in rs:
            out.append(w - s * float(level_asym(np.array(q >> (8 - r)), r, z)))
        return out

    for g in range(G):
        cols = range(128 * g, 128 * g + 128)
        for n in range(N):
            seg = W[n, 128 * g:128 * g + 128]
            lo, hi = float(np.min(seg)), float(np.max(seg))
            best = None
            for a in alphas:
                s, z = matgptq_asym_grid(lo, hi, a)
                t = 0.0
                for k in cols:
                    q = matgptq_best_code_asym(W[n, k], s, z, rs, lams)
                    for lam, d in zip(lams, slice_err(W[n, k], s, z, q)):
                        t += lam * d * d
                if best is None or t < best[0]:
                    best = (t, s, z)
            scales[n, g], zeros[n, g] = best[1], best[2]
        for k in cols:
            for n in range(N):
                s, z = scales[n, g], zeros[n, g]
                q = matgptq_best_code_asym(W[n, k], s, z, rs, lams)
                codes[n, k] = q
                e = 0.0
                for lam, d in zip(lams, slice_err(W[n, k], s, z, q)):
                    e += lam * d
                e /= lsum
                W[n, k + 1:] -= (e / U[k, k]) * U[k, k + 1:]
    return codes, scales, zeros
