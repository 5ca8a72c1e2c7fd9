"""Pins of the oracle's asymmetric variant ("MatGPTQ: Efficient and Accurate
Inference over Nested Quantized Models", captions of Tables 4-7, "asymmetric
MatGPTQ"; the reading: a per-group zero point z in code units, fp16-stored,
shared by every r, level u_r = 2^(8-r) q_r + 2^(7-r) - z).  Each pin fixes
the result by something other than the oracle itself: the symmetric oracle
at z = 128, exact rational arithmetic, a closed form, linearity in z, the
dequantized column, and the stored layout; planted mistakes in a scratch
copy of the C oracle must fail them."""
import ctypes
import os
import subprocess
import tempfile
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as wl


def _case(N=4, K=256, M=3, seed=0):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, (N, K)).astype(np.uint8)
    s = (rng.random((N, K // 128)) * 0.01 + 1e-3).astype(np.float32)
    z = (rng.random((N, K // 128)) * 255.0).astype(np.float32)
    X = rng.standard_normal((M, K)).astype(np.float32)
    return codes, s, z, X


def _exact_asym(X, codes, s, z, r):
    s16 = oracle.scales_f16(s).astype(np.float64)
    z16 = oracle.zeros_f16(z).astype(np.float64)
    M, K = X.shape
    N = codes.shape[0]
    Y = np.empty((M, N))
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                q_r = int(codes[n, k]) >> (8 - r)
                u = Fraction(2 ** (8 - r)) * q_r + Fraction(2) ** (7 - r) - Fraction(float(z16[n, k // 128]))
                acc += Fraction(float(X[m, k])) * Fraction(float(s16[n, k // 128])) * u
            Y[m, n] = float(acc)
    return Y


@pytest.mark.parametrize("r", [8, 5, 4, 2, 1])
def test_z128_is_the_symmetric_oracle(r):
    codes, s, _, X = _case(N=6, K=384, M=4, seed=r)
    z = np.full_like(s, 128.0)
    assert np.array_equal(oracle.gemm_asym(X, codes, s, z, r), oracle.gemm(X, codes, s, r))
    ms, ns = np.array([0, 3, 2]), np.array([5, 0, 4])
    assert np.array_equal(oracle.gemm_asym_at(X, codes, s, z, r, ms, ns),
                          oracle.gemm_at(X, codes, s, r, ms, ns))


@pytest.mark.parametrize("r", [8, 6, 3, 1])
def test_asym_exact_rational_bruteforce(r):
    codes, s, z, X = _case(N=3, K=256, M=2, seed=10 + r)
    Y = oracle.gemm_asym(X, codes, s, z, r)
    ref = _exact_asym(X, codes, s, z, r)
    assert np.max(np.abs(Y - ref) / (np.abs(ref) + 1e-30)) < 1e-12


@pytest.mark.parametrize("r", [8, 4, 2])
def test_ones_over_one_group_closed_form(r):
    # X = 1 on group g only: y[n] = s (2^(8-r) sum q_r + 128 (2^(7-r) - z))
    codes, s, z, _ = _case(N=5, K=384, M=1, seed=20 + r)
    g = 1
    X = np.zeros((1, 384), np.float32)
    X[0, 128 * g:128 * (g + 1)] = 1.0
    Y = oracle.gemm_asym(X, codes, s, z, r)[0]
    s16 = oracle.scales_f16(s).astype(np.float64)[:, g]
    z16 = oracle.zeros_f16(z).astype(np.float64)[:, g]
    qsum = (codes[:, 128 * g:128 * (g + 1)].astype(np.int64) >> (8 - r)).sum(axis=1)
    want = s16 * (2.0 ** (8 - r) * qsum + 128 * (2.0 ** (7 - r) - z16))
    assert np.allclose(Y, want, rtol=1e-13, atol=0)


def test_linear_in_the_zero_point():
    # raising z of (row n, group g) by d lowers y[m, n] by s d sum_{k in g} x,
    # and nothing else
    codes, s, z, X = _case(N=4, K=384, M=3, seed=30)
    z = oracle.zeros_f16(z).astype(np.float32)       # exact fp16 values
    n, g, d = 2, 2, np.float32(16.0)
    z2 = z.copy()
    z2[n, g] += d
    Y1, Y2 = oracle.gemm_asym(X, codes, s, z, 4), oracle.gemm_asym(X, codes, s, z2, 4)
    s16 = float(oracle.scales_f16(s)[n, g])
    diff = Y2 - Y1
    want = -s16 * float(d) * X[:, 128 * g:128 * (g + 1)].astype(np.float64).sum(axis=1)
    assert np.allclose(diff[:, n], want, rtol=1e-12, atol=1e-15)
    others = np.delete(diff, n, axis=1)
    assert np.all(others == 0)


@pytest.mark.parametrize("r", [8, 3])
def test_one_hot_gives_dequantized_column(r):
    codes, s, z, _ = _case(N=5, K=256, M=1, seed=40 + r)
    Wr = oracle.dequant_asym(codes, s, z, r)
    for k in (0, 77, 128, 255):
        X = np.zeros((1, 256), np.float32)
        X[0, k] = 1.0
        assert np.array_equal(oracle.gemm_asym(X, codes, s, z, r)[0], Wr[:, k])


def test_zeros_stored_layout():
    _, s, z, _ = _case(N=130, K=384, M=1, seed=50)
    st = oracle.zeros_stored(z)
    z16 = oracle.zeros_f16(z)
    G = 3
    for (n, g) in ((0, 0), (127, 2), (128, 1), (129, 0)):
        assert st[((n // 128) * G + g) * 128 + n % 128] == z16[n, g]
    assert np.all(st[((1 * G + 0) * 128 + 2):((1 * G + 0) * 128 + 128)] == 0)   # padding rows


def test_generator_asym_recipe():
    codes, s, z, W = wl.gen_weights_asym(64, 256, seed=3)
    assert codes.dtype == np.uint8 and s.shape == z.shape == (64, 2)
    # z is real and may fall outside [0, 255] (a group whose values are all
    # of one sign); it must still fit fp16
    assert np.all(s > 0) and np.all(np.isfinite(z)) and np.all(np.abs(z) < 65504)
    # the midpoint level reconstructs W to within half a step plus the fp16
    # rounding of s (2^-11 relative, times up to 255 steps) and of z
    Wr = oracle.dequant_asym(codes, s, z, 8)
    step = np.repeat(oracle.scales_f16(s).astype(np.float64), 128, axis=1)
    assert np.all(np.abs(Wr - W) <= (0.5 + 256 * 2.0 ** -11 + 0.05) * step + 1e-6)


MUTATIONS = {
    "z_sign": ("return a * (double)q_r + b - z;", "return a * (double)q_r + b + z;"),
    "z_dropped": ("return a * (double)q_r + b - z;", "return a * (double)q_r + b - 128.0;"),
    "z_index": ("level_asym(q_r, r, z16[n * G + k / 128])", "level_asym(q_r, r, z16[n * G + k % G])"),
    "z_half_step": ("return a * (double)q_r + b - z;", "return a * (double)q_r - z;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_asym_mutation_is_caught(name):
    old, new = MUTATIONS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "mq_oracle.c")).read()
    assert src.count(old) >= 1
    d = tempfile.mkdtemp(prefix="mq_mut_asym_")
    c, so = os.path.join(d, "m.c"), os.path.join(d, "m.so")
    open(c, "w").write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-o", so, c])
    lib = ctypes.CDLL(so)
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.oracle_gemm_asym_f64_at.argtypes = [P, P, P, P, I64, I, I64, P, P, P]
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    codes, s, z, X = _case(N=3, K=256, M=2, seed=60)
    s16 = np.ascontiguousarray(oracle.scales_f16(s).astype(np.float64))
    z16 = np.ascontiguousarray(oracle.zeros_f16(z).astype(np.float64))
    X64 = np.ascontiguousarray(X, np.float64)
    caught = False
    for r in (8, 4):
        ms = np.repeat(np.arange(2), 3).astype(np.int64)
        ns = np.tile(np.arange(3), 2).astype(np.int64)
        out = np.empty(6)
        lib.oracle_gemm_asym_f64_at(ptr(X64), ptr(codes), ptr(s16), ptr(z16), 256, r, 6, ptr(ms), ptr(ns), ptr(out))
        ref = _exact_asym(X, codes, s, z, r)[ms, ns]
        caught |= not np.allclose(out, ref, rtol=1e-12, atol=0)
    assert caught, name
