"""Pins for the CPU oracle: it is checked against what the definitions and
the mathematics fix, never against itself or the CUDA path.

Sources: MatGPTQ pages (abstract: fewer bits are read from one parent, an
r-bit model reads exactly r bits; author-page abstract: MSB slicing) and the
dequantization w = s_g * (2^(8-r) q_r + 2^(7-r) - 128) with the
per-element tolerance 8e-3 |Y_ref| + 1e-3 rms(Y_ref).
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as wl

KINDS = ("zeros", "ones", "alternating", "single_bit", "all_codes", "random")


def _packbits_planes(codes):
    """Plane words via numpy's packbits and reshapes (an independent route to
    the layout): bit j of row-word w of plane p is bit (7 - p) of code
    k = 32 w + j; rows are padded with zeros to a multiple of 128 and the
    128 x 128 blocks (row tile t, group g) are laid out t-major, each block
    row-major with 4 words per row."""
    N, K = codes.shape
    Np, G = (N + 127) // 128 * 128, K // 128
    rows = np.zeros((8, Np, K // 32), np.uint32)
    for p in range(8):
        bits = ((codes >> (7 - p)) & 1).astype(np.uint8)
        by = np.packbits(bits, axis=1, bitorder="little")          # N x K/8
        rows[p, :N] = by.reshape(N, K // 32, 4).copy().view("<u4")[..., 0]
    # [p][t][i][g][w] -> [p][t][g][i][w]
    tiled = rows.reshape(8, Np // 128, 128, G, 4).transpose(0, 1, 3, 2, 4)
    return np.ascontiguousarray(tiled).reshape(8, -1)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("N,K", [(24, 256), (130, 384), (256, 128)])
def test_pack_matches_packbits(kind, N, K):
    codes = wl.adversarial_codes(kind, N, K, seed=3)
    assert np.array_equal(oracle.pack(codes), _packbits_planes(codes))


@pytest.mark.parametrize("kind", KINDS)
def test_pack_unpack_identity_and_prefix(kind):
    codes = wl.adversarial_codes(kind, 16, 384, seed=5)
    planes = oracle.pack(codes)
    assert np.array_equal(oracle.unpack(planes, 8, 16, 384), codes)
    for r in range(1, 9):
        # an r-bit model is exactly the first r planes: pass only that prefix
        prefix = np.ascontiguousarray(planes[:r])
        want = (codes >> (8 - r)).astype(np.uint8)
        assert np.array_equal(oracle.unpack(prefix, r, 16, 384), want)


def test_pack_single_code_positions():
    # brute force: one set code at each position lands in exactly one bit, at
    # the word the layout definition gives (written out here independently)
    N, K = 200, 384
    G = K // 128
    for n in (0, 1, 127, 128, 199):
        for k in (0, 5, 31, 32, 127, 128, 300, 383):
            for b in (0, 3, 7):
                codes = np.zeros((N, K), np.uint8)
                codes[n, k] = 1 << b
                planes = oracle.pack(codes)
                word = ((n // 128) * G + k // 128) * 512 + (n % 128) * 4 + (k % 128) // 32
                nz = np.argwhere(planes)
                assert nz.tolist() == [[7 - b, word]]
                assert planes[7 - b, word] == np.uint32(1 << (k % 32))


def test_scales_stored_layout():
    # the stored scales follow the planes' block order: (t, g) block of 128 rows
    N, K = 130, 384
    s = wl.gen_scales(N, K, seed=3)
    st = oracle.scales_stored(s)
    s16 = oracle.scales_f16(s)
    assert st.shape == (256 * 3,)
    for n in (0, 77, 127, 128, 129):
        for g in range(3):
            assert st[((n // 128) * 3 + g) * 128 + n % 128] == s16[n, g]
    assert np.all(st[(1 * 3 + 0) * 128 + 2:(1 * 3 + 1) * 128] == 0)   # padding rows


def test_slicing_is_nested():
    q = np.arange(256, dtype=np.uint8)
    for r in range(1, 9):
        for r2 in range(1, r + 1):
            assert np.array_equal(oracle.slice_codes(oracle.slice_codes(q, r) << (8 - r), r2),
                                  oracle.slice_codes(q, r2))
            assert np.array_equal(oracle.slice_codes(q, r) >> (r - r2),
                                  oracle.slice_codes(q, r2))


def test_r8_is_parent_dequantization():
    q = np.arange(256, dtype=np.uint8)
    assert np.array_equal(oracle.level(oracle.slice_codes(q, 8), 8), q - 127.5)


def test_level_closed_forms():
    for r in range(1, 9):
        qr = np.arange(2 ** r)
        v = oracle.level(qr, r)
        # symmetric grid: v(q) = -v(2^r - 1 - q); extremes +-(128 - 2^(7-r))
        assert np.array_equal(v, -v[::-1])
        assert v[-1] == 128 - 2.0 ** (7 - r) and v[0] == -v[-1]
        # uniform spacing 2^(8-r)
        assert np.all(np.diff(v) == 2.0 ** (8 - r))


def test_nesting_error_bound():
    q = np.arange(256, dtype=np.uint8)
    v8 = oracle.level(q, 8)
    for r in range(1, 9):
        vr = oracle.level(oracle.slice_codes(q, r), r)
        err = np.abs(v8 - vr)
        assert err.max() == 2.0 ** (7 - r) - 0.5


def test_hand_worked_r2_levels():
    # codes 0, 64, 128, 255 -> top-2 bits 0, 1, 2, 3 -> 64 q + 32 - 128
    q = np.array([0, 64, 128, 255], np.uint8)
    assert oracle.slice_codes(q, 2).tolist() == [0, 1, 2, 3]
    assert oracle.level(oracle.slice_codes(q, 2), 2).tolist() == [-96, -32, 32, 96]


def _exact_gemm(X, codes, s, r):
    """Exact rational Y: bf16 X, fp16 s and half-integer levels are dyadic."""
    s16 = oracle.scales_f16(s)
    M, K = X.shape
    N = codes.shape[0]
    Y = [[Fraction(0)] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                q_r = int(codes[n, k]) >> (8 - r)
                v = Fraction(2 ** (8 - r)) * q_r + Fraction(2) ** (7 - r) - 128
                acc += Fraction(float(X[m, k])) * Fraction(float(s16[n, k // 128])) * v
            Y[m][n] = acc
    return Y


@pytest.mark.parametrize("r", [8, 6, 4, 3, 2, 1])
def test_gemm_exact_rational_bruteforce(r):
    N, K, M = 5, 256, 3
    codes, s, _ = wl.gen_weights(N, K, seed=11 + r)
    _, X = wl.gen_x(M, K, seed=11 + r)
    Y = oracle.gemm(X, codes, s, r)
    Ye = _exact_gemm(X, codes, s, r)
    for m in range(M):
        for n in range(N):
            ex = float(Ye[m][n])
            assert abs(Y[m, n] - ex) <= 1e-12 * max(abs(ex), 1e-30) + 1e-300


@pytest.mark.parametrize("r", [8, 4, 2])
def test_gemm_one_hot_gives_dequantized_column(r):
    N, K = 7, 384
    codes, s, _ = wl.gen_weights(N, K, seed=21)
    W = oracle.dequant(codes, s, r)
    for k in (0, 1, 127, 128, 255, 383):
        X = np.zeros((1, K))
        X[0, k] = 1.0
        assert np.array_equal(oracle.gemm(X, codes, s, r)[0], W[:, k])


@pytest.mark.parametrize("r", [8, 5, 3, 1])
def test_gemm_ones_over_one_group_closed_form(r):
    N, K = 6, 256
    codes = wl.adversarial_codes("random", N, K, seed=31)
    s = wl.gen_scales(N, K, seed=31)
    X = np.zeros((1, K))
    X[0, 128:256] = 1.0          # group 1 only
    s16 = oracle.scales_f16(s).astype(np.float64)
    qr = (codes[:, 128:256] >> (8 - r)).astype(np.int64)
    want = s16[:, 1] * (2.0 ** (8 - r) * qr.sum(axis=1)
                        + 128 * (2.0 ** (7 - r) - 128))
    assert np.allclose(oracle.gemm(X, codes, s, r)[0], want, rtol=1e-15, atol=0)


def test_gemm_at_matches_full():
    codes, s, _ = wl.gen_weights(40, 512, seed=41)
    _, X = wl.gen_x(3, 512, seed=41)
    Y = oracle.gemm(X, codes, s, 3)
    ms = np.array([0, 2, 1, 2]); ns = np.array([0, 39, 17, 5])
    assert np.array_equal(oracle.gemm_at(X, codes, s, 3, ms, ns), Y[ms, ns])


def test_zero_scale_group_gives_zero_weights():
    codes, s, _ = wl.gen_weights(4, 256, seed=3)
    s = s.copy(); s[2, 1] = 0.0
    W = oracle.dequant(codes, s, 4)
    assert np.all(W[2, 128:256] == 0.0)


def test_scales_fp16_round_to_nearest_even():
    # values exactly halfway between fp16 neighbours round to the even one
    lo = np.float16(1.0); hi = np.nextafter(lo, np.float16(2))
    mid = (np.float32(lo) + np.float32(hi)) / 2
    assert oracle.scales_f16(np.array([mid]))[0] == lo
    assert oracle.scales_f16(np.array([70000.0]))[0] == np.inf


def test_tolerance_definition():
    Yref = np.array([1.0, -2.0, 0.0, 0.5])
    rms = np.sqrt(np.mean(Yref ** 2))
    tol = oracle.tolerance(Yref)
    assert np.allclose(tol, 8e-3 * np.abs(Yref) + 1e-3 * rms)
    assert oracle.violation_ratio(Yref + 0.5 * tol, Yref) == pytest.approx(0.5)
    assert oracle.violation_ratio(Yref + 2.0 * tol, Yref) == pytest.approx(2.0)


def test_generator_recipe():
    codes, s, W = wl.gen_weights(64, 512, seed=0)
    Wg = W.reshape(64, 4, 128)
    assert np.array_equal(s, (np.abs(Wg).max(axis=2) / np.float32(127.5)).astype(np.float32))
    assert int(np.sum(np.abs(W) > 0.2)) > 0          # outliers present
    # the max-magnitude element of each group sits at the ends of the code range:
    # +127.5 -> 255 after the clamp, -127.5 -> 0 (half to even), or 1 after
    # fp32 rounding of W / s
    amax = np.abs(Wg).argmax(axis=2)
    c = codes.reshape(64, 4, 128)
    picked = np.take_along_axis(c, amax[..., None], axis=2)[..., 0]
    assert set(np.unique(picked)).issubset({0, 1, 255})


def test_golden_config0_samples_stable():
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "config0_samples.json")))
    codes, s, _ = wl.gen_weights(512, 512, wl.layer_seed(0, 0))
    _, X = wl.gen_x(1, 512, wl.layer_seed(0, 0))
    for r, vals in g["Y"].items():
        Y = oracle.gemm(X, codes, s, int(r))[0]
        assert [float.hex(float(Y[c])) for c in g["columns"]] == vals
