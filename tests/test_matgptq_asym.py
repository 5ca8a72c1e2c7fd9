"""The library's one-shot quantizer with asymmetric levels against the
oracle: given the same U, codes, scales and zero points must be identical
(fp64 decisions in the same order; z rounded to fp32 then fp16 on both
sides)."""
import numpy as np
import pytest

import oracle
import nested_bit_weight_b200 as mq


def _H(K, seed, corr=0.9):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((4 * K, K))
    X = z.copy()
    for k in range(1, K):
        X[:, k] = corr * X[:, k - 1] + np.sqrt(1 - corr * corr) * z[:, k]
    return X.T @ X / X.shape[0]


def _W(N, K, seed):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((N, K)) * 0.02
    W += rng.standard_normal((N, K // 128)).repeat(128, axis=1) * 0.01    # off-centre groups
    W[0] = np.abs(W[0]) + 0.003                                          # a one-signed row
    return W.astype(np.float32)


def _check(W, U, **kw):
    c_ref, s_ref, z_ref = oracle.matgptq_quantize_asym(W.astype(np.float64), U, **kw)
    lam = kw.pop("lams", (1.0, 1.0, 1.0))
    codes, scales, zeros = mq.matgptq_quantize(W, U, lambdas=lam, asymmetric=True, **kw)
    assert np.array_equal(codes, c_ref)
    assert np.array_equal(scales, s_ref.astype(np.float32))
    assert np.array_equal(zeros, z_ref.astype(np.float32))
    return codes, scales, zeros


@pytest.mark.parametrize("rs,lams,alphas", [
    ((3, 4, 8), (1.0, 1.0, 1.0), (1.0, 0.95, 0.9, 0.85, 0.8)),
    ((2, 4, 6, 8), (4.0, 2.0, 1.0, 1.0), (1.0, 0.9)),
    ((8,), (1.0,), (1.0,)),
    ((1, 3), (1.0, 0.5), (1.0, 0.7)),
])
def test_codes_scales_zeros_identical_to_the_oracle(rs, lams, alphas):
    K = 256
    _check(_W(5, K, 12), oracle.matgptq_prepare(_H(K, 11)), rs=rs, lams=lams, alphas=alphas)


def test_degenerate_groups_match_the_oracle():
    # a zero group, a constant group, a centred group (z = 128) and a group
    # with a tiny range far from zero (z beyond fp16: the symmetric grid)
    K = 512
    W = _W(3, K, 21)
    W[1, :128] = 0.0
    W[1, 128:256] = 0.0123
    m = np.abs(W[2, 256:384]).max() + 1e-3
    W[2, 256], W[2, 257] = m, -m
    W[2, 384:] = np.float32(1.0) + np.arange(128, dtype=np.float32) * np.float32(1e-7)
    for U in (np.eye(K), oracle.matgptq_prepare(_H(K, 22))):
        codes, scales, zeros = _check(W, U, alphas=(1.0, 0.9))
    codes, scales, zeros = _check(W, np.eye(K), rs=(8,), lams=(1.0,), alphas=(1.0,))
    assert scales[1, 0] == 0 and zeros[1, 0] == 128 and np.all(codes[1, :128] == 0)
    assert zeros[1, 1] == 128 and zeros[2, 2] == 128 and zeros[2, 3] == 128


def test_many_groups_and_a_ragged_row_block_match_the_oracle():
    N, K = 17, 640
    _check(_W(N, K, 31), oracle.matgptq_prepare(_H(K, 32)), alphas=(1.0, 0.85))


def test_asymmetric_codes_serve_the_asymmetric_gemm_oracle():
    # the quantizer's outputs are the asymmetric format's inputs: their r-bit
    # models approximate W better than the symmetric quantizer's on
    # off-centre groups (squared error through the oracle's dequantization)
    K = 256
    W = _W(8, K, 41)
    U = oracle.matgptq_prepare(_H(K, 42))
    ca, sa, za = mq.matgptq_quantize(W, U, asymmetric=True)
    cs, ss = mq.matgptq_quantize(W, U)
    W64 = W.astype(np.float64)
    for r in (3, 4):
        ea = np.sum((W64 - oracle.dequant_asym(ca, sa, za, r)) ** 2)
        es = np.sum((W64 - oracle.dequant(cs, ss, r)) ** 2)
        assert ea < es, r


def test_zeros_out_is_required():
    W = _W(2, 128, 51)
    rs, lam, al, U = np.array([8], np.int32), np.array([1.0]), np.array([1.0]), np.eye(128)
    codes = np.empty((2, 128), np.uint8)
    scales = np.empty((2, 1), np.float32)
    status = mq.lib.mq_matgptq_quantize_asym(W.ctypes.data, 2, 128, U.ctypes.data, rs.ctypes.data,
                                             lam.ctypes.data, 1, al.ctypes.data, 1, 0,
                                             codes.ctypes.data, scales.ctypes.data, None)
    assert status == 1                                   # MQ_ERR_INVALID_ARG
