"""The library's one-shot multi-precision quantizer (host) against the
oracle: given the same U, the codes and the scales must be identical (both
sides take every decision in fp64 in the same order), the prepare step must
agree with the oracle's within rounding, and bad arguments must be refused."""
import numpy as np
import pytest

import oracle
import workloads as wl
import nested_bit_weight_b200 as mq


def _H(K, seed, corr=0.9):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((4 * K, K))
    X = z.copy()
    for k in range(1, K):                       # AR(1) columns: correlated inputs
        X[:, k] = corr * X[:, k - 1] + np.sqrt(1 - corr * corr) * z[:, k]
    return X.T @ X / X.shape[0]


def _W(N, K, seed):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((N, K)) * 0.02
    W[:, rng.integers(K, size=3)] *= 8.0        # a few outlier columns
    return W.astype(np.float32)


@pytest.mark.parametrize("rs,lams,alphas", [
    ((3, 4, 8), (1.0, 1.0, 1.0), (1.0, 0.95, 0.9, 0.85, 0.8)),
    ((2, 4, 6, 8), (4.0, 2.0, 1.0, 1.0), (1.0, 0.9, 0.8)),
    ((8,), (1.0,), (1.0,)),
    ((1, 3), (1.0, 0.5), (1.0, 0.7)),
])
def test_codes_and_scales_identical_to_the_oracle(rs, lams, alphas):
    N, K = 5, 256
    U = oracle.matgptq_prepare(_H(K, 11))
    W = _W(N, K, 12)
    c_ref, s_ref = oracle.matgptq_quantize(W.astype(np.float64), U, rs=rs, lams=lams, alphas=alphas)
    codes, scales = mq.matgptq_quantize(W, U, rs=rs, lambdas=lams, alphas=alphas)
    assert codes.shape == (N, K) and scales.shape == (N, K // 128)
    assert np.array_equal(codes, c_ref)
    assert np.array_equal(scales, s_ref.astype(np.float32))


def test_thread_count_does_not_change_the_result():
    N, K = 9, 384
    U = oracle.matgptq_prepare(_H(K, 21))
    W = _W(N, K, 22)
    a = mq.matgptq_quantize(W, U, threads=1)
    for t in (2, 4, 0, 64):
        b = mq.matgptq_quantize(W, U, threads=t)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("K", [1, 7, 128, 300, 700])
def test_prepare_agrees_with_the_oracle(K):
    H = _H(K, 31 + K)
    U = mq.matgptq_prepare(H, damp=0.01)
    ref = oracle.matgptq_prepare(H, damp=0.01)
    assert np.array_equal(U, np.triu(U))
    assert np.allclose(U, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max())
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(K)
    assert np.allclose(U.T @ U @ Hd, np.eye(K), atol=1e-8)


def test_prepare_then_quantize_is_the_oracle_pipeline():
    N, K = 4, 256
    H = _H(K, 41)
    W = _W(N, K, 42)
    codes, scales = mq.matgptq_quantize(W, mq.matgptq_prepare(H))
    c_ref, s_ref = oracle.matgptq_quantize(W.astype(np.float64), oracle.matgptq_prepare(H))
    # U agrees to ~1e-13 relative, so a code may differ only where two codes
    # tie to within that; none do on this input
    assert np.array_equal(codes, c_ref)
    assert np.allclose(scales, s_ref, rtol=1e-6)


def test_argument_errors():
    K = 128
    U = np.eye(K)
    W = _W(2, K, 51)
    bad = [
        dict(W=_W(2, 100, 1), U=np.eye(100)),               # K not a multiple of 128
        dict(rs=(3, 9), lambdas=(1.0, 1.0)),                 # width above 8
        dict(rs=(0,), lambdas=(1.0,)),                       # width below 1
        dict(rs=(3, 4), lambdas=(0.0, 0.0)),                 # all lambdas zero
        dict(rs=(3, 4), lambdas=(1.0, -1.0)),                # a negative lambda
        dict(alphas=(1.0, 0.0)),                             # a zero alpha
        dict(alphas=()),                                     # no alpha
        dict(U=np.diag(np.r_[np.ones(K - 1), 0.0])),         # zero on U's diagonal
    ]
    for kw in bad:
        args = dict(W=W, U=U)
        args.update(kw)
        with pytest.raises(mq.MQError):
            mq.matgptq_quantize(**args)
    with pytest.raises(ValueError):
        mq.matgptq_quantize(W, np.eye(64))
    with pytest.raises(ValueError):
        mq.matgptq_quantize(W, U, rs=(3, 4), lambdas=(1.0,))
    with pytest.raises(mq.MQError):
        mq.matgptq_prepare(-np.eye(8))                       # not positive definite
    with pytest.raises(mq.MQError):
        mq.matgptq_prepare(np.eye(8), damp=-1.0)
    with pytest.raises(ValueError):
        mq.matgptq_prepare(np.eye(8)[:4])


def test_degenerate_rows_and_exact_ties_match_the_oracle():
    # row 0: all zero (s = 0, every code ties: code 0); row 1: its first group
    # zero; row 2: values exactly halfway between two 8-bit levels with
    # s = 2^-7 exactly (ties to the smaller code); row 3: one nonzero weight
    K = 256
    W = np.zeros((4, K), np.float32)
    W[1, 128:] = np.linspace(-0.03, 0.05, 128, dtype=np.float32)
    q = np.arange(128) % 255
    W[2, :128] = ((q - 127.0) / 128.0).astype(np.float32)     # (q - 127) * 2^-7
    W[2, 0] = np.float32(127.5 / 128.0)                       # max |w| = 127.5 * 2^-7
    W[2, 128:] = W[2, :128]
    W[3, 200] = 0.01
    U = oracle.matgptq_prepare(_H(K, 61))
    for U_ in (np.eye(K), U):
        for rs, lams in (((8,), (1.0,)), ((3, 4, 8), (1.0, 1.0, 1.0))):
            c_ref, s_ref = oracle.matgptq_quantize(W.astype(np.float64), U_, rs=rs, lams=lams, alphas=(1.0,))
            codes, scales = mq.matgptq_quantize(W, U_, rs=rs, lambdas=lams, alphas=(1.0,))
            assert np.array_equal(codes, c_ref), rs
            assert np.array_equal(scales, s_ref.astype(np.float32)), rs
    codes, scales = mq.matgptq_quantize(W, np.eye(K), rs=(8,), lambdas=(1.0,), alphas=(1.0,))
    assert np.all(codes[0] == 0) and np.all(scales[0] == 0)
    assert np.all(codes[1, :128] == 0) and scales[1, 0] == 0 and scales[1, 1] > 0
    assert scales[2, 0] == 2.0 ** -7
    # w / s = q - 127 lies halfway between the levels q - 127.5 and q - 126.5
    # of codes q and q + 1: the smaller code wins
    assert codes[2, 0] == 255
    assert np.array_equal(codes[2, 1:128], q[1:].astype(np.uint8))


def test_single_row_single_group():
    W = _W(1, 128, 71)
    U = oracle.matgptq_prepare(_H(128, 72))
    c_ref, s_ref = oracle.matgptq_quantize(W.astype(np.float64), U)
    codes, scales = mq.matgptq_quantize(W, U)
    assert np.array_equal(codes, c_ref) and np.array_equal(scales, s_ref.astype(np.float32))


def _stress_cases():
    rng = np.random.default_rng(81)
    widths = [(1,), (2,), (1, 2), (1, 3), (2, 4), (3, 4, 8), (2, 3, 6), (1, 8), (4, 4), (5, 7, 8)]
    for i, rs in enumerate(widths):
        lams = tuple(float(x) for x in rng.choice([0.0, 0.25, 1.0, 3.0], size=len(rs)))
        if sum(lams) == 0.0:
            lams = (1.0,) + lams[1:]
        yield pytest.param(rs, lams, i, id=f"r{'-'.join(map(str, rs))}")


@pytest.mark.parametrize("rs,lams,seed", list(_stress_cases()))
def test_code_search_matches_the_oracle_on_coarse_and_mixed_widths(rs, lams, seed):
    # half the weights sit on the 2^-7 grid with s = 2^-7 (exact ties between
    # levels and between whole blocks of codes), half are random
    K = 256
    rng = np.random.default_rng(90 + seed)
    W = (rng.standard_normal((4, K)) * 0.02).astype(np.float32)
    W[:2] = (rng.integers(-127, 128, size=(2, K)) / 128.0).astype(np.float32)
    W[:2, 0] = W[:2, 128] = np.float32(127.5 / 128.0)
    U = np.eye(K) if seed % 2 else oracle.matgptq_prepare(_H(K, 91 + seed))
    c_ref, s_ref = oracle.matgptq_quantize(W.astype(np.float64), U, rs=rs, lams=lams, alphas=(1.0, 0.9))
    codes, scales = mq.matgptq_quantize(W, U, rs=rs, lambdas=lams, alphas=(1.0, 0.9))
    assert np.array_equal(codes, c_ref)
    assert np.array_equal(scales, s_ref.astype(np.float32))


def test_non_finite_weights_are_refused():
    W = _W(2, 128, 95)
    for bad in (np.nan, np.inf, -np.inf):
        W2 = W.copy()
        W2[1, 17] = bad
        with pytest.raises(mq.MQError):
            mq.matgptq_quantize(W2, np.eye(128))


@pytest.mark.parametrize("env", ["MQ_PORTABLE_HOST", "MQ_NO_AVX512"])
def test_other_host_code_paths_agree_with_the_oracle(env):
    # the portable host loops (MQ_PORTABLE_HOST=1) and the AVX2 ones
    # (MQ_NO_AVX512=1; the default takes AVX-512 for the prepare step's tile
    # product where the CPU has it), each in a fresh process: prepare within
    # rounding, quantize bit for bit
    import os
    import subprocess
    import sys
    code = (
        "import numpy as np, sys; sys.path[:0] = %r\n"
        "import oracle, nested_bit_weight_b200 as mq\n"
        "rng = np.random.default_rng(5)\n"
        "for K in (3, 130, 257, 521):\n"
        "    X = rng.standard_normal((2 * K, K)); H = X.T @ X / (2 * K)\n"
        "    U = mq.matgptq_prepare(H); ref = oracle.matgptq_prepare(H)\n"
        "    assert np.allclose(U, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max()), K\n"
        "W = (rng.standard_normal((3, 256)) * 0.02).astype(np.float32)\n"
        "U = oracle.matgptq_prepare(W.T.astype(np.float64) @ W + np.eye(256))\n"
        "c, s = mq.matgptq_quantize(W, U); cr, sr = oracle.matgptq_quantize(W.astype(np.float64), U)\n"
        "assert np.array_equal(c, cr) and np.array_equal(s, sr.astype(np.float32))\n"
        "print('ok')\n" % (sys.path,))
    out = subprocess.run([sys.executable, "-c", code], env=dict(os.environ, **{env: "1"}),
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stderr


def test_many_groups_and_a_ragged_row_block_match_the_oracle():
    # five groups (each group's feedback reaches the later groups after it)
    # and 17 rows (a full block of 16 plus one)
    N, K = 17, 640
    U = oracle.matgptq_prepare(_H(K, 101))
    W = _W(N, K, 102)
    c_ref, s_ref = oracle.matgptq_quantize(W.astype(np.float64), U, alphas=(1.0, 0.85))
    codes, scales = mq.matgptq_quantize(W, U, alphas=(1.0, 0.85))
    assert np.array_equal(codes, c_ref)
    assert np.array_equal(scales, s_ref.astype(np.float32))


def test_sixteen_groups_match_the_oracle():
    # K = 2048: every group's feedback reaches fifteen later groups through
    # the grouped update, and the window search runs over 16 scale choices
    N, K = 3, 2048
    H = wl.gen_hessian(K, 111, samples=K + 256)
    U = oracle.matgptq_prepare(H)
    W = wl.gen_float_weights(N, K, 112)
    c_ref, s_ref = oracle.matgptq_quantize(W.astype(np.float64), U, alphas=(1.0, 0.9))
    codes, scales = mq.matgptq_quantize(W, U, alphas=(1.0, 0.9))
    assert np.array_equal(codes, c_ref)
    assert np.array_equal(scales, s_ref.astype(np.float32))
