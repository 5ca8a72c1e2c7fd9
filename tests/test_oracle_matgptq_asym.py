"""Pins of the oracle's one-shot quantizer with asymmetric levels (per-group
zero point z; readings in the oracle's module): a closed-form rounding at
r = 8, equality with the symmetric quantizer on centred groups (z = 128),
the gain on one-signed groups the variant exists for, and the feedback's
gain; planted mistakes must fail them."""
import inspect
import types

import numpy as np
import pytest

import oracle


def _H(K, seed, corr=0.9):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((4 * K, K))
    X = z.copy()
    for k in range(1, K):
        X[:, k] = corr * X[:, k - 1] + np.sqrt(1 - corr * corr) * z[:, k]
    return X.T @ X / X.shape[0]


def _sq_err(W, codes, s, z, r):
    u = oracle.level_asym(codes >> (8 - r), r, np.repeat(z, 128, axis=1))
    return float(np.sum((W - np.repeat(s, 128, axis=1) * u) ** 2))


def test_r8_without_feedback_is_round_to_nearest(q=oracle):
    rng = np.random.default_rng(1)
    W = rng.standard_normal((3, 256)) * 0.02 + 0.007
    codes, scales, zeros = q.matgptq_quantize_asym(W, np.eye(256), rs=(8,), lams=(1.0,), alphas=(1.0,))
    for n in range(3):
        for g in range(2):
            seg = W[n, 128 * g:128 * g + 128]
            lo, hi = seg.min(), seg.max()
            s = (hi - lo) / 255.0
            z = float(np.float16(np.float32(128.0 - (hi + lo) / (2.0 * s))))
            assert scales[n, g] == s and zeros[n, g] == z
            # level q + 0.5 - z nearest to w / s, ties to the smaller code
            want = np.clip(np.ceil(seg / s + z - 0.5 - 0.5), 0, 255).astype(np.uint8)
            assert np.array_equal(codes[n, 128 * g:128 * g + 128], want)


def test_centred_groups_equal_the_symmetric_quantizer(q=oracle):
    rng = np.random.default_rng(2)
    W = rng.standard_normal((4, 256)) * 0.02
    for n in range(4):
        for g in range(2):
            m = np.abs(W[n, 128 * g:128 * g + 128]).max() + 1e-3
            W[n, 128 * g], W[n, 128 * g + 1] = m, -m          # hi = -lo: z = 128
    for rs, lams in (((8,), (1.0,)), ((3, 4, 8), (1.0, 1.0, 1.0))):
        ca, sa, za = q.matgptq_quantize_asym(W, np.eye(256), rs=rs, lams=lams, alphas=(1.0, 0.9))
        cs, ss = q.matgptq_quantize(W, np.eye(256), rs=rs, lams=lams, alphas=(1.0, 0.9))
        assert np.all(za == 128.0)
        assert np.array_equal(ca, cs) and np.allclose(sa, ss, rtol=1e-15, atol=0)


def test_one_signed_groups_gain_from_the_zero_point(q=oracle):
    rng = np.random.default_rng(3)
    W = np.abs(rng.standard_normal((4, 256))) * 0.02 + 0.01
    for r in (3, 4):
        ca, sa, za = q.matgptq_quantize_asym(W, np.eye(256), rs=(r,), lams=(1.0,), alphas=(1.0,))
        cs, ss = q.matgptq_quantize(W, np.eye(256), rs=(r,), lams=(1.0,), alphas=(1.0,))
        assert _sq_err(W, ca, sa, za, r) < 0.5 * _sq_err(W, cs, ss, np.full_like(ss, 128.0), r)


def test_feedback_beats_round_to_nearest_on_correlated_inputs(q=oracle):
    K = 256
    H = _H(K, seed=4)
    rng = np.random.default_rng(5)
    W = rng.standard_normal((4, K)) * 0.02 + 0.005
    U = q.matgptq_prepare(H)

    def loss(c, s, z):
        D = W - np.repeat(s, 128, axis=1) * oracle.level_asym(c, 8, np.repeat(z, 128, axis=1))
        return float(np.einsum("nk,kl,nl->", D, H, D))
    fb = q.matgptq_quantize_asym(W, U, rs=(8,), lams=(1.0,), alphas=(1.0,))
    rtn = q.matgptq_quantize_asym(W, np.eye(K), rs=(8,), lams=(1.0,), alphas=(1.0,))
    assert loss(*fb) < 0.8 * loss(*rtn)


def test_constant_group_takes_the_symmetric_grid(q=oracle):
    W = np.full((1, 128), 0.0123)
    c, s, z = q.matgptq_quantize_asym(W, np.eye(128), rs=(8,), lams=(1.0,), alphas=(1.0,))
    assert s[0, 0] == 0.0123 / 127.5 and z[0, 0] == 128.0 and np.all(c == 255)


MUTATIONS = {
    "z_sign": ("z = float(zeros_f16(np.array(128.0 - (hi + lo) / (2.0 * s))))",
               "z = float(zeros_f16(np.array(128.0 + (hi + lo) / (2.0 * s))))"),
    "z_unrounded": ("z = float(zeros_f16(np.array(128.0 - (hi + lo) / (2.0 * s))))",
                    "z = float(128.0 - (hi + lo) / (2.0 * s))"),
    "range_256": ("s = alpha * (hi - lo) / 255.0", "s = alpha * (hi - lo) / 256.0"),
    "feedback_sign": ("                W[n, k + 1:] -= (e / U[k, k]) * U[k, k + 1:]\n    return codes, scales, zeros",
                      "                W[n, k + 1:] += (e / U[k, k]) * U[k, k + 1:]\n    return codes, scales, zeros"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_fail_a_pin(name):
    old, new = MUTATIONS[name]
    src = inspect.getsource(oracle)
    assert src.count(old) == 1, name
    mod = types.ModuleType("oracle_mutant")
    mod.__dict__["__file__"] = oracle.__file__
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    pins = [test_r8_without_feedback_is_round_to_nearest, test_centred_groups_equal_the_symmetric_quantizer,
            test_one_signed_groups_gain_from_the_zero_point,
            test_feedback_beats_round_to_nearest_on_correlated_inputs,
            test_constant_group_takes_the_symmetric_grid]
    failed = 0
    for pin in pins:
        try:
            pin(q=mod)
        except AssertionError:
            failed += 1
    assert failed >= 1, name
