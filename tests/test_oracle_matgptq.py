"""Pins of the oracle's one-shot multi-precision quantizer (the GPTQ column
loop with the lambda-weighted multi-r objective and cross-bit error feedback;
readings in the oracle's module).  Each pin checks the oracle against
something other than its own formula: a closed-form rounding, a structural
property of the nested code, a hand-worked two-column propagation, and the
loss properties the method exists for; planted mistakes must fail them."""
import inspect
import types

import numpy as np
import pytest

import oracle


def _rtn8_closed_form(w, s):
    # nearest level q - 127.5 to w / s, ties to the smaller code, clamped
    t = w / s + 127.5
    return np.clip(np.ceil(t - 0.5), 0, 255).astype(np.uint8)


def _H(K, seed, corr=0.9):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((4 * K, K))
    X = z.copy()
    for k in range(1, K):                       # AR(1) columns: correlated inputs
        X[:, k] = corr * X[:, k - 1] + np.sqrt(1 - corr * corr) * z[:, k]
    return X.T @ X / X.shape[0]


def test_r8_without_feedback_is_round_to_nearest(q=oracle):
    rng = np.random.default_rng(1)
    W = rng.standard_normal((3, 256)) * 0.02
    codes, scales = q.matgptq_quantize(W, np.eye(256), rs=(8,), lams=(1.0,), alphas=(1.0,))
    for g in range(2):
        s = np.max(np.abs(W[:, 128 * g:128 * g + 128]), axis=1) / 127.5
        assert np.allclose(scales[:, g], s, rtol=0, atol=0)
        want = _rtn8_closed_form(W[:, 128 * g:128 * g + 128], s[:, None])
        assert np.array_equal(codes[:, 128 * g:128 * g + 128], want)


def test_r3_only_uses_the_top_three_bits(q=oracle):
    rng = np.random.default_rng(2)
    W = rng.standard_normal((2, 128)) * 0.02
    codes, _ = q.matgptq_quantize(W, np.eye(128), rs=(3,), lams=(1.0,), alphas=(1.0,))
    assert np.all(codes & 31 == 0)              # the free low bits take the smallest code
    assert len(np.unique(codes >> 5)) > 4


def test_two_column_feedback_worked_example(q=oracle):
    # U with U[0,0] = 2, U[0,1] = 1 (other off-diagonals 0), r = 8 only:
    # column 1 is quantised after w1 -= (w0 - s v(q0)) / 2
    K = 128
    U = np.eye(K)
    U[0, 0], U[0, 1] = 2.0, 1.0
    W = np.zeros((1, K))
    W[0, 0], W[0, 1], W[0, 2] = 0.0173, -0.0041, 0.02
    codes, scales = q.matgptq_quantize(W, U, rs=(8,), lams=(1.0,), alphas=(1.0,))
    s = 0.02 / 127.5
    assert scales[0, 0] == s
    q0 = int(_rtn8_closed_form(np.array(0.0173), s))
    e0 = 0.0173 - s * (q0 - 127.5)
    w1 = -0.0041 - e0 / 2.0 * 1.0
    assert codes[0, 0] == q0
    assert codes[0, 1] == int(_rtn8_closed_form(np.array(w1), s))
    assert codes[0, 1] != int(_rtn8_closed_form(np.array(-0.0041), s)) or abs(e0) < s / 4


def _proxy_loss(W, codes, scales, H, r):
    Wq = oracle.level(codes >> (8 - r), r) * np.repeat(scales, 128, axis=1)
    D = W - Wq
    return float(np.einsum("nk,kl,nl->", D, H, D))


def test_feedback_beats_round_to_nearest_on_correlated_inputs(q=oracle):
    K = 256
    H = _H(K, seed=3)
    rng = np.random.default_rng(4)
    W = rng.standard_normal((4, K)) * 0.02
    U = q.matgptq_prepare(H)
    c_fb, s_fb = q.matgptq_quantize(W, U, rs=(8,), lams=(1.0,), alphas=(1.0,))
    c_rtn, s_rtn = q.matgptq_quantize(W, np.eye(K), rs=(8,), lams=(1.0,), alphas=(1.0,))
    assert _proxy_loss(W, c_fb, s_fb, H, 8) < 0.8 * _proxy_loss(W, c_rtn, s_rtn, H, 8)


def test_lambda3_lowers_the_3bit_slice_error(q=oracle):
    K = 256
    H = _H(K, seed=5)
    rng = np.random.default_rng(6)
    W = rng.standard_normal((4, K)) * 0.02
    U = q.matgptq_prepare(H)
    c8, s8 = q.matgptq_quantize(W, U, rs=(3, 4, 8), lams=(0.0, 0.0, 1.0), alphas=(1.0,))
    cm, sm = q.matgptq_quantize(W, U, rs=(3, 4, 8), lams=(1.0, 1.0, 1.0), alphas=(1.0,))
    assert _proxy_loss(W, cm, sm, H, 3) < _proxy_loss(W, c8, s8, H, 3)


def test_lambda8_lowers_the_8bit_slice_error(q=oracle):
    # the other end of the same trade-off: weighting the 8-bit slice up moves
    # the shared feedback towards the parent's own errors
    K = 256
    H = _H(K, seed=8)
    rng = np.random.default_rng(9)
    W = rng.standard_normal((4, K)) * 0.02
    U = q.matgptq_prepare(H)
    c1, s1 = q.matgptq_quantize(W, U, rs=(3, 4, 8), lams=(1.0, 1.0, 1.0), alphas=(1.0,))
    c16, s16 = q.matgptq_quantize(W, U, rs=(3, 4, 8), lams=(1.0, 1.0, 16.0), alphas=(1.0,))
    assert _proxy_loss(W, c16, s16, H, 8) < 0.5 * _proxy_loss(W, c1, s1, H, 8)


def test_prepare_factor(q=oracle):
    H = _H(128, seed=7)
    U = q.matgptq_prepare(H, damp=0.01)
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(128)
    assert np.allclose(np.triu(U), U)
    assert np.allclose(U.T @ U @ Hd, np.eye(128), atol=1e-9)


MUTATIONS = {
    "feedback_sign": ("W[n, k + 1:] -= (e / U[k, k]) * U[k, k + 1:]", "W[n, k + 1:] += (e / U[k, k]) * U[k, k + 1:]"),
    "feedback_no_pivot": ("W[n, k + 1:] -= (e / U[k, k]) * U[k, k + 1:]", "W[n, k + 1:] -= e * U[k, k + 1:]"),
    "scale_127": ("/ 127.5\n            best_a", "/ 127.0\n            best_a"),
    "code_argmax": ("return int(np.argmin(cost))", "return int(np.argmax(-cost[::-1]))"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_fail_a_pin(name):
    old, new = MUTATIONS[name]
    src = inspect.getsource(oracle)
    assert old in src, name
    mod = types.ModuleType("oracle_mutant")
    mod.__dict__["__file__"] = oracle.__file__
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    pins = [test_r8_without_feedback_is_round_to_nearest, test_r3_only_uses_the_top_three_bits,
            test_two_column_feedback_worked_example, test_feedback_beats_round_to_nearest_on_correlated_inputs,
            test_lambda3_lowers_the_3bit_slice_error, test_lambda8_lowers_the_8bit_slice_error]
    failed = 0
    for pin in pins:
        try:
            pin(q=mod)
        except AssertionError:
            failed += 1
    assert failed >= 1, name
