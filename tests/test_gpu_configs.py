"""GPU parity on the full benchmark workloads: the Llama-3.1-8B batch sweep,
the Qwen3-8B mixed-r chain with outlier activation channels, and the
70B-class sweep, each against the fp64 CPU oracle.

Outputs small enough for the whole-matrix oracle are compared element by
element.  For the large ones (every point with M * N * K above
`FULL_LIMIT`), the oracle is evaluated at sampled positions that cover
every 128-row tile of W, every 32-row block of X and random places besides;
every output sums over all of K, so every split of K is covered too.  The
rms in the tolerance is then estimated from the sampled reference values.
Pass criterion: |Y - Y_ref| <= 8e-3 |Y_ref| + 1e-3 rms(Y_ref) per element.
"""
import numpy as np
import pytest

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

FULL_LIMIT = 2 * 10 ** 9          # M * N * K above this: sampled positions


_parents = {}


def _parent(config, layer_index, N, K):
    """Codes, scales and the packed parent of one workload layer (cached)."""
    import torch
    import nested_bit_weight_b200 as mq
    key = (config, layer_index, N, K)
    if key not in _parents:
        if len(_parents) >= 4:
            _parents.clear()
            torch.cuda.empty_cache()
        codes, s, _ = wl.gen_weights(N, K, wl.layer_seed(config, layer_index))
        p = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
        _parents[key] = (codes, s, p)
    return _parents[key]


def _positions(M, N, rng, per_tile=2, per_block=16, extra=768):
    ms, ns = [], []
    for t in range((N + 127) // 128):
        for _ in range(per_tile):
            ns.append(min(N - 1, t * 128 + int(rng.integers(128))))
            ms.append(int(rng.integers(M)))
    for b in range((M + 31) // 32):
        for _ in range(per_block):
            ms.append(min(M - 1, b * 32 + int(rng.integers(32))))
            ns.append(int(rng.integers(N)))
    ms += [int(v) for v in rng.integers(M, size=extra)]
    ns += [int(v) for v in rng.integers(N, size=extra)]
    return np.array(ms, np.int64), np.array(ns, np.int64)


def _check(config, layer_index, N, K, M, r, outliers=False):
    import torch
    import nested_bit_weight_b200 as mq
    codes, s, parent = _parent(config, layer_index, N, K)
    xbits, X = wl.gen_x(M, K, wl.layer_seed(config, layer_index) + M, outlier_channels=outliers)
    Xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
    Y = mq.gemm(Xd, parent, r).float().cpu().numpy().astype(np.float64)
    assert np.isfinite(Y).all()
    if M * N * K <= FULL_LIMIT:
        return oracle.violation_ratio(Y, oracle.gemm(X, codes, s, r))
    rng = np.random.default_rng(N + K + M + r)
    ms, ns = _positions(M, N, rng)
    ref = oracle.gemm_at(X, codes, s, r, ms, ns)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return oracle.violation_ratio(Y[ms, ns], ref, rms)


LLAMA = [(i, l.name, l.N, l.K) for i, l in enumerate(wl.LLAMA8B)]
LLAMA_SHAPES = [x for x in LLAMA if x[1] in ("q_proj", "k_proj", "gate_proj", "down_proj")]


@pytest.mark.parametrize("r", [8, 4, 3, 2])
@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 32, 64])
@pytest.mark.parametrize("li,name,N,K", LLAMA_SHAPES)
def test_llama8b_batch_sweep(li, name, N, K, M, r):
    # the batch sweep over the Llama-3.1-8B shapes (GEMV up to M = 8, the
    # tensor-core GEMM from M = 16)
    assert _check(2, li, N, K, M, r) <= 1.0


@pytest.mark.parametrize("M", [16, 32, 64])
@pytest.mark.parametrize("li,name,N,K", [x for x in LLAMA if x not in LLAMA_SHAPES])
def test_llama8b_other_layers_r8(li, name, N, K, M):
    # the remaining layers (own weights) at r = 8 on the GEMM path
    assert _check(2, li, N, K, M, 8) <= 1.0


QWEN = [(i, l.name, l.N, l.K) for i, l in enumerate(wl.QWEN3_8B)]


@pytest.mark.parametrize("M", [16, 64, 128])
@pytest.mark.parametrize("li,name,N,K", QWEN)
def test_qwen3_chain_mixed_r(li, name, N, K, M):
    # attention projections at r = 4, FFN at r = 3, X with x20 outlier channels
    assert _check(3, li, N, K, M, wl.QWEN3_R[name], outliers=True) <= 1.0


L70 = [(i, l.name, l.N, l.K) for i, l in enumerate(wl.LLAMA70B)
       if l.name in ("q_proj", "k_proj", "gate_proj", "down_proj")]


@pytest.mark.parametrize("r", [8, 6, 4, 3, 2])
@pytest.mark.parametrize("M", [1, 8, 32, 128, 256])
@pytest.mark.parametrize("li,name,N,K", L70)
def test_70b_sweep(li, name, N, K, M, r):
    assert _check(4, li, N, K, M, r) <= 1.0


def test_gemv_wide_range_x():
    # x spanning far more than 2^20 inside one 128-column group: the GEMV's
    # int8 slices keep x to 2^-20 of the group's largest, and what they drop
    # stays far inside the tolerance (values down to 1e-7 next to 1e2)
    import torch
    import nested_bit_weight_b200 as mq
    N, K = 1024, 1024
    codes, s, _ = wl.gen_weights(N, K, seed=77)
    parent = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
    rng = np.random.default_rng(5)
    for M in (1, 3, 8):
        x = rng.standard_normal((M, K)).astype(np.float32)
        mag = 10.0 ** rng.uniform(-7, -3, size=(M, K)).astype(np.float32)
        x = np.where(rng.random((M, K)) < 0.5, x * mag, x).astype(np.float32)
        x[:, ::128] = 1e2                                    # the largest of every group
        x[:, 5::128] = -3e-7
        Xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
        X = Xd.float().cpu().numpy()
        for r in (8, 4, 2):
            Y = mq.gemm(Xd, parent, r).float().cpu().numpy()
            assert oracle.violation_ratio(Y, oracle.gemm(X, codes, s, r)) <= 1.0, (M, r)


def test_dispatch_table_on_gpu():
    # the small-batch dispatch on the Llama-3.1-8B shapes: GEMV up to M = 3
    # everywhere, M = 4 on q/o and k/v, M = 5..6 on k/v only
    import nested_bit_weight_b200 as mq
    G, E = mq.KERNEL_GEMV, mq.KERNEL_GEMM
    table = {(4096, 4096): [G, G, G, G, E, E, E, E],
             (1024, 4096): [G, G, G, G, G, G, E, E],
             (14336, 4096): [G, G, G, E, E, E, E, E],
             (4096, 14336): [G, G, G, E, E, E, E, E]}
    for (N, K), want in table.items():
        for r in (4, 2):
            assert [mq.mq_gemm_kernel(M, N, K, r) for M in range(1, 9)] == want, (N, K, r)


@pytest.mark.parametrize("r", [4, 2])
@pytest.mark.parametrize("M", [3, 4, 5, 6, 7])
@pytest.mark.parametrize("li,name,N,K", LLAMA_SHAPES)
def test_dispatch_boundaries(li, name, N, K, M, r):
    # both sides of every GEMV / GEMM boundary of the small-batch dispatch
    # (gate/down 3|4, q 4|5, k 6|7), each kernel on its side
    assert _check(2, li, N, K, M, r) <= 1.0
