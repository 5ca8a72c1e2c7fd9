"""GPU parity of the asymmetric variant (per-group zero point z, fp16, level
2^(8-r) q_r + 2^(7-r) - z) against the fp64 oracle (oracle.gemm_asym).
Asymmetric weights run on the tcgen05 GEMM for every M (the zero-point term
s (128 - z) sum_g x is folded in fp32 from per-group sums of X)."""
import numpy as np
import pytest

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


def _asym_parent(N, K, seed):
    import torch
    import nested_bit_weight_b200 as mq
    codes, s, z, _ = wl.gen_weights_asym(N, K, seed)
    p = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(),
                       zeros=torch.from_numpy(z).cuda())
    return codes, s, z, p


@pytest.mark.parametrize("r", [8, 4, 2, 1])
@pytest.mark.parametrize("M", [1, 3, 8, 16, 33, 64, 130])
@pytest.mark.parametrize("N,K", [(37, 384), (300, 1408), (130, 2048), (1024, 4096)])
def test_asym_ragged(N, K, M, r):
    import torch
    import nested_bit_weight_b200 as mq
    codes, s, z, p = _asym_parent(N, K, seed=N + K)
    xbits, X = wl.gen_x(M, K, seed=N + M)
    Xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
    Y = mq.gemm(Xd, p, r).float().cpu().numpy().astype(np.float64)
    assert oracle.violation_ratio(Y, oracle.gemm_asym(X, codes, s, z, r)) <= 1.0


def test_asym_stored_zero_points_bit_exact():
    import torch
    import nested_bit_weight_b200 as mq
    codes, s, z, p = _asym_parent(300, 384, seed=5)
    got = p.zeros16.cpu().numpy()
    assert np.array_equal(got.view(np.uint16), oracle.zeros_stored(z).view(np.uint16))


@pytest.mark.parametrize("M", [9, 64])
def test_zero_point_128_reproduces_the_symmetric_gemm(M):
    # z = 128 everywhere: the zero-point term vanishes and the asymmetric
    # call returns exactly the symmetric GEMM's bits
    import torch
    import nested_bit_weight_b200 as mq
    N, K = 1024, 2048
    codes, s, _ = wl.gen_weights(N, K, seed=3)
    cd, sd = torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda()
    sym = mq.pack_parent(cd, sd)
    asym = mq.pack_parent(cd, sd, zeros=torch.full_like(sd, 128.0))
    xbits, _ = wl.gen_x(M, K, seed=4)
    Xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
    for r in (8, 3):
        a = mq.gemm(Xd, sym, r).view(torch.int16)
        b = mq.gemm(Xd, asym, r).view(torch.int16)
        assert torch.equal(a, b)


@pytest.mark.parametrize("M,r", [(1, 4), (16, 3), (128, 4)])
def test_asym_llama_gate(M, r):
    import torch
    import nested_bit_weight_b200 as mq
    N, K = 14336, 4096
    codes, s, z, p = _asym_parent(N, K, seed=41)
    xbits, X = wl.gen_x(M, K, seed=42 + M, outlier_channels=True)
    Xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
    Y = mq.gemm(Xd, p, r).float().cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(M)
    ns = np.concatenate([t * 128 + rng.integers(128, size=2) for t in range(N // 128)])
    ms = rng.integers(M, size=ns.shape[0])
    ref = oracle.gemm_asym_at(X, codes, s, z, r, ms, ns)
    rms = float(np.sqrt(np.mean(ref * ref)))
    assert oracle.violation_ratio(Y[ms, ns], ref, rms) <= 1.0
    mq.mq_device_status()
