"""GPU parity of mq_gemm against the fp64 CPU oracle.

Pass criterion (per element): |Y - Y_ref| <= 8e-3 |Y_ref| + 1e-3 rms(Y_ref),
rms over the whole output (oracle.violation_ratio <= 1).
"""
import numpy as np
import pytest

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


def _run(codes, s, xbits, r, parent=None):
    import torch
    import nested_bit_weight_b200 as mq
    if parent is None:
        parent = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
    X = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
    Y = mq.gemm(X, parent, r)
    torch.cuda.synchronize()
    return Y.float().cpu().numpy().astype(np.float64), parent


def _case(N, K, M, r, seed, outliers=False):
    codes, s, _ = wl.gen_weights(N, K, seed)
    xbits, X = wl.gen_x(M, K, seed, outlier_channels=outliers)
    Y, _ = _run(codes, s, xbits, r)
    Yref = oracle.gemm(X, codes, s, r)
    return oracle.violation_ratio(Y, Yref)


@pytest.mark.parametrize("r", [8, 7, 6, 5, 4, 3, 2, 1])
def test_single_layer_512(r):
    # the 512 x 512 single-layer workload at M = 1, seed 0
    assert _case(512, 512, 1, r, wl.layer_seed(0, 0)) <= 1.0


def test_golden_samples_config0():
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "config0_samples.json")))
    codes, s, _ = wl.gen_weights(512, 512, wl.layer_seed(0, 0))
    xbits, X = wl.gen_x(1, 512, wl.layer_seed(0, 0))
    parent = None
    for r, vals in g["Y"].items():
        Y, parent = _run(codes, s, xbits, int(r), parent)
        ref = np.array([float.fromhex(v) for v in vals])
        Yref_full = oracle.gemm(X, codes, s, int(r))[0]
        rms = float(np.sqrt(np.mean(Yref_full ** 2)))
        assert oracle.violation_ratio(Y[0, g["columns"]], ref, rms) <= 1.0


@pytest.fixture(params=["tc", "via_gemm"])
def gemv_variant(request):
    import nested_bit_weight_b200 as mq
    old = mq.mq_get_gemv_variant()
    mq.mq_set_gemv_variant(mq.GEMV_TC if request.param == "tc" else mq.GEMV_VIA_GEMM)
    yield request.param
    mq.mq_set_gemv_variant(old)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("r", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("N,K", [(37, 384), (300, 1408), (1, 128), (130, 2048)])
def test_gemv_ragged(N, K, M, r, gemv_variant):
    assert _case(N, K, M, r, seed=N * 7 + K + M) <= 1.0


@pytest.mark.parametrize("r", [1, 2, 3, 4, 5, 6, 7, 8])
def test_gemv_one_hot_columns(r, gemv_variant):
    # X = e_k picks column k of W_r: every column position of a group, exactly
    # up to the bf16 rounding of the output
    import torch
    import nested_bit_weight_b200 as mq
    N, K = 48, 256
    codes = wl.adversarial_codes("random", N, K, seed=r)
    s = wl.gen_scales(N, K, seed=r)
    parent = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
    W = oracle.dequant(codes, s, r)
    M = 8
    for k0 in range(0, K, M):
        X = np.zeros((M, K), np.float32)
        for m in range(M):
            X[m, k0 + m] = 1.0
        Xd = torch.from_numpy(X).cuda().to(torch.bfloat16)
        Y = mq.gemm(Xd, parent, r).float().cpu().numpy()
        want = W[:, k0:k0 + M].T
        assert np.allclose(Y, want, rtol=2 ** -8, atol=0), (r, k0)


@pytest.mark.parametrize("M", [9, 12, 15, 16, 33, 64])
@pytest.mark.parametrize("r", [2, 4, 8])
def test_batched_ragged(M, r):
    assert _case(200, 640, M, r, seed=M + r) <= 1.0


@pytest.mark.parametrize("kind", ["zeros", "ones", "alternating", "single_bit"])
@pytest.mark.parametrize("r", [1, 2, 3, 4, 8])
def test_adversarial_codes(kind, r):
    N, K, M = 64, 512, 3
    codes = wl.adversarial_codes(kind, N, K)
    s = wl.gen_scales(N, K, seed=5, zero_groups=17)
    xbits, X = wl.gen_x(M, K, seed=5)
    Y, _ = _run(codes, s, xbits, r)
    Yref = oracle.gemm(X, codes, s, r)
    assert oracle.violation_ratio(Y, Yref) <= 1.0


def test_all_zero_scales_give_zero():
    N, K = 16, 256
    codes = wl.adversarial_codes("random", N, K)
    s = np.zeros((N, K // 128), np.float32)
    xbits, _ = wl.gen_x(2, K, seed=1)
    Y, _ = _run(codes, s, xbits, 4)
    assert np.all(Y == 0.0)


def test_deterministic_and_workspace_reusable():
    # split-K shape: the arrival tickets must be back at zero after each call,
    # otherwise a later call would skip the final reduction (NaN survives)
    import torch
    import nested_bit_weight_b200 as mq
    N, K = 1024, 14336
    assert mq.mq_gemm_workspace_bytes(1, N, K, 3) > 0
    codes, s, _ = wl.gen_weights(N, K, seed=9)
    xbits, X = wl.gen_x(1, K, seed=9)
    parent = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
    Xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
    outs = []
    for _ in range(3):
        Y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        mq.gemm(Xd, parent, 3, Y=Y)
        outs.append(Y.float().cpu().numpy())
    assert not np.isnan(outs[0]).any()
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])
    assert oracle.violation_ratio(outs[0], oracle.gemm(X, codes, s, 3)) <= 1.0


@pytest.mark.parametrize("N,K,M,r", [(2048, 14336, 1, 4), (2048, 14336, 8, 8), (2048, 14336, 8, 2),
                                      (1024, 14336, 4, 3), (2000, 8192, 8, 6), (300, 28672, 3, 5)])
def test_gemv_stage_ring_and_k_segments(N, K, M, r):
    # more items per CTA than shared-memory stages (the ring wraps), and long
    # K (row tiles whose groups are split between CTAs: the GEMV sums them in
    # a cluster through distributed shared memory, the GEMM through the
    # workspace, both in a fixed order); twice, bit-identical (some of these
    # shapes and batches take the GEMM under the small-batch dispatch)
    import torch
    import nested_bit_weight_b200 as mq
    codes, s, _ = wl.gen_weights(N, K, seed=N + K + M + r)
    xbits, X = wl.gen_x(M, K, seed=N + K + M + r)
    parent = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
    Xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
    Y1 = mq.gemm(Xd, parent, r).float().cpu().numpy()
    Y2 = mq.gemm(Xd, parent, r).float().cpu().numpy()
    assert np.array_equal(Y1, Y2)
    assert oracle.violation_ratio(Y1.astype(np.float64), oracle.gemm(X, codes, s, r)) <= 1.0


LLAMA = [(l.name, l.N, l.K) for l in wl.LLAMA8B]


@pytest.mark.parametrize("r", [4, 3, 2])
@pytest.mark.parametrize("name,N,K", LLAMA)
def test_llama_layers_full_m1(name, N, K, r, gemv_variant):
    # full-size decode layers at M = 1: every output against the oracle
    seed = wl.layer_seed(1, [l[0] for l in LLAMA].index(name))
    assert _case(N, K, 1, r, seed) <= 1.0


@pytest.mark.parametrize("r", [4, 2])
@pytest.mark.parametrize("M", [2, 4, 8])
@pytest.mark.parametrize("name,N,K", [l for l in LLAMA if l[0] in ("gate_proj", "down_proj", "k_proj")])
def test_llama_layers_full_small_batch(name, N, K, M, r):
    # full-size layers at M = 2..8 (GEMV batch classes 2, 4 and 8; clusters
    # and whole-tile splits): every output against the oracle
    seed = wl.layer_seed(2, [l[0] for l in LLAMA].index(name))
    assert _case(N, K, M, r, seed) <= 1.0


def test_workspace_shared_across_shapes():
    # a larger split-K call followed by a smaller one on the same workspace
    import torch
    import nested_bit_weight_b200 as mq
    N, K = 37, 384
    codes, s, _ = wl.gen_weights(N, K, seed=77)
    parent = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
    need = max(mq.mq_gemm_workspace_bytes(M, N, K, r) for M in (1, 8) for r in (2, 3))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for M, r in ((8, 2), (1, 3), (8, 3), (1, 2)):
        xbits, X = wl.gen_x(M, K, seed=M)
        Xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        mq.mq_gemm(Xd, parent.view(r), Y, ws)
        Yh = Y.float().cpu().numpy()
        assert oracle.violation_ratio(Yh, oracle.gemm(X, codes, s, r)) <= 1.0


def test_no_device_wait_timed_out():
    # every launch above and these ones completed without a bounded wait giving up
    import torch
    import nested_bit_weight_b200 as mq
    for (N, K, M, r) in ((4096, 4096, 1, 4), (1024, 4096, 2, 2), (640, 1280, 5, 3), (512, 512, 32, 8)):
        codes, s, _ = wl.gen_weights(N, K, seed=N + M)
        xb, _ = wl.gen_x(M, K, seed=K + M)
        p = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
        X = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
        mq.gemm(X, p, r)
    mq.mq_device_status()


@pytest.mark.parametrize("name,N,K", [("gate_proj", 28672, 8192), ("down_proj", 8192, 28672)])
def test_70b_layers_full(name, N, K):
    # 70B-class shapes at M = 1, 8, 32 and r = 4, 2 (GEMV with clusters or
    # whole tiles, the GEMM fallback where the X operand does not fit, and
    # the GEMM): every output against the oracle
    codes, s, _ = wl.gen_weights(N, K, wl.layer_seed(4, 4 if name == "gate_proj" else 6))
    parent = None
    for M in (1, 8, 32):
        xbits, X = wl.gen_x(M, K, wl.layer_seed(4, 0) + M)
        for r in (4, 2):
            Y, parent = _run(codes, s, xbits, r, parent)
            ratio = oracle.violation_ratio(Y, oracle.gemm(X, codes, s, r))
            assert ratio <= 1.0, (M, r, ratio)


@pytest.mark.parametrize("name,N,K,M", [("gate_proj", 12288, 4096, 64), ("q_proj", 4096, 4096, 128),
                                        ("down_proj", 4096, 12288, 16)])
def test_qwen_chain_outlier_x(name, N, K, M):
    # Qwen3-8B chain: attention at r = 4, FFN at r = 3, X with x20 outlier channels
    r = wl.QWEN3_R[name]
    codes, s, _ = wl.gen_weights(N, K, wl.layer_seed(3, 0))
    xbits, X = wl.gen_x(M, K, wl.layer_seed(3, 0) + M, outlier_channels=True)
    Y, _ = _run(codes, s, xbits, r)
    assert oracle.violation_ratio(Y, oracle.gemm(X, codes, s, r)) <= 1.0


@pytest.mark.parametrize("M", [1, 3, 16])
def test_weights_written_by_the_previous_kernel(M):
    # stream order (programmatic dependent launch): a torch kernel writes the
    # weights and mq_gemm follows at once on the same stream, no sync; torch's
    # kernels do not let dependents start early, so the early weight reads of
    # the GEMV and the GEMM see the new weights (the contract in mq.h)
    import torch
    import nested_bit_weight_b200 as mq
    N, K = 2048, 4096
    ca, sa, _ = wl.gen_weights(N, K, seed=501)
    cb, sb, _ = wl.gen_weights(N, K, seed=502)
    A = mq.pack_parent(torch.from_numpy(ca).cuda(), torch.from_numpy(sa).cuda())
    B = mq.pack_parent(torch.from_numpy(cb).cuda(), torch.from_numpy(sb).cuda())
    xbits, X = wl.gen_x(M, K, seed=503)
    Xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
    ref_a, ref_b = oracle.gemm(X, ca, sa, 4), oracle.gemm(X, cb, sb, 4)
    planes_a, scales_a = A.planes.clone(), A.scales16.clone()
    outs = []
    for src_p, src_s in ((B.planes, B.scales16), (planes_a, scales_a), (B.planes, B.scales16)):
        A.planes.copy_(src_p)
        A.scales16.copy_(src_s)
        outs.append(mq.gemm(Xd, A, 4))            # no synchronisation in between
    got = [o.float().cpu().numpy().astype(np.float64) for o in outs]
    assert oracle.violation_ratio(got[0], ref_b) <= 1.0
    assert oracle.violation_ratio(got[1], ref_a) <= 1.0
    assert oracle.violation_ratio(got[2], ref_b) <= 1.0
