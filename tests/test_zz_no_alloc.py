"""mq_gemv_noalloc: the workspace-free M <= 8 entry point, for callers that
cannot allocate device memory (plugins whose host owns all device memory,
servers that reserve the GPU for their own pool, loops that cannot take
cudaMalloc's device synchronisation).  Its output must match mq_gemm's on the
same inputs within the parity tolerance, on two calls in a row.  Collected
last on purpose, so a run that stops at the first failure has already run
every other test."""
import ctypes

import numpy as np
import pytest

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


def _noalloc():
    import nested_bit_weight_b200 as mq
    f = mq.lib.mq_gemv_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.POINTER(mq.MqWeights), ctypes.c_int64,
                  ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    return f


def _layer(N, K, M, seed):
    import torch
    import nested_bit_weight_b200 as mq
    codes, s, _ = wl.gen_weights(N, K, seed=seed)
    xbits, X = wl.gen_x(M, K, seed=seed)
    parent = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
    Xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
    return codes, s, X, parent, Xd


def _check_twice(N, K, M, r, seed):
    """mq_gemv_noalloc twice in a row against mq_gemm and the oracle."""
    import torch
    import nested_bit_weight_b200 as mq
    codes, s, X, parent, Xd = _layer(N, K, M, seed)
    ref = mq.gemm(Xd, parent, r).float().cpu().numpy().astype(np.float64)
    fn = _noalloc()
    w = parent.view(r)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = fn(Xd.data_ptr(), ctypes.byref(w), M, N, K, Y.data_ptr(), stream)
        assert st == 0, mq.lib.mq_last_error_string().decode()
        got = Y.float().cpu().numpy().astype(np.float64)
        assert oracle.violation_ratio(got, ref) <= 1.0
        assert oracle.violation_ratio(got, oracle.gemm(X, codes, s, r)) <= 1.0


@pytest.mark.parametrize("M,r", [(1, 3), (3, 2), (8, 4)])
def test_noalloc_matches_mq_gemm_twice(M, r):
    # by default M = 1 and 3 take the tensor-core GEMV (no scratch) and M = 8
    # the GEMM, which uses the built-in scratch
    _check_twice(1024, 4096, M, r, seed=31 + M)


def test_noalloc_scratch_through_the_gemm():
    # the GEMM route keeps its split-K partial sums, X operand and arrival
    # tickets in the built-in array: two shapes in a row, each twice, so the
    # second shape reuses tickets and partials the first one left
    import nested_bit_weight_b200 as mq
    old = mq.mq_get_gemv_variant()
    mq.mq_set_gemv_variant(mq.GEMV_VIA_GEMM)
    try:
        for (N, K, M, r) in ((1024, 4096, 3, 2), (300, 14336, 8, 5)):
            assert mq.mq_gemm_workspace_bytes(M, N, K, r) > 64 * 1024   # tickets + partials
            _check_twice(N, K, M, r, seed=N + M)
    finally:
        mq.mq_set_gemv_variant(old)


def test_noalloc_rejects_oversized_and_large_m():
    import torch
    import nested_bit_weight_b200 as mq
    fn = _noalloc()
    N, K = 16, 256
    codes, s, _ = wl.gen_weights(N, K, seed=1)
    parent = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
    w = parent.view(4)
    X = torch.zeros((9, K), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((9, N), dtype=torch.bfloat16, device="cuda")
    assert fn(X.data_ptr(), ctypes.byref(w), 9, N, K, Y.data_ptr(), None) == 1
    # a scratch need above 16 MiB is refused before any launch: on the GEMM
    # route (M = 1, N = 2^17, K = 4096) the partial sums of the row tiles
    # shared between CTAs alone exceed it
    old = mq.mq_get_gemv_variant()
    mq.mq_set_gemv_variant(mq.GEMV_VIA_GEMM)
    try:
        big = mq.MqWeights(w.planes, w.scales, 1 << 17, 4096, 128, 2)
        assert mq.mq_gemm_workspace_bytes(1, 1 << 17, 4096, 2) > (16 << 20)
        assert fn(X.data_ptr(), ctypes.byref(big), 1, 1 << 17, 4096, Y.data_ptr(), None) == 6
    finally:
        mq.mq_set_gemv_variant(old)
