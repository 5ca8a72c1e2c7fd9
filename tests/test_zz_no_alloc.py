"""mq_gemv_noalloc: the workspace-free M <= 8 entry point, for callers that
cannot allocate device memory (plugins whose host owns all device memory,
servers that reserve the GPU for their own pool, loops that cannot take
cudaMalloc's device synchronisation).  Its output must match mq_gemm's on the
same inputs within the parity tolerance, on two calls in a row (the second
call reuses the library's built-in scratch).  Collected last on purpose, so a
run that stops at the first failure has already run every other test."""
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


@pytest.mark.parametrize("M,r", [(1, 3), (3, 2), (8, 4)])
def test_noalloc_matches_mq_gemm_twice(M, r):
    import torch
    import nested_bit_weight_b200 as mq
    N, K = 1024, 4096                      # split K: the scratch holds partials and tickets
    assert mq.mq_gemm_workspace_bytes(M, N, K, r) > 64 * 1024
    codes, s, _ = wl.gen_weights(N, K, seed=31 + M)
    xbits, X = wl.gen_x(M, K, seed=31 + M)
    parent = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
    Xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
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
    # a workspace need above 16 MiB is refused before any launch
    # (M = 1, N = 128, K = 2^20: the GEMM fallback's operand copy of X alone is 32 MiB)
    big = mq.MqWeights(w.planes, w.scales, 128, 1 << 20, 128, 2)
    assert mq.mq_gemm_workspace_bytes(1, 128, 1 << 20, 2) > (16 << 20)
    assert fn(X.data_ptr(), ctypes.byref(big), 1, 128, 1 << 20, Y.data_ptr(), None) == 6
