"""The bounded-wait timeout path, run on a GPU without a fault or a trap.

A test-hook build of the library (libmq_testhooks.so: every bounded wait
gives up after 5 ms, and mq_test_drop_x_arrivals() makes one GEMM CTA drop
one arrival of its X operand) is loaded next to nothing else of the package.
One call then times out inside the kernel: the waiting thread gives up,
the CTA's other roles stop, its tensor memory is freed and the launch ends;
mq_device_status() reports MQ_ERR_TIMEOUT once and clears the flag.  The
next call on the same workspace (its tickets returned to zero) matches the
oracle, so the context and the library stay usable."""
import ctypes
import os

import numpy as np
import pytest

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MQ_ERR_TIMEOUT = 5


class _W(ctypes.Structure):
    _fields_ = [("planes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("group", ctypes.c_int32), ("r", ctypes.c_int32),
                ("zeros", ctypes.c_void_p)]


def _hooks_lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_mq_build", os.path.join(ROOT, "nested_bit_weight_b200", "_build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    path = b.build_test_hooks()            # no-op when up to date
    L = ctypes.CDLL(path)
    P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    L.mq_plane_bytes.restype = SZ
    L.mq_plane_bytes.argtypes = [I64, I64, I]
    L.mq_scale_bytes.restype = SZ
    L.mq_scale_bytes.argtypes = [I64, I64, I]
    L.mq_gemm_workspace_bytes.restype = SZ
    L.mq_gemm_workspace_bytes.argtypes = [I64, I64, I64, I]
    L.mq_pack.restype = I
    L.mq_pack.argtypes = [P, P, I64, I64, I, P, P, P]
    L.mq_gemm.restype = I
    L.mq_gemm.argtypes = [P, ctypes.POINTER(_W), I64, I64, I64, P, P, SZ, P]
    L.mq_device_status.restype = I
    L.mq_test_drop_x_arrivals.restype = I
    L.mq_test_drop_x_arrivals.argtypes = [I]
    return L


def test_bounded_wait_times_out_and_the_next_call_is_exact():
    import torch
    L = _hooks_lib()
    N, K, M, r = 1024, 1024, 16, 4
    codes, s, _ = wl.gen_weights(N, K, seed=91)
    xbits, X = wl.gen_x(M, K, seed=91)
    cd, sd = torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda()
    planes = torch.empty(L.mq_plane_bytes(N, K, 8) // 4, dtype=torch.int32, device="cuda")
    scales = torch.empty(L.mq_scale_bytes(N, K, 128) // 2, dtype=torch.float16, device="cuda")
    assert L.mq_pack(cd.data_ptr(), sd.data_ptr(), N, K, 128, planes.data_ptr(),
                     scales.data_ptr(), None) == 0
    w = _W(planes.data_ptr(), scales.data_ptr(), N, K, 128, r)
    Xd = torch.from_numpy(xbits.view(np.int16)).cuda()
    Y = torch.empty((M, N), dtype=torch.int16, device="cuda")
    ws = torch.zeros(max(L.mq_gemm_workspace_bytes(M, N, K, r), 256), dtype=torch.uint8, device="cuda")
    assert L.mq_device_status() == 0

    # one CTA loses an arrival: its MMA thread gives up after 5 ms
    assert L.mq_test_drop_x_arrivals(1) == 0
    assert L.mq_gemm(Xd.data_ptr(), ctypes.byref(w), M, N, K, Y.data_ptr(), ws.data_ptr(),
                     ws.numel(), None) == 0
    assert L.mq_device_status() == MQ_ERR_TIMEOUT
    assert L.mq_device_status() == 0                      # reported once, then cleared
    assert int(ws[:64 * 1024].view(torch.int32).abs().sum()) == 0   # tickets back to zero

    # the next calls run normally and match the oracle
    ref = oracle.gemm(X, codes, s, r)
    for _ in range(2):
        Y.fill_(0)
        assert L.mq_gemm(Xd.data_ptr(), ctypes.byref(w), M, N, K, Y.data_ptr(), ws.data_ptr(),
                         ws.numel(), None) == 0
        assert L.mq_device_status() == 0
        got = Y.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)
        assert oracle.violation_ratio(got, ref) <= 1.0
