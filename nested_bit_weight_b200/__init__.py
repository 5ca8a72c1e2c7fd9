"""Python binding of libmq (nested r-bit weight GEMM on B200).

Argument marshalling only: every computation runs in libmq's CUDA kernels.
The function names follow the C ABI in include/mq.h (mq_pack, mq_slice,
mq_gemm, mq_unpack, ...).  PyTorch supplies device memory and streams.

If libmq.so has not been built, importing this package raises; there is no
CPU or PyTorch fallback for any step.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "MQError", "MqWeights", "NestedWeights", "lib", "library_path",
    "mq_plane_bytes", "mq_scale_bytes", "mq_pack", "mq_slice", "mq_gemm",
    "mq_gemm_workspace_bytes", "mq_unpack", "mq_version", "pack_parent", "gemm",
    "mq_set_gemv_variant", "mq_get_gemv_variant", "GEMV_TC", "GEMV_VIA_GEMM",
    "mq_device_status", "mq_gemm_kernel", "uses_gemv", "KERNEL_GEMV", "KERNEL_GEMM",
    "MqCall", "mq_gemm_chain", "gemm_chain", "pack_fused", "workspace_for", "mq_pack_zeros",
    "MqChoice", "bitwidth_search", "layer_errors", "matgptq_prepare", "matgptq_quantize",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libmq.so")

MQ_OK = 0
STATUS = {0: "MQ_OK", 1: "MQ_ERR_INVALID_ARG", 2: "MQ_ERR_UNSUPPORTED",
          3: "MQ_ERR_MISALIGNED", 4: "MQ_ERR_CUDA", 5: "MQ_ERR_TIMEOUT",
          6: "MQ_ERR_WORKSPACE"}


class MQError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class MqWeights(ctypes.Structure):
    """Mirror of the C struct mq_weights (a view, owns nothing)."""
    _fields_ = [("planes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("group", ctypes.c_int32), ("r", ctypes.c_int32),
                ("zeros", ctypes.c_void_p)]                # fp16 zero points or None (symmetric)


class MqChoice(ctypes.Structure):
    """One candidate of mq_bitwidth_search (mq_choice in include/mq.h)."""
    _fields_ = [("r", ctypes.c_int32), ("bytes", ctypes.c_uint64), ("error", ctypes.c_double)]


class MqCall(ctypes.Structure):
    """One product of mq_gemm_chain (mq_call in include/mq.h)."""
    _fields_ = [("X", ctypes.c_void_p), ("w", ctypes.POINTER(MqWeights)),
                ("M", ctypes.c_int64), ("Y", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(library_path):
        raise ImportError(
            f"{library_path} is missing: build it with "
            "`python nested_bit_weight_b200/_build.py` (nvcc, sm_100a)")
    L = ctypes.CDLL(library_path)
    P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    W = ctypes.POINTER(MqWeights)
    sig = {
        "mq_plane_bytes": (SZ, [I64, I64, I]),
        "mq_scale_bytes": (SZ, [I64, I64, I]),
        "mq_pack": (I, [P, P, I64, I64, I, P, P, P]),
        "mq_slice": (I, [W, I, W]),
        "mq_gemm_workspace_bytes": (SZ, [I64, I64, I64, I]),
        "mq_gemm": (I, [P, W, I64, I64, I64, P, P, SZ, P]),
        "mq_unpack": (I, [W, P, P]),
        "mq_last_error": (I, []),
        "mq_device_status": (I, []),
        "mq_last_error_string": (ctypes.c_char_p, []),
        "mq_status_string": (ctypes.c_char_p, [I]),
        "mq_version": (ctypes.c_char_p, []),
        "mq_set_gemv_variant": (I, [I]),
        "mq_get_gemv_variant": (I, []),
        "mq_gemm_kernel": (I, [I64, I64, I64, I]),
        "mq_gemm_chain": (I, [ctypes.POINTER(MqCall), I, P, SZ, P]),
        "mq_pack_zeros": (I, [P, I64, I64, I, P, P]),
        "mq_bitwidth_search": (I, [ctypes.POINTER(MqChoice), I, I, ctypes.c_uint64,
                                   ctypes.POINTER(I), ctypes.POINTER(ctypes.c_double)]),
        "mq_matgptq_prepare": (I, [P, I64, ctypes.c_double, P]),
        "mq_matgptq_quantize": (I, [P, I64, I64, P, P, P, I, P, I, I, P, P]),
        "mq_matgptq_quantize_asym": (I, [P, I64, I64, P, P, P, I, P, I, I, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    return L


lib = _load()


def _check(status: int) -> None:
    if status != MQ_OK:
        raise MQError(status, lib.mq_last_error_string().decode())


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


# ------------------------------------------------------------------ raw C ABI

def mq_plane_bytes(N: int, K: int, r: int) -> int:
    return lib.mq_plane_bytes(N, K, r)


def mq_scale_bytes(N: int, K: int, group: int = 128) -> int:
    return lib.mq_scale_bytes(N, K, group)


def mq_gemm_workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    return lib.mq_gemm_workspace_bytes(M, N, K, r)


GEMV_TC, GEMV_VIA_GEMM = 0, 1


def mq_set_gemv_variant(variant: int) -> None:
    _check(lib.mq_set_gemv_variant(variant))


def mq_get_gemv_variant() -> int:
    return lib.mq_get_gemv_variant()


KERNEL_GEMV, KERNEL_GEMM = 1, 2


def mq_gemm_kernel(M: int, N: int, K: int, r: int) -> int:
    """KERNEL_GEMV or KERNEL_GEMM: the kernel mq_gemm would run (0: invalid)."""
    return lib.mq_gemm_kernel(M, N, K, r)


def uses_gemv(M: int, N: int, K: int, r: int) -> bool:
    return mq_gemm_kernel(M, N, K, r) == KERNEL_GEMV


def mq_device_status() -> None:
    """Synchronise the device; raise if a bounded wait in an earlier launch gave up."""
    _check(lib.mq_device_status())


def mq_version() -> str:
    return lib.mq_version().decode()


def mq_pack(codes, scales, planes_out, scales_out, stream=None) -> None:
    """codes uint8 [N, K], scales fp32 [N, K/128] -> planes_out (the 8 tiled
    planes, mq_plane_bytes(N, K, 8) bytes), scales_out (fp16 in the tiled
    block order, mq_scale_bytes(N, K) bytes); all on device."""
    N, K = codes.shape
    _check(lib.mq_pack(codes.data_ptr(), scales.data_ptr(), N, K, 128,
                       planes_out.data_ptr(), scales_out.data_ptr(), _stream(stream)))


def mq_slice(parent: MqWeights, r: int) -> MqWeights:
    out = MqWeights()
    _check(lib.mq_slice(ctypes.byref(parent), r, ctypes.byref(out)))
    return out


def mq_gemm(X, w: MqWeights, Y, workspace=None, stream=None) -> None:
    """Y[M, N] = X[M, K] . W_r^T (bf16 device tensors)."""
    M, K = X.shape
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.mq_gemm(X.data_ptr(), ctypes.byref(w), M, w.N, K, Y.data_ptr(),
                       ws_ptr, ws_bytes, _stream(stream)))


def mq_gemm_chain(calls, workspace=None, stream=None) -> None:
    """Enqueue the products [(X, w, Y), ...] back to back (X, Y bf16 device
    tensors, w an MqWeights view): a call may read the previous call's Y."""
    arr = (MqCall * len(calls))()
    keep = []
    for i, (X, w, Y) in enumerate(calls):
        wp = ctypes.pointer(w)
        keep.append(wp)
        arr[i] = MqCall(X.data_ptr(), wp, X.shape[0], Y.data_ptr())
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.mq_gemm_chain(arr, len(calls), ws_ptr, ws_bytes, _stream(stream)))


def mq_unpack(w: MqWeights, codes_out, stream=None) -> None:
    _check(lib.mq_unpack(ctypes.byref(w), codes_out.data_ptr(), _stream(stream)))


# ------------------------------------------------------------- owning helpers

class NestedWeights:
    """A packed 8-bit parent (device tensors) and its r-bit views; zeros16
    (fp16 zero points, asymmetric variant) or None."""

    def __init__(self, planes, scales16, N: int, K: int, zeros16=None):
        self.planes, self.scales16, self.N, self.K = planes, scales16, N, K
        self.zeros16 = zeros16
        self.parent = MqWeights(planes.data_ptr(), scales16.data_ptr(), N, K, 128, 8,
                                zeros16.data_ptr() if zeros16 is not None else None)

    def view(self, r: int) -> MqWeights:
        return mq_slice(self.parent, r)


def mq_pack_zeros(zeros, zeros_out, stream=None) -> None:
    """zero points fp32 [N, K/128] -> fp16 in the scales' tiled order (device)."""
    N, G = zeros.shape
    _check(lib.mq_pack_zeros(zeros.data_ptr(), N, G * 128, 128, zeros_out.data_ptr(), _stream(stream)))


def pack_parent(codes, scales, stream=None, zeros=None) -> NestedWeights:
    """Allocate the 8-plane buffer and fp16 scales with torch, then mq_pack;
    with `zeros` (fp32 [N, K/128]) the asymmetric variant."""
    import torch
    N, K = codes.shape
    planes = torch.empty(mq_plane_bytes(N, K, 8) // 4, dtype=torch.int32, device=codes.device)
    s16 = torch.empty(mq_scale_bytes(N, K, 128) // 2, dtype=torch.float16, device=codes.device)
    mq_pack(codes, scales, planes, s16, stream)
    z16 = None
    if zeros is not None:
        z16 = torch.empty(mq_scale_bytes(N, K, 128) // 2, dtype=torch.float16, device=codes.device)
        mq_pack_zeros(zeros, z16, stream)
    return NestedWeights(planes, s16, N, K, z16)


def pack_fused(codes_list, scales_list, stream=None) -> NestedWeights:
    """One parent for several layers that share X (q|k|v, gate|up): their
    rows concatenated (codes uint8 [N_i, K], scales fp32 [N_i, K/128] device
    tensors), so one launch computes all of them; Y's columns follow the same
    order (layer i at rows offsets[i] .. offsets[i] + N_i of W)."""
    import torch
    codes = torch.cat(list(codes_list), dim=0).contiguous()
    scales = torch.cat(list(scales_list), dim=0).contiguous()
    w = pack_parent(codes, scales, stream)
    offs, o = [], 0
    for c in codes_list:
        offs.append(o)
        o += c.shape[0]
    w.offsets = offs
    return w


def workspace_for(device, need: int):
    """The cached zero-initialised workspace of `device`, at least `need` bytes."""
    import torch
    key = device.index
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(max(need, 1 << 20), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def gemm_chain(calls, stream=None):
    """[(X, NestedWeights, r, Y or None), ...] -> the Y tensors, enqueued as
    one mq_gemm_chain (consecutive launches overlap)."""
    import torch
    views, outs, need = [], [], 0
    for X, weights, r, Y in calls:
        if Y is None:
            Y = torch.empty((X.shape[0], weights.N), dtype=torch.bfloat16, device=X.device)
        views.append((X, weights.view(r), Y))
        outs.append(Y)
        need = max(need, mq_gemm_workspace_bytes(X.shape[0], weights.N, weights.K, r))
    ws = workspace_for(calls[0][0].device, need) if need else None
    mq_gemm_chain(views, ws, stream)
    return outs


def bitwidth_search(table, budget_bytes: int):
    """table[l] = [(r, bytes, error), ...] per layer -> (index chosen per
    layer, summed error): the least summed error within the byte budget
    (mq_bitwidth_search; exact)."""
    L, C = len(table), len(table[0])
    arr = (MqChoice * (L * C))()
    for l, row in enumerate(table):
        if len(row) != C:
            raise ValueError("every layer needs the same number of candidates")
        for j, (r, nbytes, err) in enumerate(row):
            arr[l * C + j] = MqChoice(r, nbytes, err)
    out = (ctypes.c_int * L)()
    total = ctypes.c_double()
    _check(lib.mq_bitwidth_search(arr, L, C, budget_bytes, out, ctypes.byref(total)))
    return list(out), total.value


def matgptq_prepare(H, damp: float = 0.01):
    """U (K x K, fp64, upper) with U^T U = (H + damp * mean(diag H) * I)^-1
    (mq_matgptq_prepare, host)."""
    import numpy as np
    H = np.ascontiguousarray(H, np.float64)
    if H.ndim != 2 or H.shape[0] != H.shape[1]:
        raise ValueError("H must be a square matrix")
    K = H.shape[0]
    U = np.empty((K, K), np.float64)
    _check(lib.mq_matgptq_prepare(H.ctypes.data, K, float(damp), U.ctypes.data))
    return U


def matgptq_quantize(W, U, rs=(3, 4, 8), lambdas=(1.0, 1.0, 1.0),
                     alphas=(1.0, 0.95, 0.9, 0.85, 0.8), threads: int = 0, asymmetric: bool = False):
    """(codes uint8 N x K, scales fp32 N x K/128): the parent codes of the
    nested format from float weights W by the multi-precision column loop
    (mq_matgptq_quantize, host; the inputs of pack_parent).  asymmetric=True:
    (codes, scales, zeros) by mq_matgptq_quantize_asym (zeros: the input of
    pack_parent's `zeros`)."""
    import numpy as np
    W = np.ascontiguousarray(W, np.float32)
    U = np.ascontiguousarray(U, np.float64)
    if W.ndim != 2 or U.shape != (W.shape[1], W.shape[1]):
        raise ValueError("need W of N x K and U of K x K")
    if len(rs) != len(lambdas):
        raise ValueError("one lambda per bit width")
    N, K = W.shape
    rs_a = np.ascontiguousarray(rs, np.int32)
    lam_a = np.ascontiguousarray(lambdas, np.float64)
    al_a = np.ascontiguousarray(alphas, np.float64)
    codes = np.empty((N, K), np.uint8)
    scales = np.empty((N, max(K // 128, 1)), np.float32)
    args = (W.ctypes.data, N, K, U.ctypes.data, rs_a.ctypes.data, lam_a.ctypes.data, len(rs_a),
            al_a.ctypes.data, len(al_a), int(threads), codes.ctypes.data, scales.ctypes.data)
    if asymmetric:
        zeros = np.empty_like(scales)
        _check(lib.mq_matgptq_quantize_asym(*args, zeros.ctypes.data))
        return codes, scales, zeros
    _check(lib.mq_matgptq_quantize(*args))
    return codes, scales


def layer_errors(X, weights: NestedWeights, rs, stream=None):
    """{r: ||X W_r^T - X W_8^T||^2 / ||X W_8^T||^2} for one layer, the outputs
    computed by mq_gemm and reduced on the host in fp64 (the sensitivities a
    bit-width search consumes)."""
    import numpy as np
    ref = gemm(X, weights, 8, stream=stream).float().cpu().numpy().astype(np.float64)
    den = float(np.sum(ref * ref))
    out = {}
    for r in rs:
        y = gemm(X, weights, r, stream=stream).float().cpu().numpy().astype(np.float64)
        out[r] = float(np.sum((y - ref) ** 2)) / den
    return out


_ws_cache: dict = {}


def gemm(X, weights: NestedWeights, r: int, Y=None, stream=None):
    """Y = X . W_r^T with a cached, zero-initialised workspace per device."""
    import torch
    M, K = X.shape
    w = weights.view(r)
    if Y is None:
        Y = torch.empty((M, weights.N), dtype=torch.bfloat16, device=X.device)
    need = mq_gemm_workspace_bytes(M, weights.N, K, r)
    ws = workspace_for(X.device, need) if need else None
    mq_gemm(X, w, Y, ws, stream)
    return Y
