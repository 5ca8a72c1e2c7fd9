"""Precision of the GEMM's tensor-core operands, measured on the CPU.

The batched kernel multiplies the exact r-bit levels v_r (bf16 holds them
exactly: at most 8 significant bits) and applies the fp16 scale of each
128-column group in fp32 afterwards, instead of folding s * v into one
16-bit operand and accumulating all of K in the tensor core.  These probes
show why, on the recipe's weights and activations (outlier weights x10,
outlier X channels x20) against the fp64 oracle and the tolerance
|Y - Y_ref| <= 8e-3 |Y_ref| + 1e-3 rms(Y_ref):

* s * v rounded to bf16 fails about 5 % of the outputs;
* s * v rounded to fp16 (X converted to fp16, exact for these values) uses
  most of the tolerance and fails outright on a 4096 x 4096 layer at
  M = 64 with outlier channels;
* the exact levels with the scale applied per group, followed by the bf16
  rounding of Y the kernel does, use under half of it.
"""
import numpy as np
import pytest

import oracle
import workloads as wl


def _bf16(a: np.ndarray) -> np.ndarray:
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def _ratios(N, K, M, r, seed, outliers):
    codes, s, _ = wl.gen_weights(N, K, seed)
    _, X = wl.gen_x(M, K, seed, outlier_channels=outliers)
    W = oracle.dequant(codes, s, r)               # exact s16 * v_r in fp64
    X64 = X.astype(np.float64)
    Yref = X64 @ W.T
    y_bf16_ops = X64 @ _bf16(W).T
    y_fp16_ops = X.astype(np.float16).astype(np.float64) @ W.astype(np.float16).astype(np.float64).T
    y_exact_bf16_out = _bf16(Yref)
    return {"bf16_ops": oracle.violation_ratio(y_bf16_ops, Yref),
            "bf16_ops_fail_frac": float(np.mean(np.abs(y_bf16_ops - Yref) > oracle.tolerance(Yref))),
            "fp16_ops": oracle.violation_ratio(y_fp16_ops, Yref),
            "exact_bf16_out": oracle.violation_ratio(y_exact_bf16_out, Yref)}


def test_operand_precision_small_layer():
    got = _ratios(1024, 4096, 64, 4, seed=3000, outliers=True)
    assert got["bf16_ops"] > 3.0 and got["bf16_ops_fail_frac"] > 0.02
    assert got["fp16_ops"] > 0.6                  # most of the budget, before Y is rounded
    assert got["exact_bf16_out"] < 0.5            # what the kernel's arithmetic leaves


def test_fp16_operands_fail_on_a_full_layer():
    got = _ratios(4096, 4096, 64, 4, seed=3000, outliers=True)
    assert got["fp16_ops"] > 1.0
    assert got["exact_bf16_out"] < 0.5
