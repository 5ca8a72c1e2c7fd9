"""Planted mistakes in a scratch copy of the C oracle must fail the pins.

Each mutation is a plausible slip (a dropped term, a wrong sign, a wrong
index, a transposed bit order).  The copy is compiled to a temporary
library; the real oracle is never modified.
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
import workloads as wl

SRC = os.path.join(os.path.dirname(oracle.__file__), "mq_oracle.c")

MUTATIONS = {
    "level_sign": ("b - 128.0", "b + 128.0"),
    "level_drop_half_step": ("a * (double)q_r + b - 128.0", "a * (double)q_r - 128.0"),
    "slice_shift": ("codes[n * K + k] >> (8 - r);\n            double w",
                    "codes[n * K + k] >> (7 - r);\n            double w"),
    "scale_index": ("s16[n * G + k / 128] * level(q_r, r);\n            acc += X[m * K + k]",
                    "s16[n * G + k % G] * level(q_r, r);\n            acc += X[m * K + k]"),
    "x_transposed": ("acc += X[m * K + k] * w;\n        }\n        out[i]",
                     "acc += X[k * 1 + m] * w;\n        }\n        out[i]"),
    "plane_order": ("(q >> (7 - p)) & 1u", "(q >> p) & 1u"),
    "bit_order": ("|= bit << (k % 32);", "|= bit << (31 - k % 32);"),
    "block_row": ("(n % 128) * 4 + (k % 128) / 32;", "(n % 128) + (k % 128) / 32 * 128;"),
    "block_order": ("((n / 128) * G + k / 128) * 512", "((k / 128) * G + n / 128) * 512"),
}


def _build_mutant(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, name
    d = tempfile.mkdtemp(prefix="mq_mut_")
    c = os.path.join(d, "m.c")
    so = os.path.join(d, "m.so")
    open(c, "w").write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-o", so, c])
    lib = ctypes.CDLL(so)
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.oracle_pack.argtypes = [P, I64, I64, P]
    lib.oracle_gemm_f64_at.argtypes = [P, P, P, I64, I, I64, P, P, P]
    return lib


def _pins_pass(lib):
    """Re-run the independent pins against the mutant; True if all hold."""
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    # pin 1: layout against numpy packbits
    codes = wl.adversarial_codes("random", 130, 256, seed=1)
    planes = np.empty((8, 256 * 8), np.uint32)
    lib.oracle_pack(ptr(codes), 130, 256, ptr(planes))
    from tests.test_oracle import _packbits_planes, _exact_gemm
    if not np.array_equal(planes, _packbits_planes(codes)):
        return False
    # pin 2: exact rational dot products on a tiny shape, several r
    for r in (8, 3, 2):
        cw, s, _ = wl.gen_weights(3, 256, seed=5)
        _, X = wl.gen_x(2, 256, seed=5)
        X = np.ascontiguousarray(X, np.float64)
        s16 = np.ascontiguousarray(oracle.scales_f16(s).astype(np.float64))
        ms = np.repeat(np.arange(2), 3).astype(np.int64)
        ns = np.tile(np.arange(3), 2).astype(np.int64)
        out = np.empty(6)
        lib.oracle_gemm_f64_at(ptr(X), ptr(cw), ptr(s16), 256, r, 6,
                               ptr(ms), ptr(ns), ptr(out))
        Ye = _exact_gemm(X, cw, s, r)
        for i in range(6):
            ex = float(Ye[ms[i]][ns[i]])
            if not abs(out[i] - ex) <= 1e-12 * abs(ex) + 1e-300:
                return False
    return True


def test_unmutated_copy_passes():
    src = open(SRC).read()
    d = tempfile.mkdtemp(prefix="mq_mut_")
    open(os.path.join(d, "m.c"), "w").write(src)
    MUTATIONS["_none"] = ("", "")
    try:
        assert _pins_pass(_build_mutant("_none"))
    finally:
        del MUTATIONS["_none"]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name):
    assert not _pins_pass(_build_mutant(name))
