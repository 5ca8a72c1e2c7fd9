"""Per-layer sensitivities measured through mq_gemm (||X W_r^T - X W_8^T||^2
/ ||X W_8^T||^2 on seeded X) against the same quantity from the fp64 oracle,
and the bit-width search they drive (a Llama-3.1-8B decoder layer, r in
{2, 3, 4}, where the errors stand far above the bf16 rounding of Y)."""
import numpy as np
import pytest

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


def test_layer_sensitivities_and_search():
    import torch
    import nested_bit_weight_b200 as mq
    rs = (2, 3, 4)
    M = 16
    names = ("q_proj", "k_proj", "o_proj", "down_proj")
    gpu_table, ref_table = [], []
    for i, l in enumerate(wl.LLAMA8B):
        if l.name not in names:
            continue
        codes, s, _ = wl.gen_weights(l.N, l.K, wl.layer_seed(1, i))
        p = mq.pack_parent(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda())
        xbits, X = wl.gen_x(M, l.K, wl.layer_seed(1, i) + 77)
        Xd = torch.from_numpy(xbits.view(np.int16)).cuda().view(torch.bfloat16)
        got = mq.layer_errors(Xd, p, rs)
        y8 = oracle.gemm(X, codes, s, 8)
        den = float(np.sum(y8 * y8))
        row_gpu, row_ref = [], []
        for r in rs:
            yr = oracle.gemm(X, codes, s, r)
            ref = float(np.sum((yr - y8) ** 2)) / den
            assert abs(got[r] - ref) <= 0.02 * ref, (l.name, r, got[r], ref)
            nbytes = mq.mq_plane_bytes(l.N, l.K, r)
            row_gpu.append((r, nbytes, got[r]))
            row_ref.append((r, nbytes, ref))
        gpu_table.append(row_gpu)
        ref_table.append(row_ref)
    lo = sum(row[0][1] for row in ref_table)
    hi = sum(row[-1][1] for row in ref_table)
    for budget in (lo, (lo + hi) // 2, (2 * lo + hi) // 3, hi):
        pick_gpu, _ = mq.bitwidth_search(gpu_table, budget)
        pick_ref, best = mq.bitwidth_search(ref_table, budget)
        # the GPU-measured table leads to an optimal choice for the oracle's
        # errors (up to their 2 % agreement)
        val = sum(ref_table[l][pick_gpu[l]][2] for l in range(len(ref_table)))
        assert val <= best * 1.04 + 1e-30, (budget, pick_gpu, pick_ref)
