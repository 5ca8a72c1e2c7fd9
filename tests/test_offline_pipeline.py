"""The offline half of the method end to end on the host: the one-shot
quantizer gives each layer one 8-bit parent, each width r of it has a proxy
loss tr(dW_r H dW_r^T) (through the oracle's dequantization, stored fp16
scales included) and a byte cost (the library's size functions), and the
budget-aware search picks one width per layer; its pick must be an optimum
of exhaustive enumeration and fit the budget."""
import numpy as np

import oracle
import workloads as wl
import nested_bit_weight_b200 as mq

RS = (2, 3, 4, 8)


def _layer_table(N, K, seed):
    H = wl.gen_hessian(K, seed, samples=2 * K)
    W = wl.gen_float_weights(N, K, seed + 1)
    codes, scales = mq.matgptq_quantize(W, mq.matgptq_prepare(H), rs=(3, 4, 8))
    W64 = W.astype(np.float64)
    row = []
    for r in RS:
        D = W64 - oracle.dequant(codes, scales, r)
        loss = float(np.einsum("nk,kl,nl->", D, H, D))
        nbytes = mq.mq_plane_bytes(N, K, r) + mq.mq_scale_bytes(N, K, 128)
        row.append((r, nbytes, loss))
    return row


def test_quantize_then_search_within_a_budget():
    shapes = [(64, 256), (128, 256), (64, 384), (192, 128)]
    table = [_layer_table(N, K, 300 + 10 * i) for i, (N, K) in enumerate(shapes)]
    # the losses fall from 2 to 3 to 4 bits on every layer; with lambda =
    # (1, 1, 1) the 8-bit slice follows the shared feedback of the coarse
    # slices and can cost more than the 4-bit one, which the search must see
    for row in table:
        losses = [e for _, _, e in row]
        assert losses[0] > losses[1] > losses[2]
    all8 = sum(row[-1][1] for row in table)
    for frac in (0.3, 0.45, 0.6, 1.0):
        budget = int(all8 * frac)
        pick, total = mq.bitwidth_search(table, budget)
        ref = oracle.bitwidth_search_exhaustive([[e for _, _, e in row] for row in table],
                                                [[b for _, b, _ in row] for row in table], budget)
        assert ref is not None
        best_err, best_bytes, optima = ref
        assert tuple(pick) in [tuple(p) for p in optima]
        assert sum(table[l][j][1] for l, j in enumerate(pick)) <= budget
        assert np.isclose(total, best_err, rtol=1e-12)
    # with every choice affordable, each layer takes its least-loss width
    pick, _ = mq.bitwidth_search(table, all8)
    for l, j in enumerate(pick):
        assert table[l][j][2] == min(e for _, _, e in table[l])
