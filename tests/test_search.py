"""Budget-aware per-layer bit-width search (mq_bitwidth_search, host only):
the exact dynamic program against exhaustive enumeration (oracle/), its
tie rule, budget monotonicity and its argument errors.  No GPU."""
import math

import numpy as np
import pytest

import nested_bit_weight_b200 as mq
import oracle


def test_exhaustive_oracle_hand_worked():
    # 2 layers x 2 widths, worked by hand: within 30 bytes the best is the
    # wide first layer (20 B, 1.0) with the narrow second (10 B, 3.0)
    errs = [[5.0, 1.0], [3.0, 0.5]]
    nb = [[10, 20], [10, 20]]
    e, b, picks = oracle.bitwidth_search_exhaustive(errs, nb, 30)
    assert (e, b, picks) == (4.0, 30, [(1, 0)])
    assert oracle.bitwidth_search_exhaustive(errs, nb, 19) is None
    e, b, picks = oracle.bitwidth_search_exhaustive(errs, nb, 40)
    assert (e, b, picks) == (1.5, 40, [(1, 1)])


def _table(errs, nb, rs=None):
    return [[(rs[j] if rs else j, nb[l][j], errs[l][j]) for j in range(len(errs[l]))]
            for l in range(len(errs))]


@pytest.mark.parametrize("seed", range(60))
def test_dp_matches_exhaustive(seed):
    rng = np.random.default_rng(seed)
    L, C = int(rng.integers(1, 6)), int(rng.integers(1, 5))
    unit = int(rng.choice([1, 3, 512, 1 << 19]))
    nb = (rng.integers(1, 9, size=(L, C)) * unit).tolist()
    errs = rng.random((L, C)).tolist()
    lo, hi = sum(min(r) for r in nb), sum(max(r) for r in nb)
    budget = int(rng.integers(lo, hi + 1))
    pick, total = mq.bitwidth_search(_table(errs, nb), budget)
    e, b, picks = oracle.bitwidth_search_exhaustive(errs, nb, budget)
    assert sum(nb[l][pick[l]] for l in range(L)) <= budget
    assert math.isclose(total, e, rel_tol=1e-12, abs_tol=1e-15)
    assert math.isclose(sum(errs[l][pick[l]] for l in range(L)), e, rel_tol=1e-12, abs_tol=1e-15)
    if len(picks) == 1:                    # a unique optimum: the same indices
        assert tuple(pick) == picks[0]


def test_ties_take_fewer_bytes():
    # equal errors: the cheaper candidate; equal errors and bytes: the lower index
    pick, _ = mq.bitwidth_search([[(4, 20, 1.0), (2, 10, 1.0)]], 100)
    assert pick == [1]
    pick, _ = mq.bitwidth_search([[(4, 10, 1.0), (3, 10, 1.0)]], 100)
    assert pick == [0]


def test_budget_monotone_and_extremes():
    # a Llama-like table: the error falls with r, the bytes grow with r
    rs = [2, 3, 4, 6, 8]
    shapes = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096),
              (4096, 14336)]
    sens = [1.0, 0.3, 0.3, 0.8, 0.5, 0.5, 1.2]
    table = [[(r, mq.mq_plane_bytes(N, K, r), s * 4.0 ** (-r)) for r in rs]
             for (N, K), s in zip(shapes, sens)]
    lo = sum(row[0][1] for row in table)
    hi = sum(row[-1][1] for row in table)
    prev = math.inf
    for budget in np.linspace(lo, hi, 25).astype(np.int64):
        pick, total = mq.bitwidth_search(table, int(budget))
        assert total <= prev + 1e-18
        prev = total
    assert mq.bitwidth_search(table, lo)[0] == [0] * 7            # everything at r = 2
    assert mq.bitwidth_search(table, hi)[0] == [4] * 7            # everything at r = 8


def test_argument_errors():
    with pytest.raises(mq.MQError) as e:
        mq.bitwidth_search([[(2, 10, 1.0)], [(2, 10, 1.0)]], 19)    # nothing fits
    assert e.value.status == 2
    with pytest.raises(mq.MQError) as e:
        mq.bitwidth_search([[(2, 10, -1.0)]], 100)                   # negative error
    assert e.value.status == 1
    with pytest.raises(mq.MQError) as e:
        mq.bitwidth_search([[(2, 10, float("nan"))]], 100)
    assert e.value.status == 1
    with pytest.raises(mq.MQError) as e:
        mq.bitwidth_search([[(2, 1, 1.0), (3, 2, 0.5)]] * 64, 1 << 24)  # 64 x 2^24 cells
    assert e.value.status == 2
