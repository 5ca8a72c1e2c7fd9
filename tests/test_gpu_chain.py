"""One decoder layer as a chain of launches: the Qwen3-8B linears at mixed
bit widths (attention r = 4, FFN r = 3), with q|k|v and gate|up each packed
as one fused parent, enqueued by mq_gemm_chain so that consecutive launches
overlap through programmatic dependent launch.  The o projection's output is
the gate|up input (a read of the previous launch's Y), the other inputs are
seeded X with x20 outlier channels.  Every output is checked against the fp64
oracle of its own layer; the oracle's gate|up input is the oracle's o output
rounded to bf16 (nothing computed on the GPU enters the oracle)."""
import numpy as np
import pytest

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

FULL_LIMIT = 2 * 10 ** 9


def _bf16_round(x: np.ndarray) -> np.ndarray:
    """fp64 -> the nearest bf16 (ties to even), as float32 values."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def _ratio(Y, X, codes, s, r, seed):
    """Violation ratio of Y against the oracle (whole output, or sampled
    positions covering every 128-row tile and every 32-row X block)."""
    M, N = Y.shape
    K = X.shape[1]
    if M * N * K <= FULL_LIMIT:
        return oracle.violation_ratio(Y, oracle.gemm(X, codes, s, r))
    rng = np.random.default_rng(seed)
    ns = np.concatenate([np.minimum(N - 1, t * 128 + rng.integers(128, size=2)) for t in range((N + 127) // 128)])
    ms = rng.integers(M, size=ns.shape[0])
    ms = np.concatenate([ms, rng.integers(M, size=512)])
    ns = np.concatenate([ns, rng.integers(N, size=512)])
    ref = oracle.gemm_at(X, codes, s, r, ms, ns)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return oracle.violation_ratio(Y[ms, ns], ref, rms)


@pytest.mark.parametrize("M", [1, 16, 64])
def test_qwen3_decoder_layer_chain(M):
    import torch
    import nested_bit_weight_b200 as mq
    L = {l.name: (i, l) for i, l in enumerate(wl.QWEN3_8B)}
    W = {}
    for name, (i, l) in L.items():
        codes, s, _ = wl.gen_weights(l.N, l.K, wl.layer_seed(3, i))
        W[name] = (codes, s)
    dev = lambda a: torch.from_numpy(a).cuda()
    qkv = mq.pack_fused([dev(W[n][0]) for n in ("q_proj", "k_proj", "v_proj")],
                        [dev(W[n][1]) for n in ("q_proj", "k_proj", "v_proj")])
    gu = mq.pack_fused([dev(W[n][0]) for n in ("gate_proj", "up_proj")],
                       [dev(W[n][1]) for n in ("gate_proj", "up_proj")])
    o = mq.pack_parent(dev(W["o_proj"][0]), dev(W["o_proj"][1]))
    down = mq.pack_parent(dev(W["down_proj"][0]), dev(W["down_proj"][1]))
    assert qkv.N == 4096 + 1024 + 1024 and qkv.offsets == [0, 4096, 5120]
    assert gu.N == 2 * 12288 and gu.offsets == [0, 12288]

    xa_bits, xa = wl.gen_x(M, 4096, wl.layer_seed(3, 0) + M, outlier_channels=True)
    xo_bits, xo = wl.gen_x(M, 4096, wl.layer_seed(3, 3) + M, outlier_channels=True)
    xd_bits, xd = wl.gen_x(M, 12288, wl.layer_seed(3, 6) + M, outlier_channels=True)
    bf = lambda b: torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16)
    Xa, Xo, Xd = bf(xa_bits), bf(xo_bits), bf(xd_bits)
    Yo = torch.empty((M, 4096), dtype=torch.bfloat16, device="cuda")
    Yqkv, Yo, Ygu, Yd = mq.gemm_chain([(Xa, qkv, 4, None), (Xo, o, 4, Yo),
                                       (Yo, gu, 3, None), (Xd, down, 3, None)])
    mq.mq_device_status()
    host = lambda t: t.float().cpu().numpy().astype(np.float64)
    Yqkv, Yo_h, Ygu, Yd = host(Yqkv), host(Yo), host(Ygu), host(Yd)

    for name, lo in (("q_proj", 0), ("k_proj", 4096), ("v_proj", 5120)):
        N = L[name][1].N
        assert _ratio(Yqkv[:, lo:lo + N], xa, *W[name], 4, seed=N + M) <= 1.0, name
    assert _ratio(Yo_h, xo, *W["o_proj"], 4, seed=7 + M) <= 1.0
    # the oracle's own o output, rounded to bf16, is its gate|up input
    xg = _bf16_round(oracle.gemm(xo, *W["o_proj"], 4))
    for name, lo in (("gate_proj", 0), ("up_proj", 12288)):
        assert _ratio(Ygu[:, lo:lo + 12288], xg, *W[name], 3, seed=lo + M) <= 1.0, name
    assert _ratio(Yd, xd, *W["down_proj"], 3, seed=11 + M) <= 1.0
