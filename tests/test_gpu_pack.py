"""GPU parity of the bit-plane packer and unpacker against the CPU oracle
(bit-exact: these are integer results)."""
import numpy as np
import pytest

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _pack(codes, scales):
    import nested_bit_weight_b200 as mq
    return mq.pack_parent(_dev(codes), _dev(scales))


KINDS = ("zeros", "ones", "alternating", "single_bit", "all_codes", "random")


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("N,K", [(1, 128), (7, 384), (64, 512), (33, 1280), (130, 256),
                                 (256, 384)])
def test_pack_bit_exact(kind, N, K):
    # whole buffers, padding rows included (they must be zero on both sides)
    codes = wl.adversarial_codes(kind, N, K, seed=N + K)
    s = wl.gen_scales(N, K, seed=N)
    w = _pack(codes, s)
    got = w.planes.cpu().numpy().view(np.uint32).reshape(8, -1)
    assert np.array_equal(got, oracle.pack(codes))
    s16 = w.scales16.cpu().numpy()
    assert np.array_equal(s16.view(np.uint16), oracle.scales_stored(s).view(np.uint16))


@pytest.mark.parametrize("r", range(1, 9))
def test_unpack_bit_exact(r):
    import torch
    import nested_bit_weight_b200 as mq
    N, K = 96, 640
    codes, s, _ = wl.gen_weights(N, K, seed=r)
    w = _pack(codes, s)
    out = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    mq.mq_unpack(w.view(r), out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), oracle.unpack(oracle.pack(codes), r, N, K))
    assert np.array_equal(out.cpu().numpy(), oracle.slice_codes(codes, r))


def test_pack_large_layer():
    # full Llama gate/up size (14336 x 4096): every word against the C oracle
    N, K = 14336, 4096
    codes, s, _ = wl.gen_weights(N, K, seed=4)
    w = _pack(codes, s)
    got = w.planes.cpu().numpy().view(np.uint32).reshape(8, -1)
    assert np.array_equal(got, oracle.pack(codes))
    assert np.array_equal(w.scales16.cpu().numpy().view(np.uint16),
                          oracle.scales_stored(s).view(np.uint16))


@pytest.mark.parametrize("bad", [-1.0, float("nan"), 1e6])
def test_pack_rejects_unstorable_scale(bad):
    import nested_bit_weight_b200 as mq
    codes = wl.adversarial_codes("random", 4, 256)
    s = wl.gen_scales(4, 256, seed=1)
    s[1, 1] = bad
    with pytest.raises(mq.MQError) as e:
        _pack(codes, s)
    assert e.value.status == 2


def test_pack_zero_scale_is_kept():
    codes = wl.adversarial_codes("random", 8, 256)
    s = wl.gen_scales(8, 256, seed=2, zero_groups=5)
    w = _pack(codes, s)
    assert np.array_equal(w.scales16.cpu().numpy().view(np.uint16),
                          oracle.scales_stored(s).view(np.uint16))
