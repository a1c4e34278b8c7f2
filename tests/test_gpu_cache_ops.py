"""reshape_and_cache and copy_blocks on the GPU, bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import cache_ops
from tests.gpu_helpers import dev_bf16, host_bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D,bs,T", [(128, 16, 256), (128, 32, 37), (64, 16, 1), (64, 32, 1000)])
def test_reshape_and_cache_bit_exact(pkv, D, bs, T):
    rng = wl.rng_for(200 + T)
    NB, Hkv = 97, 5
    kc = wl.bf16_normal(rng, (NB, Hkv, bs, D))
    vc = wl.bf16_normal(rng, (NB, Hkv, bs, D))
    k = wl.bf16_normal(rng, (T, Hkv, D))
    v = wl.bf16_normal(rng, (T, Hkv, D))
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int64)
    slots[rng.random(T) < 0.1] = -1                      # skipped rows
    exp_k, exp_v = cache_ops.reshape_and_cache(k, v, kc, vc, slots)
    dkc, dvc = dev_bf16(kc), dev_bf16(vc)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.reshape_and_cache(dev_bf16(k), dev_bf16(v), dkc, dvc, torch.from_numpy(slots).cuda(), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert np.array_equal(host_bits(dkc), exp_k) and np.array_equal(host_bits(dvc), exp_v)


def test_reshape_and_cache_empty_and_bad_slot(pkv):
    rng = wl.rng_for(210)
    NB, Hkv, bs, D = 8, 2, 16, 128
    kc = wl.bf16_normal(rng, (NB, Hkv, bs, D))
    dkc, dvc = dev_bf16(kc), dev_bf16(kc)
    empty = torch.empty((0, Hkv, D), dtype=torch.bfloat16, device="cuda")
    pkv.reshape_and_cache(empty, empty, dkc, dvc, torch.empty(0, dtype=torch.int64, device="cuda"))
    k = wl.bf16_normal(rng, (3, Hkv, D))
    slots = np.array([5, NB * bs, 7], np.int64)         # the middle one is past the pool
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.reshape_and_cache(dev_bf16(k), dev_bf16(k), dkc, dvc, torch.from_numpy(slots).cuda(), status=status)
    torch.cuda.synchronize()
    assert status.item() == pkv.PKV_DEV_BAD_SLOT
    exp, _ = cache_ops.reshape_and_cache(k, k, kc, kc, np.array([5, -1, 7]))
    assert np.array_equal(host_bits(dkc), exp)


@pytest.mark.parametrize("layers,n", [(1, 1), (3, 17), (2, 0)])
def test_copy_blocks_bit_exact(pkv, layers, n):
    rng = wl.rng_for(220 + n)
    NB, Hkv, bs, D = 64, 8, 16, 128
    ks = [wl.bf16_normal(rng, (NB, Hkv, bs, D)) for _ in range(layers)]
    vs = [wl.bf16_normal(rng, (NB, Hkv, bs, D)) for _ in range(layers)]
    perm = rng.permutation(NB)
    pairs = np.stack([perm[:n], perm[n:2 * n]], axis=1).astype(np.int64).reshape(-1, 2)
    exp_k, exp_v = cache_ops.copy_blocks(ks, vs, pairs)
    dks, dvs = [dev_bf16(a) for a in ks], [dev_bf16(a) for a in vs]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.copy_blocks(dks, dvs, torch.from_numpy(pairs).cuda(), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for l in range(layers):
        assert np.array_equal(host_bits(dks[l]), exp_k[l]) and np.array_equal(host_bits(dvs[l]), exp_v[l])


@pytest.mark.parametrize("layers,n", [(1, 5), (2, 17)])
def test_copy_blocks_8bit_pools_bit_exact(pkv, layers, n):
    """Copy-on-write over e4m3 pools: the same bytewise copy, every code kept."""
    rng = wl.rng_for(240 + n)
    NB, Hkv, bs, D = 48, 8, 16, 128
    ks = [rng.integers(0, 256, size=(NB, Hkv, bs, D), dtype=np.uint8) for _ in range(layers)]
    vs = [rng.integers(0, 256, size=(NB, Hkv, bs, D), dtype=np.uint8) for _ in range(layers)]
    perm = rng.permutation(NB)
    pairs = np.stack([perm[:n], perm[n:2 * n]], axis=1).astype(np.int64)
    exp_k, exp_v = cache_ops.copy_blocks(ks, vs, pairs)
    dks = [torch.from_numpy(a).cuda() for a in ks]
    dvs = [torch.from_numpy(a).cuda() for a in vs]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.copy_blocks(dks, dvs, torch.from_numpy(pairs).cuda(), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for l in range(layers):
        assert np.array_equal(dks[l].cpu().numpy(), exp_k[l]) and np.array_equal(dvs[l].cpu().numpy(), exp_v[l])


def test_copy_blocks_bad_pair(pkv):
    rng = wl.rng_for(230)
    kc = wl.bf16_normal(rng, (4, 1, 16, 64))
    dk, dv = dev_bf16(kc), dev_bf16(kc)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.copy_blocks([dk], [dv], torch.tensor([[0, 9], [1, 2]], dtype=torch.int64, device="cuda"), status=status)
    torch.cuda.synchronize()
    assert status.item() == pkv.PKV_DEV_BAD_PAIR
    exp, _ = cache_ops.copy_blocks([kc], [kc], np.array([[1, 2]]))
    assert np.array_equal(host_bits(dk), exp[0])


@pytest.mark.parametrize("nbytes", [16, 48, 4096 + 32, (64 << 20) + 208])
def test_stream_read_folds_every_word(pkv, nbytes):
    """The bandwidth reference reads every byte once: its XOR of all 32-bit words equals
    numpy's on seeded bytes (sizes down to one 16-byte chunk, ragged grid tails)."""
    rng = np.random.default_rng(nbytes)
    host = rng.integers(0, 256, size=nbytes, dtype=np.uint8)
    buf = torch.from_numpy(host).cuda()
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.stream_read(buf, sink)
    torch.cuda.synchronize()
    want = np.bitwise_xor.reduce(host.view(np.uint32))
    assert np.uint32(sink.cpu().numpy().view(np.uint32)[0]) == want
