"""Cache write and copy-on-write block copy on the GPU: bit-exact against the
oracle's host scatter and memcpy."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_480_b200 as pkv
from paged_kv_cache_480_b200 import workloads as wl
from gpu_helpers import raw, same_bits

pytestmark = pytest.mark.gpu


def _rand_raw(shape, dtype, gen):
    t = torch.randn(shape, generator=gen, device="cuda").to(wl.torch_dtype(dtype))
    return t


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("stride_pad", [0, 3])
def test_reshape_and_cache_bit_exact(dtype, D, stride_pad):
    gen = torch.Generator(device="cuda").manual_seed(31)
    NB, Hkv, bs, T = 40, 4, 16, 150
    kc = _rand_raw((NB, Hkv, bs, D), dtype, gen)
    vc = _rand_raw((NB, Hkv, bs, D), dtype, gen)
    # key/value as a slice of a wider per-token row (token stride > Hkv * D)
    pad = stride_pad * (16 // torch.tensor([], dtype=wl.torch_dtype(dtype)).element_size())
    kbig = _rand_raw((T, Hkv * D + pad), dtype, gen)
    vbig = _rand_raw((T, Hkv * D + pad), dtype, gen)
    k = kbig[:, :Hkv * D].view(T, Hkv, D) if pad == 0 else kbig.as_strided((T, Hkv, D), (Hkv * D + pad, D, 1))
    v = vbig[:, :Hkv * D].view(T, Hkv, D) if pad == 0 else vbig.as_strided((T, Hkv, D), (Hkv * D + pad, D, 1))
    rng = np.random.default_rng(5)
    slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
    slots[::7] = -1
    hk, hv = raw(kc, dtype), raw(vc, dtype)
    oracle.reshape_and_cache(raw(k, dtype), raw(v, dtype), hk, hv, slots, bs)
    pkv.reshape_and_cache(k, v, kc, vc, torch.from_numpy(slots).cuda())
    assert pkv.read_device_errors() == 0
    assert same_bits(raw(kc, dtype), hk) and same_bits(raw(vc, dtype), hv)


def test_reshape_and_cache_out_of_pool_slot_is_flagged():
    gen = torch.Generator(device="cuda").manual_seed(32)
    kc = _rand_raw((4, 2, 16, 64), "bf16", gen)
    vc = kc.clone()
    before = kc.clone()
    k = _rand_raw((2, 2, 64), "bf16", gen)
    slots = torch.tensor([4 * 16 + 3, 5], dtype=torch.int64, device="cuda")
    pkv.reshape_and_cache(k, k, kc, vc, slots)
    assert pkv.read_device_errors() & 2
    changed = (kc.view(torch.int16) != before.view(torch.int16)).any(dim=-1)
    assert changed.sum().item() == 2 and changed[0, :, 5].all()   # only slot 5 written


@pytest.mark.parametrize("layers", [1, 3])
def test_copy_blocks_bit_exact(layers):
    gen = torch.Generator(device="cuda").manual_seed(33)
    NB, Hkv, bs, D = 64, 32, 16, 128
    ks = [_rand_raw((NB, Hkv, bs, D), "bf16", gen) for _ in range(layers)]
    vs = [_rand_raw((NB, Hkv, bs, D), "bf16", gen) for _ in range(layers)]
    rng = np.random.default_rng(4)
    ids = rng.permutation(NB)
    mapping = np.stack([ids[:20], ids[20:40]], axis=1).astype(np.int64)   # distinct src / dst
    host = [raw(t, "bf16") for t in ks + vs]
    oracle.copy_blocks(host, mapping)
    pkv.copy_blocks(ks, vs, torch.from_numpy(mapping).cuda())
    assert pkv.read_device_errors() == 0
    for t, h in zip(ks + vs, host):
        assert same_bits(raw(t, "bf16"), h)


def test_copy_blocks_bad_pair_is_flagged():
    gen = torch.Generator(device="cuda").manual_seed(34)
    k = _rand_raw((8, 2, 16, 64), "f16", gen)
    v = _rand_raw((8, 2, 16, 64), "f16", gen)
    before = k.clone()
    mapping = torch.tensor([[1, 2], [3, 99]], dtype=torch.int64, device="cuda")
    pkv.copy_blocks([k], [v], mapping)
    assert pkv.read_device_errors() & 8
    assert torch.equal(k[2].view(torch.int16), before[1].view(torch.int16))
    assert torch.equal(k[3].view(torch.int16), before[3].view(torch.int16))


def test_copy_blocks_overlapping_pairs_are_skipped_and_flagged():
    """Pairs whose result would depend on the order of the copies (a
    destination that is another pair's source, two pairs with one
    destination) are skipped and set PKV_DEVERR_COPY_OVERLAP; the other pairs,
    including several that share one source, are copied as the oracle copies
    them."""
    gen = torch.Generator(device="cuda").manual_seed(35)
    k = _rand_raw((16, 2, 16, 64), "bf16", gen)
    v = _rand_raw((16, 2, 16, 64), "bf16", gen)
    mapping = np.array([[1, 2], [2, 3],          # chain: 2 is a destination and a source
                        [4, 5], [6, 5],          # one destination twice
                        [7, 8], [7, 9], [10, 11]], np.int64)   # clean (one shared source)
    clean = mapping[4:]
    host = [raw(k, "bf16"), raw(v, "bf16")]
    oracle.copy_blocks(host, clean)
    pkv.copy_blocks([k], [v], torch.from_numpy(mapping).cuda())
    assert pkv.read_device_errors() == 32
    assert same_bits(raw(k, "bf16"), host[0]) and same_bits(raw(v, "bf16"), host[1])


def test_swap_blocks_repeated_destination_is_skipped_and_flagged():
    gen = torch.Generator(device="cuda").manual_seed(36)
    kd = _rand_raw((8, 2, 16, 64), "f16", gen)
    kh = torch.zeros((6, 2, 16, 64), dtype=torch.float16).pin_memory()
    mapping = np.array([[0, 1], [3, 1], [2, 4]], np.int64)     # pool-to-pool: a source may equal a destination id
    ref = raw(kh, "f16")
    oracle.swap_blocks([raw(kd, "f16")], [ref], mapping[2:])
    pkv.swap_blocks([kd], [kh], torch.from_numpy(mapping).cuda())
    torch.cuda.synchronize()
    assert pkv.read_device_errors() == 32
    assert same_bits(raw(kh, "f16"), ref)
