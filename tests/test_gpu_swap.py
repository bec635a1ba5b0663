"""swap_blocks between the GPU pool and a pinned host pool, and preemption by
swapping end to end: bit-exact copies against the oracle's memcpy, and the
attention of a sequence that was swapped out and back in (to new blocks)
equal to the oracle's over the never-moved cache."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_480_b200 as pkv
from paged_kv_cache_480_b200 import binding
from paged_kv_cache_480_b200 import workloads as wl
from gpu_helpers import compare, host_copy, oracle_step, raw, same_bits

pytestmark = pytest.mark.gpu


def _pools(NB_dev, NB_host, shape, dtype, seed):
    gen = torch.Generator(device="cuda").manual_seed(seed)
    dev = torch.randn((NB_dev,) + shape, generator=gen, device="cuda").to(wl.torch_dtype(dtype))
    host = torch.randn((NB_host,) + shape).to(wl.torch_dtype(dtype)).pin_memory()
    return dev, host


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_swap_out_and_in_bit_exact(dtype):
    shape = (8, 16, 128)
    kd, kh = _pools(64, 40, shape, dtype, 1)
    vd, vh = _pools(64, 40, shape, dtype, 2)
    rng = np.random.default_rng(3)
    out_map = np.stack([rng.choice(64, 25, replace=False), rng.choice(40, 25, replace=False)], 1)
    ref_h = [raw(kh, dtype), raw(vh, dtype)]
    oracle.swap_blocks([raw(kd, dtype), raw(vd, dtype)], ref_h, out_map)
    m = torch.from_numpy(out_map.astype(np.int64)).cuda()
    pkv.swap_blocks([kd, vd], [kh, vh], m)                 # device -> pinned host
    torch.cuda.synchronize()
    assert pkv.read_device_errors() == 0
    assert same_bits(raw(kh, dtype), ref_h[0]) and same_bits(raw(vh, dtype), ref_h[1])
    in_map = np.stack([rng.choice(40, 30, replace=False), rng.choice(64, 30, replace=False)], 1)
    ref_d = [raw(kd, dtype), raw(vd, dtype)]
    oracle.swap_blocks([raw(kh, dtype), raw(vh, dtype)], ref_d, in_map)
    pinned_map = torch.from_numpy(in_map.astype(np.int64)).pin_memory()   # mapping in pinned memory
    pkv.swap_blocks([kh, vh], [kd, vd], pinned_map)         # pinned host -> device
    torch.cuda.synchronize()
    assert pkv.read_device_errors() == 0
    assert same_bits(raw(kd, dtype), ref_d[0]) and same_bits(raw(vd, dtype), ref_d[1])


def test_pageable_host_memory_is_rejected():
    kd, _ = _pools(8, 4, (2, 16, 64), "bf16", 4)
    pageable = torch.zeros((4, 2, 16, 64), dtype=torch.bfloat16)
    m = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    with pytest.raises(binding.PagedKVError) as e:
        pkv.swap_blocks([kd], [pageable], m)
    assert e.value.status == 1


def test_bad_pair_is_flagged():
    kd, kh = _pools(8, 4, (2, 16, 64), "bf16", 5)
    before = kh.clone()
    m = torch.tensor([[0, 1], [3, 9]], dtype=torch.int64, device="cuda")
    pkv.swap_blocks([kd], [kh], m)
    torch.cuda.synchronize()
    assert pkv.read_device_errors() & 8
    assert torch.equal(kh[1].view(torch.int16), kd[0].cpu().view(torch.int16))
    assert torch.equal(kh[3].view(torch.int16), before[3].view(torch.int16))


def test_preemption_by_swap_end_to_end():
    """Sequences prefilled through the block manager; one is swapped out to the
    host pool, the others keep decoding, then it comes back to new blocks:
    every output matches the oracle on an unmoved copy of the data."""
    lay = wl.custom_layout("bf16", 32, 32, 128, 16, [300, 47, 129, 800], seed=50, pool_factor=1.0)
    S, Hkv, D, bs = lay.num_seqs, lay.num_kv_heads, lay.head_size, lay.block_size
    ten = wl.make_tensors(lay, device="cuda", pending_new_token=False)
    host = host_copy(ten, "bf16")
    ref = oracle_step(lay, host, write_new=False)
    NB = 2 * lay.num_blocks
    gpu_bm = pkv.BlockManager(NB, bs)
    host_bm = pkv.BlockManager(lay.num_blocks, bs)
    kc = torch.full((NB, Hkv, bs, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    kh = torch.zeros((lay.num_blocks, Hkv, bs, D), dtype=torch.bfloat16).pin_memory()
    vh = torch.zeros_like(kh).pin_memory()
    # prefill: copy each sequence's blocks from the workload pool into manager-chosen blocks
    for s in range(S):
        gpu_bm.allocate(s, int(lay.context_lens[s]))
        n = -(-int(lay.context_lens[s]) // bs)
        mapping = np.stack([lay.block_tables[s, :n], gpu_bm.block_table(s)], 1).astype(np.int64)
        pkv.swap_blocks([ten["k_cache"], ten["v_cache"]], [kc, vc], torch.from_numpy(mapping).cuda())
    victim = 2
    pairs = gpu_bm.swap_out(host_bm, victim)
    pkv.swap_blocks([kc, vc], [kh, vh], torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    # reuse the freed device blocks for a new sequence to make sure nothing stale is read
    gpu_bm.allocate(99, 16 * len(pairs))
    scrub = torch.from_numpy(gpu_bm.block_table(99).astype(np.int64)).cuda()
    kc[scrub] = float("nan")
    vc[scrub] = float("nan")
    back = host_bm.swap_out(gpu_bm, victim)
    pkv.swap_blocks([kh, vh], [kc, vc], torch.from_numpy(back).cuda())
    MB = lay.max_blocks_per_seq
    tables, lens = gpu_bm.fill_tables(np.arange(S), MB)
    assert np.array_equal(lens, lay.context_lens)
    out = torch.empty_like(ten["q"])
    pkv.paged_attention_decode(out, ten["q"], kc, vc, torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens).cuda(), lay.scale, max_context_len=lay.max_context_len)
    assert pkv.read_device_errors() == 0
    compare(out, ref, "bf16")
