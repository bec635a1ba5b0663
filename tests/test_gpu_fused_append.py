"""The fused cache write + decode (paged_attention_decode_append) against the
two-call path and the oracle: caches bit-identical to reshape_and_cache's,
attention within the bar, bad slots flagged."""
import numpy as np
import pytest
import torch

import paged_kv_cache_480_b200 as pkv
from paged_kv_cache_480_b200 import workloads as wl
from gpu_helpers import compare, host_copy, oracle_step, raw, same_bits

pytestmark = pytest.mark.gpu


def _fused(lay, ten, ps=0, key=None, value=None, slots=None):
    dev = ten["q"].device
    bt = torch.from_numpy(lay.block_tables).to(dev)
    cl = torch.from_numpy(lay.context_lens).to(dev)
    sm = torch.from_numpy(lay.slot_mapping if slots is None else slots).to(dev)
    out = torch.full_like(ten["q"], float("nan"))
    pkv.paged_attention_decode_append(out, ten["q"], ten["k_new"] if key is None else key,
                                      ten["v_new"] if value is None else value, ten["k_cache"],
                                      ten["v_cache"], sm, bt, cl, lay.scale,
                                      max_context_len=max(lay.max_context_len, 1), partition_size=ps)
    return out, pkv.read_device_errors()


CASES = [
    ("opt13b_f16", dict(num_seqs=16), 0),
    ("llama7b_bf16", dict(num_seqs=48), 0),
    ("llama7b_bf16", dict(num_seqs=48, block_size=32), 0),
    ("gqa_long_bf16", dict(num_seqs=4), 0),
    ("tiny_mha_f32", dict(), 0),
    ("tiny_mha_f32", dict(), 16),
]


@pytest.mark.parametrize("name,kw,ps", CASES)
def test_fused_append_matches_oracle_and_two_call_path(name, kw, ps):
    lay = wl.make_layout(name, **kw)
    ten = wl.make_tensors(lay, device="cuda")
    host = host_copy(ten, lay.dtype)
    out, err = _fused(lay, ten, ps)
    assert err == 0
    ref = oracle_step(lay, host)             # oracle: scatter, then attention
    assert same_bits(raw(ten["k_cache"], lay.dtype), host["k_cache"])
    assert same_bits(raw(ten["v_cache"], lay.dtype), host["v_cache"])
    compare(out, ref, lay.dtype)


@pytest.mark.parametrize("dtype,G,D,bs", [("bf16", 8, 128, 16), ("f16", 4, 64, 32), ("f32", 1, 128, 16),
                                          ("bf16", 2, 128, 32), ("bf16", 3, 128, 16), ("f32", 3, 64, 16),
                                          ("bf16", 16, 128, 16), ("f16", 16, 64, 32), ("bf16", 64, 128, 16),
                                          ("f16", 64, 128, 32)])
def test_fused_append_edge_lengths(dtype, G, D, bs):
    lens = [0, 1, 15, 16, 17, 255, 256, 257, 513, 1000]
    lay = wl.custom_layout(dtype, 2 * G, 2, D, bs, lens, seed=40 + G)
    ten = wl.make_tensors(lay, device="cuda")
    host = host_copy(ten, dtype)
    out, err = _fused(lay, ten)
    assert err == 0
    ref = oracle_step(lay, host)
    assert same_bits(raw(ten["k_cache"], dtype), host["k_cache"])
    assert same_bits(raw(ten["v_cache"], dtype), host["v_cache"])
    compare(out, ref, dtype)


def test_fused_append_strided_key_value():
    lay = wl.custom_layout("bf16", 8, 4, 128, 16, [30, 200, 1], seed=41)
    ten = wl.make_tensors(lay, device="cuda")
    host = host_copy(ten, "bf16")
    # new K/V as slices of a wider per-token row
    wide = torch.zeros((3, 4 * 128 * 2 + 64), dtype=torch.bfloat16, device="cuda")
    key = wide[:, :512].view(3, 4, 128)
    value = wide[:, 512:1024].view(3, 4, 128)
    key.copy_(ten["k_new"])
    value.copy_(ten["v_new"])
    out, err = _fused(lay, ten, key=key, value=value)
    assert err == 0
    ref = oracle_step(lay, host)
    assert same_bits(raw(ten["k_cache"], "bf16"), host["k_cache"])
    compare(out, ref, "bf16")


def test_slot_that_is_not_the_last_position_is_flagged_and_skipped():
    lay = wl.custom_layout("f16", 4, 4, 64, 16, [40, 40], seed=42)
    ten = wl.make_tensors(lay, device="cuda", pending_new_token=False)
    before = ten["k_cache"].clone()
    slots = lay.slot_mapping.copy()
    slots[1] -= 1                       # points one position too early
    slots[0] = -1                       # no new token for sequence 0
    out, err = _fused(lay, ten, slots=slots)
    assert err & 2
    assert torch.equal(ten["k_cache"].view(torch.int16), before.view(torch.int16))   # nothing written
