"""FP8 (E4M3) KV cache on the GPU against the oracle: the quantising cache
write bit for bit, and decode attention over E4M3 caches within the
output dtype's bar (fp32 q: 1e-5 relative; 16-bit: 1e-2 / 1e-3)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_480_b200 as pkv
from paged_kv_cache_480_b200 import workloads as wl
from gpu_helpers import compare, raw, same_bits

pytestmark = pytest.mark.gpu

KS, VS = 1.0 / 64, 1.0 / 48


def _u8(t):
    return t.detach().contiguous().cpu().numpy().copy()


def _step(lay, ten, ps=0):
    dev = ten["q"].device
    bt = torch.from_numpy(lay.block_tables).to(dev)
    cl = torch.from_numpy(lay.context_lens).to(dev)
    sm = torch.from_numpy(lay.slot_mapping).to(dev)
    pkv.reshape_and_cache_fp8kv(ten["k_new"], ten["v_new"], ten["k_cache"], ten["v_cache"], sm, KS, VS)
    out = torch.full_like(ten["q"], float("nan"))
    pkv.paged_attention_decode_fp8kv(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, lay.scale,
                                     KS, VS, max_context_len=max(lay.max_context_len, 1),
                                     partition_size=ps)
    return out, pkv.read_device_errors()


def _oracle(lay, host):
    oracle.reshape_and_cache_fp8(host["k_new"], host["v_new"], lay.dtype, host["k_cache"], host["v_cache"],
                                 lay.slot_mapping, lay.block_size, KS, VS)
    return oracle.paged_attention_fp8(host["q"], lay.dtype, host["k_cache"], host["v_cache"], KS, VS,
                                      lay.block_tables, lay.context_lens, lay.scale, lay.num_kv_heads,
                                      lay.block_size)


def _check(lay, ps=0):
    ten = wl.make_tensors_fp8(lay, device="cuda", k_scale=KS, v_scale=VS)
    host = {"q": raw(ten["q"], lay.dtype), "k_new": raw(ten["k_new"], lay.dtype),
            "v_new": raw(ten["v_new"], lay.dtype), "k_cache": _u8(ten["k_cache"]),
            "v_cache": _u8(ten["v_cache"])}
    out, err = _step(lay, ten, ps)
    assert err == 0
    ref = _oracle(lay, host)
    assert same_bits(_u8(ten["k_cache"]), host["k_cache"]) and same_bits(_u8(ten["v_cache"]), host["v_cache"])
    return compare(out, ref, lay.dtype)


@pytest.mark.parametrize("name,kw", [("opt13b_f16", dict(num_seqs=24)), ("llama7b_bf16", dict(num_seqs=64)),
                                     ("llama7b_bf16", dict(num_seqs=64, block_size=32)),
                                     ("gqa_long_bf16", dict(num_seqs=4)), ("tiny_mha_f32", dict())])
def test_fp8_step_matches_oracle(name, kw):
    _check(wl.make_layout(name, **kw))


@pytest.mark.parametrize("dtype,G,D,bs", [("bf16", 8, 128, 16), ("bf16", 4, 64, 32), ("f16", 8, 64, 16),
                                          ("f16", 1, 128, 32), ("bf16", 2, 64, 16), ("f32", 8, 128, 16),
                                          ("f32", 1, 64, 32), ("bf16", 3, 128, 16), ("f16", 3, 64, 32),
                                          ("f32", 3, 128, 16), ("bf16", 16, 128, 16), ("f16", 16, 128, 32),
                                          ("bf16", 64, 128, 16), ("f32", 64, 64, 16)])
def test_fp8_edge_lengths(dtype, G, D, bs):
    lay = wl.custom_layout(dtype, 2 * G, 2, D, bs, [0, 1, 15, 16, 17, 255, 257, 513, 1000], seed=60 + G + D)
    _check(lay)


def test_fp8_mqa_long():
    """The MQA workload's shape (64 query heads over one KV head) over E4M3 caches."""
    _check(wl.make_layout("mqa_long_bf16", num_seqs=4))


def test_fp8_forced_partitions():
    lay = wl.custom_layout("bf16", 16, 2, 128, 16, [1, 47, 700, 2048], seed=61)
    _check(lay, ps=48)


def test_fp8_cache_write_saturates_and_keeps_nan():
    kc = torch.zeros((2, 1, 16, 64), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    k = torch.tensor([[1e4, -1e4, float("nan"), 3.0] * 16], dtype=torch.float32, device="cuda").view(1, 1, 64)
    sm = torch.tensor([5], dtype=torch.int64, device="cuda")
    pkv.reshape_and_cache_fp8kv(k, k.clone(), kc, vc, sm, 1.0, 1.0)
    row = kc[0, 0, 5, :4].cpu().tolist()
    assert row == [0x7e, 0xfe, 0x7f, oracle.e4m3_bits(3.0)]
    assert pkv.read_device_errors() == 0
