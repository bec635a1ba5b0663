"""Parity of paged decode attention (CUDA, through the C ABI) with the fp64
CPU oracle, element by element on the same seeded inputs.

Full-size workloads (the oracle handles them in seconds) and small cases
that span several partitions with ragged tails, every head size, block
size, group size and element type, empty and one-token contexts, and the
device-side checks."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_480_b200 as pkv
from paged_kv_cache_480_b200 import workloads as wl
from gpu_helpers import check_step, compare, compare_scaled, gpu_step, host_copy, oracle_step, raw, same_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_kv_cache_480_b200 import build
    build.build()
    pkv.load_library()


# ---------------------------------------------------------------------------
# keys whose logits jump far above the rest of the context
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name,ps", [("llama7b_bf16", 0), ("gqa_long_bf16", 0), ("gqa_long_bf16", 512),
                                     ("opt13b_f16", 0), ("tiny_mha_f32", 16), ("mqa_long_bf16", 0),
                                     ("mqa_long_bf16", 512)])
def test_decode_logit_jumps(name, ps):
    """Unit-variance inputs with the keys of random context positions scaled
    by 8: single keys dominate their rows, wherever they fall in a slice,
    block or partition (the merge sees partitions with very different
    maxima)."""
    lay = wl.make_layout(name, num_seqs=min(8, wl.make_layout(name).num_seqs))
    lay.value_scale = 1.0
    ten = wl.make_tensors(lay, device="cuda")
    rng = np.random.default_rng(5)
    bs = lay.block_size
    for s, L in enumerate(lay.context_lens):
        L = int(L)
        if L < 2:
            continue
        for pos in rng.choice(np.arange(L - 1), size=min(6, L - 1), replace=False):   # not the new token
            ten["k_cache"][int(lay.block_tables[s, pos // bs]), :, int(pos % bs), :] *= 8
    host = host_copy(ten, lay.dtype)
    out, err = gpu_step(lay, ten, ps)
    assert err == 0
    compare_scaled(out, oracle_step(lay, host), lay.dtype)


# ---------------------------------------------------------------------------
# the named workloads at full size
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("ps", [0, 16, 48])
def test_tiny_mha_f32(ps):
    lay = wl.make_layout("tiny_mha_f32")
    check_step(lay, partition_size=ps)


def test_opt13b_f16():
    lay = wl.make_layout("opt13b_f16")
    # q/K/V ~ N(0,1)/sqrt(128) makes the softmax nearly uniform: also bound
    # the normwise relative error so a wrong kernel cannot pass on size alone
    check_step(lay, rel_bar=1e-2)


def test_opt13b_shapes_unit_variance_f16():
    lay = wl.make_layout("opt13b_f16", num_seqs=16)
    lay.value_scale = 1.0
    check_step(lay, rel_bar=1e-2)


@pytest.mark.parametrize("bs", [16, 32])
def test_llama7b_bf16(bs):
    lay = wl.make_layout("llama7b_bf16", block_size=bs)
    check_step(lay, rel_bar=2e-2)


def test_gqa_long_bf16():
    lay = wl.make_layout("gqa_long_bf16")
    check_step(lay, rel_bar=2e-2)


def test_mqa_long_bf16():
    """64 query heads over one KV head at 16K-32K tokens: eight 8-head slices
    per KV head, split contexts and the merge."""
    lay = wl.make_layout("mqa_long_bf16")
    check_step(lay, rel_bar=2e-2)


# ---------------------------------------------------------------------------
# edge cases at small sizes
# ---------------------------------------------------------------------------
EDGE_LENS = [0, 1, 15, 16, 17, 255, 256, 257, 511, 512, 513, 1000, 33]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 6, 8, 16, 64])
def test_edge_lengths(dtype, D, bs, G):
    Hkv = 2
    lay = wl.custom_layout(dtype, num_heads=Hkv * G, num_kv_heads=Hkv, head_size=D, block_size=bs,
                           context_lens=EDGE_LENS, seed=7 + G + D + bs)
    check_step(lay)


@pytest.mark.parametrize("dtype,H,D,bs", [("bf16", 256, 128, 16), ("f16", 160, 64, 32), ("bf16", 130, 128, 32)])
def test_groups_beyond_128_heads(dtype, H, D, bs):
    """One KV head for more than 128 query heads: slices of 128 rows on the
    tensor cores (the last slice partly filled)."""
    lay = wl.custom_layout(dtype, num_heads=H, num_kv_heads=1, head_size=D, block_size=bs,
                           context_lens=[0, 1, 17, 255, 256, 257, 1000, 2049], seed=70 + H)
    check_step(lay)


def test_wide_group_more_sequences_than_threads():
    """The tensor-core decode's range search scans the lengths one block of
    threads (352) at a time: 700 sequences take two passes over two chunks,
    with empty and one-token contexts among them."""
    rng = np.random.default_rng(71)
    lens = rng.integers(0, 400, 700)
    lens[::97] = 0
    lens[5::89] = 1
    lay = wl.custom_layout("bf16", num_heads=32, num_kv_heads=2, head_size=128, block_size=16,
                           context_lens=lens.tolist(), seed=71)
    check_step(lay)


@pytest.mark.parametrize("ps_blocks", [1, 3, 32])
def test_forced_partitions(ps_blocks):
    lay = wl.custom_layout("bf16", 16, 2, 128, 16, [1, 47, 48, 49, 700, 1025, 2048, 16], seed=3)
    check_step(lay, partition_size=16 * ps_blocks)


def test_split_and_single_pass_agree():
    lay = wl.custom_layout("f16", 8, 8, 128, 16, [300, 512, 33, 511], seed=21)
    ten = wl.make_tensors(lay, device="cuda")
    outs = []
    for ps in (512, 16, 64):
        t2 = {k: v.clone() for k, v in ten.items()}
        out, err = gpu_step(lay, t2, partition_size=ps)
        assert err == 0
        outs.append(out.float())
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() <= 2e-3


def test_one_token_context_is_exact():
    lay = wl.custom_layout("bf16", 8, 4, 128, 16, [1] * 9, seed=5)
    ten = wl.make_tensors(lay, device="cuda")
    out, err = gpu_step(lay, ten)
    assert err == 0
    # out[s, h] must equal the new token's V row (the only context token), bit for bit
    want = ten["v_new"].repeat_interleave(2, dim=1)
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))


def test_empty_contexts_give_zero():
    lay = wl.custom_layout("f16", 4, 4, 64, 16, [0, 0, 5], seed=6)
    ten = wl.make_tensors(lay, device="cuda")
    out, err = gpu_step(lay, ten)
    assert err == 0
    assert torch.equal(out[:2], torch.zeros_like(out[:2]))


def test_block_permutation_invariance_bitwise():
    lay = wl.custom_layout("bf16", 8, 2, 128, 16, [100, 300, 17], seed=8)
    ten = wl.make_tensors(lay, device="cuda", pending_new_token=False)
    out1, err = gpu_step(lay, ten, write_new=False)
    assert err == 0
    perm = torch.randperm(lay.num_blocks, generator=torch.Generator().manual_seed(1))
    k2 = torch.empty_like(ten["k_cache"])
    v2 = torch.empty_like(ten["v_cache"])
    k2[perm.cuda()] = ten["k_cache"]
    v2[perm.cuda()] = ten["v_cache"]
    pn = perm.numpy()
    lay.block_tables = np.where(lay.block_tables >= 0, pn[np.maximum(lay.block_tables, 0)], -1).astype(np.int32)
    ten2 = dict(ten, k_cache=k2, v_cache=v2)
    out2, err = gpu_step(lay, ten2, write_new=False)
    assert err == 0
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_repeated_calls_are_bit_identical():
    """The work counter resets after every call; results do not depend on which warp ran what."""
    lay = wl.make_layout("llama7b_bf16", num_seqs=64)
    ten = wl.make_tensors(lay, device="cuda", pending_new_token=False)
    outs = [gpu_step(lay, ten, write_new=False)[0] for _ in range(4)]
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


def test_own_workspace_and_stream():
    lay = wl.custom_layout("bf16", 32, 32, 128, 16, [700, 1300, 90], seed=9)
    ten = wl.make_tensors(lay, device="cuda", pending_new_token=False)
    host = host_copy(ten, "bf16")
    ref = oracle_step(lay, host, write_new=False)
    need = pkv.paged_attention_workspace_size(3, 32, 32, 128, 16, 1300, 2, 0)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    out = torch.empty_like(ten["q"])
    bt = torch.from_numpy(lay.block_tables).cuda()
    cl = torch.from_numpy(lay.context_lens).cuda()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        for _ in range(3):
            pkv.paged_attention_decode(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, lay.scale,
                                       max_context_len=1300, workspace=ws, stream=s)
    s.synchronize()
    assert pkv.read_device_errors() == 0
    compare(out, ref, "bf16")
    assert torch.count_nonzero(ws[:256]).item() == 0     # counters left at zero


# ---------------------------------------------------------------------------
# device-side checks: bad inputs are skipped and reported, never faulted on
# ---------------------------------------------------------------------------
def test_bad_block_id_is_flagged():
    lay = wl.custom_layout("bf16", 4, 4, 64, 16, [40, 40], seed=10)
    ten = wl.make_tensors(lay, device="cuda", pending_new_token=False)
    lay.block_tables[1, 1] = lay.num_blocks + 5
    out, err = gpu_step(lay, ten, write_new=False)
    assert err & 1
    assert pkv.read_device_errors() == 0            # reading clears the bits


def test_context_beyond_bound_is_flagged():
    lay = wl.custom_layout("f16", 4, 4, 64, 16, [40, 30], seed=11)
    ten = wl.make_tensors(lay, device="cuda", pending_new_token=False)
    bt = torch.from_numpy(lay.block_tables).cuda()
    cl = torch.tensor([40, 30], dtype=torch.int32, device="cuda")
    out = torch.empty_like(ten["q"])
    # claim a bound of 32 tokens: sequence 0 exceeds it and is treated as empty
    pkv.paged_attention_decode(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, lay.scale,
                               max_context_len=32)
    assert pkv.read_device_errors() & 4
    assert torch.equal(out[0], torch.zeros_like(out[0]))


# ---------------------------------------------------------------------------
# bounded waits that run out: the call reports it, the next call is whole
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("G", [1, 8, 16])
def test_wait_limit_gives_up_then_next_call_is_exact(G):
    """With the wait limit at 0 every wait for a stage's copies gives up at
    once: the call returns, sets PKV_DEVERR_WAIT and leaves the workspace's
    counters at zero, so the next normal call on the same workspace matches
    the oracle element by element."""
    lay = wl.custom_layout("bf16", 2 * G, 2, 128, 16, [700, 1300, 90, 1, 0, 513], seed=40 + G)
    ten = wl.make_tensors(lay, device="cuda", pending_new_token=False)
    host = host_copy(ten, "bf16")
    ref = oracle_step(lay, host, write_new=False)
    need = pkv.paged_attention_workspace_size(lay.num_seqs, lay.num_heads, 2, 128, 16, 1300, 2, 0)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    bt = torch.from_numpy(lay.block_tables).cuda()
    cl = torch.from_numpy(lay.context_lens).cuda()
    out = torch.empty_like(ten["q"])
    assert pkv.read_device_errors() == 0
    try:
        pkv.set_wait_limit(0)
        pkv.paged_attention_decode(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, lay.scale,
                                   max_context_len=1300, workspace=ws)
        bits = pkv.read_device_errors()
    finally:
        pkv.set_wait_limit(-1)
    assert bits & 16, bits
    assert torch.count_nonzero(ws[:256]).item() == 0     # counters reset on the give-up path too
    out.fill_(float("nan"))
    pkv.paged_attention_decode(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, lay.scale,
                               max_context_len=1300, workspace=ws)
    assert pkv.read_device_errors() == 0
    compare(out, ref, "bf16")
