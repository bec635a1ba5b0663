"""Paged prefill / chunked-prefill attention (tensor-core kernel) against the
oracle: every output element within the 16-bit bar (max-abs 1e-2, mean-abs
1e-3) at sizes the oracle finishes in seconds that span several query and
key tiles with ragged tails; at the full workload sizes, sampled query rows
against the decode oracle over the same cache with the context cut at the
query's position (query i of n at position L - n + i sees L - n + i + 1
keys)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_480_b200 as pkv
from paged_kv_cache_480_b200 import workloads as wl
from gpu_helpers import compare, compare_scaled, raw

pytestmark = pytest.mark.gpu


def _gpu(lay, ten, max_query_len=None):
    dev = ten["q"].device
    bt = torch.from_numpy(lay.block_tables).to(dev)
    cl = torch.from_numpy(lay.context_lens).to(dev)
    qsl = torch.from_numpy(lay.extra["query_start_loc"]).to(dev)
    if max_query_len is None:
        max_query_len = max(int(lay.extra["query_lens"].max()), 1)
    out = torch.full_like(ten["q"], float("nan"))
    pkv.paged_attention_prefill(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, qsl, lay.scale,
                                max_query_len=max_query_len)
    return out, pkv.read_device_errors()


def _oracle(lay, ten):
    return oracle.paged_prefill(raw(ten["q"], lay.dtype), raw(ten["k_cache"], lay.dtype),
                                raw(ten["v_cache"], lay.dtype), lay.block_tables, lay.context_lens,
                                lay.extra["query_start_loc"], lay.scale, lay.dtype, lay.num_kv_heads,
                                lay.block_size)


def _layout(dtype, H, Hkv, D, bs, lens, nq, seed=0):
    return wl.make_prefill_layout(context_lens=lens, query_lens=nq, dtype=dtype, num_heads=H,
                                  num_kv_heads=Hkv, head_size=D, block_size=bs, seed=wl.BASE_SEED + 100 + seed)


CASES = [
    # dtype, H, Hkv, D, bs, context lens, query lens
    ("bf16", 4, 4, 64, 16, [20, 37, 5, 200], [20, 10, 1, 200]),      # prompt, chunk, decode step, 2 query tiles
    ("f16", 8, 2, 128, 16, [70, 16, 333], [33, 16, 300]),            # G = 4: 32 queries per tile
    ("bf16", 8, 1, 64, 32, [100, 3, 517], [64, 3, 517]),             # G = 8: 16 queries per tile
    ("bf16", 16, 8, 128, 32, [1000, 130], [129, 130]),               # G = 2
    ("f16", 32, 32, 128, 16, [257, 64, 65, 1], [257, 64, 1, 1]),
    ("bf16", 4, 4, 128, 16, [128, 256, 64], [128, 256, 64]),         # exact multiples of the tiles
    ("bf16", 8, 8, 128, 16, [2000], [700]),                          # the K/V ring wraps many times
    ("f16", 16, 2, 64, 16, [777, 400], [300, 399]),                  # G = 8, D = 64
    ("bf16", 6, 2, 128, 16, [300, 90, 47], [300, 45, 47]),            # G = 3: 42 queries, 2 zero rows per tile
    ("f16", 15, 3, 64, 32, [260, 129], [100, 129]),                  # G = 5: 25 queries, 3 zero rows
    ("bf16", 32, 2, 128, 16, [500, 17, 9], [40, 17, 1]),             # G = 16: 8 queries per tile
    ("f16", 64, 1, 128, 32, [300, 70], [9, 5]),                      # G = 64 (MQA): 2 queries per tile
    ("bf16", 128, 1, 64, 16, [200, 3], [4, 3]),                      # G = 128: 1 query per tile
]


@pytest.mark.parametrize("dtype,H,Hkv,D,bs,lens,nq", CASES)
def test_prefill_matches_oracle(dtype, H, Hkv, D, bs, lens, nq):
    lay = _layout(dtype, H, Hkv, D, bs, lens, nq)
    ten = wl.make_prefill_tensors(lay, device="cuda")
    out, err = _gpu(lay, ten)
    assert err == 0, f"device check bits {err}"
    compare(out, _oracle(lay, ten), dtype)


def test_prefill_empty_query_lists():
    """Sequences with no queries this call take no rows and disturb nothing."""
    lay = _layout("bf16", 8, 4, 128, 16, [50, 300, 17, 90], [0, 130, 0, 90], seed=1)
    ten = wl.make_prefill_tensors(lay, device="cuda")
    out, err = _gpu(lay, ten)
    assert err == 0
    compare(out, _oracle(lay, ten), "bf16")


def test_prefill_single_query_equals_decode():
    """n = 1 per sequence is a decode step: the decode kernel on the same cache agrees."""
    lay = _layout("bf16", 32, 8, 128, 16, [900, 33, 1, 4100], [1, 1, 1, 1], seed=2)
    ten = wl.make_prefill_tensors(lay, device="cuda")
    out, err = _gpu(lay, ten)
    assert err == 0
    dev = torch.device("cuda")
    dec = torch.full_like(out, float("nan"))
    pkv.paged_attention_decode(dec, ten["q"], ten["k_cache"], ten["v_cache"],
                               torch.from_numpy(lay.block_tables).to(dev),
                               torch.from_numpy(lay.context_lens).to(dev), lay.scale,
                               max_context_len=lay.max_context_len)
    ref = _oracle(lay, ten)
    compare(out, ref, "bf16")
    compare(dec, ref, "bf16")
    assert (out.float() - dec.float()).abs().max().item() <= 1.6e-2


def test_prefill_too_many_queries_is_flagged():
    """n > L: the sequence is skipped (rows untouched) and the context bit set."""
    lay = _layout("bf16", 4, 4, 64, 16, [40, 60], [20, 30], seed=3)
    lay.context_lens = np.array([40, 20], np.int32)          # second: 30 queries but 20 tokens
    ten = wl.make_prefill_tensors(lay, device="cuda")
    out, err = _gpu(lay, ten)
    assert err & 4
    qsl = lay.extra["query_start_loc"]
    assert torch.isnan(out[qsl[1]:qsl[2]].float()).all()
    first = out[:qsl[1]]
    lay1 = _layout("bf16", 4, 4, 64, 16, [40], [20], seed=3)
    ten1 = {k: v for k, v in ten.items()}
    ten1["q"] = ten["q"][:qsl[1]].contiguous()
    lay1.block_tables, lay1.context_lens = lay.block_tables[:1], lay.context_lens[:1]
    compare(first, _oracle(lay1, ten1), "bf16")


def test_prefill_bad_block_id_is_flagged():
    lay = _layout("f16", 8, 8, 64, 16, [100], [100], seed=4)
    ten = wl.make_prefill_tensors(lay, device="cuda")
    lay.block_tables = lay.block_tables.copy()
    lay.block_tables[0, 2] = lay.num_blocks + 5
    out, err = _gpu(lay, ten)
    assert err & 1
    # keys 32..47 read as zeros: every output is still finite
    assert torch.isfinite(out.float()).all()


def test_prefill_query_bound_too_small_is_flagged():
    lay = _layout("bf16", 4, 4, 64, 16, [300], [300], seed=5)
    ten = wl.make_prefill_tensors(lay, device="cuda")
    out, err = _gpu(lay, ten, max_query_len=100)
    assert err & 4
    assert torch.isnan(out.float()).all()


def test_prefill_rejects_f32_and_bad_shapes():
    lay = _layout("bf16", 4, 4, 64, 16, [30], [30], seed=6)
    ten = wl.make_prefill_tensors(lay, device="cuda")
    dev = torch.device("cuda")
    bt = torch.from_numpy(lay.block_tables).to(dev)
    cl = torch.from_numpy(lay.context_lens).to(dev)
    qsl = torch.from_numpy(lay.extra["query_start_loc"]).to(dev)
    q32 = ten["q"].float()
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_attention_prefill(torch.empty_like(q32), q32, ten["k_cache"].float(),
                                    ten["v_cache"].float(), bt, cl, qsl, lay.scale, max_query_len=30)
    with pytest.raises(pkv.PagedKVError):      # bound above the token count
        pkv.paged_attention_prefill(torch.empty_like(ten["q"]), ten["q"], ten["k_cache"], ten["v_cache"],
                                    bt, cl, qsl, lay.scale, max_query_len=31)


JUMPS = [
    # dtype, H, Hkv, D, bs, context lens, query lens
    ("bf16", 8, 8, 128, 16, [700, 390], [700, 200]),
    ("f16", 16, 2, 64, 32, [600, 333], [300, 333]),
    ("bf16", 16, 4, 128, 32, [900], [260]),
]


@pytest.mark.parametrize("dtype,H,Hkv,D,bs,lens,nq", JUMPS)
def test_prefill_logit_jumps(dtype, H, Hkv, D, bs, lens, nq):
    """Keys scaled by 8 at random positions past the first key tile: their
    logits rise far above everything a row saw before, anywhere inside a key
    tile, so the row's reference moves in the middle of a tile whose earlier
    weights are already taken.  The inputs are checked to contain such rows."""
    lay = _layout(dtype, H, Hkv, D, bs, lens, nq, seed=7)
    ten = wl.make_prefill_tensors(lay, device="cuda")
    rng = np.random.default_rng(11)
    k = ten["k_cache"]
    for s, L in enumerate(lay.context_lens):
        for pos in rng.choice(np.arange(140, int(L)), size=8, replace=False):
            k[int(lay.block_tables[s, pos // bs]), :, int(pos % bs), :] *= 8
    # rows whose keys past the first tile reach 8 (log2 units) above that tile's maximum
    qf, kf = ten["q"].float().cpu().numpy(), k.float().cpu().numpy()
    qsl, nqs, G = lay.extra["query_start_loc"], lay.extra["query_lens"], H // Hkv
    jumps = 0
    for s, L in enumerate(lay.context_lens):
        L, n = int(L), int(nqs[s])
        keys = np.concatenate([kf[lay.block_tables[s, b]] for b in range((L + bs - 1) // bs)], axis=1)[:, :L]
        for i in range(max(0, 128 - (L - n)), n):
            pos = L - n + i
            lg = np.einsum("hd,hkd->hk", qf[qsl[s] + i].reshape(Hkv, G, D).reshape(H, D),
                           np.repeat(keys[:, :pos + 1], G, axis=0)) * lay.scale * np.log2(np.e)
            jumps += int((lg[:, 128:].max(axis=1) > lg[:, :128].max(axis=1) + 8).sum())
    assert jumps > 0
    out, err = _gpu(lay, ten)
    assert err == 0
    compare_scaled(out, _oracle(lay, ten), dtype)


@pytest.mark.parametrize("name", sorted(wl.PREFILL_CONFIGS))
def test_prefill_full_size_sampled(name):
    """The full workload in the launch the bench times; 48 sampled query rows
    checked against the decode oracle with the context cut at the query."""
    lay = wl.make_prefill_layout(name)
    ten = wl.make_prefill_tensors(lay, device="cuda")
    out, err = _gpu(lay, ten)
    assert err == 0
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(7)
    qsl, nq = lay.extra["query_start_loc"], lay.extra["query_lens"]
    seqs = rng.integers(0, lay.num_seqs, 48)
    picks = []
    for s in seqs:
        i = int(rng.integers(0, nq[s])) if rng.random() < 0.75 else int(nq[s]) - 1
        picks.append((int(s), i))
    rows = np.array([qsl[s] + i for s, i in picks])
    lens = np.array([lay.context_lens[s] - nq[s] + i + 1 for s, i in picks], np.int32)
    tables = lay.block_tables[[s for s, _ in picks]]
    q_rows = raw(ten["q"][torch.from_numpy(rows).cuda()], lay.dtype)
    ref = oracle.paged_attention(q_rows, raw(ten["k_cache"], lay.dtype), raw(ten["v_cache"], lay.dtype),
                                 tables, lens, lay.scale, lay.dtype, lay.num_kv_heads, lay.block_size)
    compare(out[torch.from_numpy(rows).cuda()], ref, lay.dtype)


@pytest.mark.parametrize("G", [1, 3, 16])
def test_prefill_wait_limit_gives_up_then_next_call_is_exact(G):
    """With the wait limit at 0 every role's first wait gives up: the call
    returns with PKV_DEVERR_WAIT set (each role lets its copies land, the MMA
    role waits for its issued products, the tensor memory is freed), and the
    next normal call matches the oracle."""
    lay = _layout("bf16", 2 * G, 2, 128, 16, [300, 40, 129], [300, 7, 129], seed=8 + G)
    ten = wl.make_prefill_tensors(lay, device="cuda")
    assert pkv.read_device_errors() == 0
    try:
        pkv.set_wait_limit(0)
        _, bits = _gpu(lay, ten)
    finally:
        pkv.set_wait_limit(-1)
    assert bits & 16, bits
    out, err = _gpu(lay, ten)
    assert err == 0
    compare(out, _oracle(lay, ten), "bf16")
