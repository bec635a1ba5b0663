"""Parallel sampling with copy-on-write, end to end (the cow_bf16 workload).

GPU side: the library's block manager allocates each prompt's prefix,
forks the samples (shared, reference-counted blocks), and every generation
step asks it for slots and copy-on-write pairs, then runs copy_blocks and
reshape_and_cache on the device; a final decode attends over every sample.
Oracle side: the reference block-manager model, host scatter/memcpy and the
fp64 attention replay the same steps on host copies.  Physical ids may
differ; the attention output and the copy counts may not.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_480_b200 as pkv
from oracle.block_manager_model import BlockManagerModel
from paged_kv_cache_480_b200 import workloads as wl
from gpu_helpers import compare, raw

pytestmark = pytest.mark.gpu

BF16_NAN = 0x7fc0


def check_cache_contents(cache, host, gpu_tables, model_tables, lens, bs, chunk=512):
    """Every sequence's keys (or values) read through the GPU manager's table
    equal, bit for bit, those read through the model's table from the oracle's
    pool: each GPU block pairs with one model block, and their rows holding
    context tokens are identical."""
    pair_rows = {}
    for s, L in enumerate(lens):
        for j in range(-(-int(L) // bs)):
            key = (int(gpu_tables[s, j]), int(model_tables[s, j]))
            pair_rows[key] = max(pair_rows.get(key, 0), min(bs, int(L) - j * bs))
    gb = np.array([k[0] for k in pair_rows], np.int64)
    mb = np.array([k[1] for k in pair_rows], np.int64)
    nv = np.array(list(pair_rows.values()), np.int64)
    assert len(np.unique(gb)) == len(gb) and len(np.unique(mb)) == len(mb), "blocks pair up one to one"
    dev_host = torch.from_numpy(host.view(np.int16))
    cache16 = cache.view(torch.int16)
    for a in range(0, len(gb), chunk):
        g = torch.from_numpy(gb[a:a + chunk]).to(cache.device)
        m = torch.from_numpy(mb[a:a + chunk])
        got = cache16[g]                                   # [n, Hkv, bs, D]
        want = dev_host[m].to(cache.device)
        rows = torch.arange(bs, device=cache.device)[None, :] < torch.from_numpy(nv[a:a + chunk]).to(cache.device)[:, None]
        bad = (got != want).any(dim=-1) & rows[:, None, :]
        assert not bad.any().item(), f"{int(bad.sum())} cache rows differ"


def run_scenario(sc):
    dev = "cuda"
    NB, Hkv, bs, D = sc.num_blocks, sc.num_kv_heads, sc.block_size, sc.head_size
    bm = pkv.BlockManager(NB, bs, free_order=np.random.default_rng(sc.seed + 1).permutation(NB))
    model = BlockManagerModel(NB, bs)
    kc = torch.full((NB, Hkv, bs, D), float("nan"), dtype=torch.bfloat16, device=dev)
    vc = torch.full_like(kc, float("nan"))
    hk = np.full((NB, Hkv, bs, D), BF16_NAN, np.uint16)
    hv = hk.copy()

    pk, pv = wl.cow_prefix_kv(sc, dev)
    hpk, hpv = raw(pk, "bf16"), raw(pv, "bf16")
    pos = 0
    for p in range(sc.num_prompts):
        root, L = p * sc.samples, int(sc.prefix_lens[p])
        bm.allocate(root, L)
        model.allocate(root, L)
        t = np.arange(L)
        gslots = bm.block_table(root)[t // bs].astype(np.int64) * bs + t % bs
        mslots = np.asarray(model.tables[root], np.int64)[t // bs] * bs + t % bs
        pkv.reshape_and_cache(pk[pos:pos + L], pv[pos:pos + L], kc, vc, torch.from_numpy(gslots).to(dev))
        oracle.reshape_and_cache(hpk[pos:pos + L], hpv[pos:pos + L], hk, hv, mslots, bs)
        pos += L
        for j in range(1, sc.samples):
            bm.fork(root, root + j)
            model.fork(root, root + j)

    copies = []
    for step in range(sc.max_steps()):
        act = sc.active(step)
        gslots, gpairs = bm.append_slots(act)
        mres = [model.append_slot(int(s)) for s in act]
        mslots = np.array([r[0] for r in mres], np.int64)
        mpairs = np.array([r[1] for r in mres if r[1] is not None], np.int64).reshape(-1, 2)
        assert len(gpairs) == len(mpairs)
        copies.append(len(gpairs))
        if len(gpairs):
            pkv.copy_blocks([kc], [vc], torch.from_numpy(np.ascontiguousarray(gpairs)).to(dev))
            oracle.copy_blocks([hk, hv], mpairs)
        k, v = wl.cow_step_kv(sc, step, dev)
        pkv.reshape_and_cache(k, v, kc, vc, torch.from_numpy(gslots).to(dev))
        oracle.reshape_and_cache(raw(k, "bf16"), raw(v, "bf16"), hk, hv, mslots, bs)

    seqs = np.arange(sc.num_seqs)
    lens = sc.final_lens()
    MB = int(-(-lens.max() // bs))
    gt, gl = bm.fill_tables(seqs, MB)
    assert np.array_equal(gl, lens)
    mt = np.full((sc.num_seqs, MB), -1, np.int32)
    for s in seqs:
        mt[s, :len(model.tables[s])] = model.tables[s]
    check_cache_contents(kc, hk, gt, mt, lens, bs)
    check_cache_contents(vc, hv, gt, mt, lens, bs)
    q = wl.cow_queries(sc, dev)
    out = torch.empty_like(q)
    pkv.paged_attention_decode(out, q, kc, vc, torch.from_numpy(gt).to(dev),
                               torch.from_numpy(gl).to(dev), sc.scale, max_context_len=int(lens.max()))
    assert pkv.read_device_errors() == 0
    ref = oracle.paged_attention(raw(q, "bf16"), hk, hv, mt, lens, sc.scale, "bf16", Hkv, bs)
    stats = compare(out, ref, "bf16", rel_bar=2e-2)
    return copies, stats, bm, model


def test_cow_small():
    sc = wl.make_cow_scenario(num_prompts=4, samples=8, prefix=100, own_max=40)
    copies, stats, bm, model = run_scenario(sc)
    assert copies[0] > 0
    assert bm.num_free() == model.num_free()
    assert bm.utilisation() == pytest.approx(model.utilisation())


def test_cow_full_workload():
    """64 prompts x 8 samples, prefixes of 1024 - r tokens, U{0..256} own tokens each."""
    sc = wl.make_cow_scenario()
    copies, stats, bm, model = run_scenario(sc)
    # every prompt's shared last prefix block is partly filled and held by all
    # 8 samples: a writer copies it while another holder remains, so with k
    # writers there are min(k, 7) copies (samples that never write keep theirs)
    starters = (sc.own_tokens > 0).sum(axis=1)
    assert copies[0] == int(np.minimum(starters, sc.samples - 1).sum())
    assert sum(copies) == copies[0]


def test_cow_whole_block_prefix_needs_no_copy():
    """A prefix of exactly 1024 tokens fills its blocks: no copy is ever made."""
    sc = wl.make_cow_scenario(num_prompts=8, r_max=0, own_max=20)
    copies, stats, bm, model = run_scenario(sc)
    assert sum(copies) == 0
