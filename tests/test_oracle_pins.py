"""Pins of the CPU oracle to things other than itself (CPU only).

Each test ties an oracle function to an independent fact: a library routine
on a contiguous layout (torch's scaled_dot_product_attention, numpy's fp16
rounding, torch's bf16 widening, numpy fancy indexing), a closed form, an
invariant of the definition, or a brute-force search.  Chosen so that a
dropped scale, a transposed or mis-indexed operand, a wrong head grouping,
a missing max-subtraction or a partition off-by-one fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_480_b200 import workloads as wl

HERE = os.path.dirname(os.path.abspath(__file__))


# ---------------------------------------------------------------------------
# helpers: contiguous K/V scattered into a shuffled pool by the test itself
# ---------------------------------------------------------------------------
def _raw_from_torch(t, dtype):
    t = t.contiguous()
    if dtype == "f32":
        return t.numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


def build_paged(rng, lens, H, Hkv, D, bs, dtype, value_scale=1.0, pool_extra=3):
    """Contiguous per-sequence K/V plus the same data in a paged pool.

    Returns (q, Kc, Vc, kc_raw, vc_raw, q_raw, tables) where Kc/Vc are lists
    of float64 [Hkv, L, D] (exact values of the stored format).
    """
    tdt = wl.torch_dtype(dtype)
    nblk = [-(-L // bs) for L in lens]
    NB = sum(nblk) + pool_extra
    ids = rng.permutation(NB)
    tables = np.full((len(lens), max(1, max(nblk))), -1, np.int32)
    kc = torch.full((NB, Hkv, bs, D), float("nan"), dtype=tdt)
    vc = torch.full((NB, Hkv, bs, D), float("nan"), dtype=tdt)
    Kc, Vc = [], []
    pos = 0
    for s, L in enumerate(lens):
        K = (torch.from_numpy(rng.standard_normal((Hkv, L, D))) * value_scale).to(tdt)
        V = (torch.from_numpy(rng.standard_normal((Hkv, L, D))) * value_scale).to(tdt)
        tables[s, :nblk[s]] = ids[pos:pos + nblk[s]]
        pos += nblk[s]
        for t in range(L):
            kc[tables[s, t // bs], :, t % bs, :] = K[:, t, :]
            vc[tables[s, t // bs], :, t % bs, :] = V[:, t, :]
        Kc.append(K.double())
        Vc.append(V.double())
    q = (torch.from_numpy(rng.standard_normal((len(lens), H, D))) * value_scale).to(tdt)
    return q.double(), Kc, Vc, _raw_from_torch(kc, dtype), _raw_from_torch(vc, dtype), \
        _raw_from_torch(q, dtype), tables


def sdpa_reference(q, Kc, Vc, scale, G):
    """torch SDPA (fp64, CPU) on the contiguous K/V; heads grouped h // G."""
    outs = []
    for s in range(q.shape[0]):
        K = Kc[s].repeat_interleave(G, dim=0)     # [H, L, D]
        V = Vc[s].repeat_interleave(G, dim=0)
        if K.shape[1] == 0:
            outs.append(torch.zeros(q.shape[1], q.shape[2], dtype=torch.float64))
            continue
        o = torch.nn.functional.scaled_dot_product_attention(
            q[s][:, None, :], K, V, scale=scale)     # [H, 1, D]
        outs.append(o[:, 0, :])
    return torch.stack(outs).numpy()


CASES = [
    # dtype, H, Hkv, D, bs, lens
    ("f32", 4, 4, 64, 16, [1, 17, 33, 100]),
    ("f16", 8, 2, 128, 16, [5, 16, 47, 130]),
    ("bf16", 8, 1, 64, 32, [31, 32, 33, 70]),
    ("bf16", 16, 2, 128, 16, [200, 3]),
]


@pytest.mark.parametrize("dtype,H,Hkv,D,bs,lens", CASES)
def test_paged_attention_matches_sdpa_on_contiguous_kv(dtype, H, Hkv, D, bs, lens):
    rng = np.random.default_rng(1234)
    q, Kc, Vc, kc, vc, qr, tables = build_paged(rng, lens, H, Hkv, D, bs, dtype)
    scale = 1.0 / math.sqrt(D)
    got = oracle.paged_attention(qr, kc, vc, tables, np.array(lens, np.int32), scale, dtype, Hkv, bs)
    ref = sdpa_reference(q, Kc, Vc, scale, H // Hkv)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_scale_is_applied():
    rng = np.random.default_rng(5)
    q, Kc, Vc, kc, vc, qr, tables = build_paged(rng, [40], 2, 2, 64, 16, "f32")
    lens = np.array([40], np.int32)
    a = oracle.paged_attention(qr, kc, vc, tables, lens, 0.125, "f32", 2, 16)
    b = oracle.paged_attention(qr, kc, vc, tables, lens, 0.5, "f32", 2, 16)
    np.testing.assert_allclose(a, sdpa_reference(q, Kc, Vc, 0.125, 1), atol=1e-12)
    np.testing.assert_allclose(b, sdpa_reference(q, Kc, Vc, 0.5, 1), atol=1e-12)
    assert np.abs(a - b).max() > 1e-3


def test_gqa_grouping_is_contiguous():
    """Query head h reads KV head h // G: agrees with repeat_interleave, not with tiling."""
    rng = np.random.default_rng(9)
    H, Hkv, D = 8, 2, 64
    q, Kc, Vc, kc, vc, qr, tables = build_paged(rng, [50, 9], H, Hkv, D, 16, "f32")
    lens = np.array([50, 9], np.int32)
    got = oracle.paged_attention(qr, kc, vc, tables, lens, 0.125, "f32", Hkv, 16)
    np.testing.assert_allclose(got, sdpa_reference(q, Kc, Vc, 0.125, H // Hkv), atol=1e-12)
    tiled = []
    for s in range(2):
        K = Kc[s].repeat(H // Hkv, 1, 1)
        V = Vc[s].repeat(H // Hkv, 1, 1)
        o = torch.nn.functional.scaled_dot_product_attention(q[s][:, None, :], K, V, scale=0.125)
        tiled.append(o[:, 0, :])
    assert np.abs(got - torch.stack(tiled).numpy()).max() > 1e-3


def test_one_token_context_returns_v_exactly():
    rng = np.random.default_rng(3)
    for dtype in ("f32", "f16", "bf16"):
        q, Kc, Vc, kc, vc, qr, tables = build_paged(rng, [1, 1], 4, 2, 64, 16, dtype)
        out = oracle.paged_attention(qr, kc, vc, tables, np.array([1, 1], np.int32), 0.3, dtype, 2, 16)
        for s in range(2):
            for h in range(4):
                assert np.array_equal(out[s, h], Vc[s][h // 2, 0].numpy())
        # rounding the exact value back to the stored format is the identity
        v_raw = np.stack([np.stack([vc[tables[s, 0], h // 2, 0] for h in range(4)]) for s in range(2)])
        assert np.array_equal(oracle.round_to(out, dtype), v_raw)


def test_equal_keys_give_mean_of_v():
    rng = np.random.default_rng(4)
    lens = [37]
    q, Kc, Vc, kc, vc, qr, tables = build_paged(rng, lens, 2, 2, 64, 16, "f32")
    # overwrite every key of the context with one key
    for t in range(lens[0]):
        kc[tables[0, t // 16], :, t % 16, :] = kc[tables[0, 0], :, 0, :]
    out = oracle.paged_attention(qr, kc, vc, tables, np.array(lens, np.int32), 0.125, "f32", 2, 16)
    np.testing.assert_allclose(out[0], Vc[0].mean(dim=1).numpy(), atol=1e-14)


def test_weights_sum_to_one_and_two_token_closed_form():
    rng = np.random.default_rng(6)
    q, Kc, Vc, kc, vc, qr, tables = build_paged(rng, [2, 90], 2, 1, 64, 16, "f32")
    lens = np.array([2, 90], np.int32)
    scale = 0.2
    w = oracle.attention_weights(qr, kc, vc, tables, lens, scale, "f32", 1, 16, 1, 1)
    assert w.shape == (90,) and (w >= 0).all()
    assert abs(w.sum() - 1.0) < 1e-14
    # two tokens: w0 = logistic(z0 - z1) with z = scale * q.k (plain dot products)
    qv = q[0, 0].numpy()
    z0 = scale * float(qv @ Kc[0][0, 0].numpy())
    z1 = scale * float(qv @ Kc[0][0, 1].numpy())
    sig = 1.0 / (1.0 + math.exp(-(z0 - z1)))
    out = oracle.paged_attention(qr, kc, vc, tables, lens, scale, "f32", 1, 16)
    expect = sig * Vc[0][0, 0].numpy() + (1.0 - sig) * Vc[0][0, 1].numpy()
    np.testing.assert_allclose(out[0, 0], expect, atol=1e-14)


def test_large_logits_do_not_overflow():
    """Logits far beyond exp's range: the result must still be the softmax."""
    rng = np.random.default_rng(8)
    q, Kc, Vc, kc, vc, qr, tables = build_paged(rng, [20], 1, 1, 64, 16, "f32")
    lens = np.array([20], np.int32)
    out = oracle.paged_attention(qr, kc, vc, tables, lens, 400.0, "f32", 1, 16)
    assert np.isfinite(out).all()
    np.testing.assert_allclose(out, sdpa_reference(q, Kc, Vc, 400.0, 1), atol=1e-12)


def test_block_permutation_invariance():
    """Moving physical blocks (table rewritten to match) changes nothing, bit for bit."""
    rng = np.random.default_rng(10)
    lens = [45, 16, 77]
    q, Kc, Vc, kc, vc, qr, tables = build_paged(rng, lens, 4, 2, 64, 16, "bf16")
    L = np.array(lens, np.int32)
    a = oracle.paged_attention(qr, kc, vc, tables, L, 0.125, "bf16", 2, 16)
    perm = rng.permutation(kc.shape[0])          # new position of old block b is perm[b]
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    t2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1).astype(np.int32)
    b = oracle.paged_attention(qr, kc2, vc2, t2, L, 0.125, "bf16", 2, 16)
    assert np.array_equal(a, b)


def test_empty_context_gives_zero():
    rng = np.random.default_rng(11)
    q, Kc, Vc, kc, vc, qr, tables = build_paged(rng, [0, 5], 2, 2, 64, 16, "f16")
    out = oracle.paged_attention(qr, kc, vc, tables, np.array([0, 5], np.int32), 0.1, "f16", 2, 16)
    assert np.array_equal(out[0], np.zeros_like(out[0]))
    assert np.isfinite(out).all()


@pytest.mark.parametrize("ps", [16, 32, 48, 64, 1000])
def test_partition_merge_equals_single_pass(ps):
    rng = np.random.default_rng(12)
    lens = [1, 16, 17, 63, 64, 65, 130]
    q, Kc, Vc, kc, vc, qr, tables = build_paged(rng, lens, 4, 2, 64, 16, "bf16")
    L = np.array(lens, np.int32)
    P = -(-max(lens) // ps)
    acc, m, l = oracle.partition_stats(qr, kc, vc, tables, L, 0.125, "bf16", 2, 16, ps, P)
    merged = oracle.lse_merge(acc, m, l)
    full = oracle.paged_attention(qr, kc, vc, tables, L, 0.125, "bf16", 2, 16)
    np.testing.assert_allclose(merged, full, rtol=0, atol=1e-13)
    for s, n in enumerate(lens):
        nparts = -(-n // ps)
        assert np.isneginf(m[s, :, nparts:]).all() and (l[s, :, nparts:] == 0).all()
        assert (l[s, :, :nparts] >= 1.0).all()      # the max term contributes exp(0) = 1
        # m of a partition is the largest logit in it (via SDPA-independent dots)
        for h in range(4):
            z = 0.125 * (Kc[s][h // 2].numpy() @ q[s, h].numpy())
            for p in range(nparts):
                assert m[s, h, p] == pytest.approx(z[p * ps:(p + 1) * ps].max(), abs=1e-13)


def test_lse_merge_of_two_halves_by_hand():
    """Merge identity on explicit numbers: two parts with known softmax sums."""
    acc = np.array([[[2.0, 4.0], [1.0, -1.0]]])      # [R=1, P=2, D=2]
    m = np.array([[0.0, math.log(3.0)]])
    l = np.array([[2.0, 1.0]])
    # weights exp(m - M) with M = log 3: [1/3, 1]; out = (acc0/3 + acc1) / (2/3 + 1)
    expect = (acc[0, 0] / 3.0 + acc[0, 1]) / (2.0 / 3.0 + 1.0)
    np.testing.assert_allclose(oracle.lse_merge(acc, m, l)[0], expect, atol=1e-15)


# ---------------------------------------------------------------------------
# storage-format widening and rounding
# ---------------------------------------------------------------------------
def test_decode_all_f16_and_bf16_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    f16 = oracle.decode(bits, "f16")
    ref16 = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(np.isnan(f16), np.isnan(ref16))
    ok = ~np.isnan(ref16)
    assert np.array_equal(f16[ok], ref16[ok])
    bf = oracle.decode(bits, "bf16")
    refbf = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    ok = ~np.isnan(refbf)
    assert np.array_equal(bf[ok], refbf[ok]) and np.isnan(bf[~ok]).all()
    # the C loader (used inside the attention) agrees with the widening above
    lib = oracle._load()
    for b in (0x0001, 0x03ff, 0x0400, 0x3c00, 0x7bff, 0xfbff, 0x8001):
        arr = np.array([b], np.uint16)
        assert lib.orc_load(arr.ctypes.data, oracle.F16, 0) == ref16[b]


def _probe_values(rng, lo_exp, hi_exp, n=4000):
    mag = np.exp2(rng.uniform(lo_exp, hi_exp, n))
    return np.concatenate([mag, -mag, [0.0, -0.0]])


def test_f16_rounding_matches_numpy():
    rng = np.random.default_rng(13)
    x = _probe_values(rng, -27, 17)
    # exact ties: midpoints of adjacent fp16 values
    b = np.arange(0, 0x7bff, 37, dtype=np.uint16)
    lo = b.view(np.float16).astype(np.float64)
    hi = (b + 1).view(np.float16).astype(np.float64)
    x = np.concatenate([x, (lo + hi) / 2, [65504.0, 65519.9, 65520.0, 1e6, 2.0 ** -25, 3 * 2.0 ** -26]])
    got = np.array([oracle.f16_bits(v) for v in x], np.uint16)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def _nearest_even_table(dtype):
    bits = np.arange(65536, dtype=np.uint16)
    vals = oracle.decode(bits, dtype) if dtype == "f16" else \
        torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    keep = np.isfinite(vals) & ~((vals == 0) & (bits != 0) & (bits != 0x8000))
    return bits[keep], vals[keep]


def test_bf16_rounding_is_nearest_even_by_brute_force():
    bits, vals = _nearest_even_table("bf16")
    pos = vals >= 0
    pb, pv = bits[pos & (bits < 0x8000)], vals[pos & (bits < 0x8000)]
    order = np.argsort(pv)
    pb, pv = pb[order], pv[order]
    rng = np.random.default_rng(14)
    mags = np.exp2(rng.uniform(-135, 127, 3000))
    mids = (pv[:-1] + pv[1:])[::97] / 2
    for x in np.concatenate([mags, mids, pv[::211]]):
        i = np.searchsorted(pv, x)
        cands = [j for j in (i - 1, i) if 0 <= j < len(pv)]
        dist = [abs(pv[j] - x) for j in cands]
        best = [cands[k] for k in range(len(cands)) if dist[k] == min(dist)]
        if len(best) > 1:
            best = [j for j in best if pb[j] % 2 == 0]
        want = int(pb[best[0]])
        assert oracle.bf16_bits(x) == want, (x, hex(oracle.bf16_bits(x)), hex(want))
        assert oracle.bf16_bits(-x) == (want | 0x8000)
    # overflow threshold: halfway between the largest finite value and 2^128
    top = (2 - 2.0 ** -7) * 2.0 ** 127
    assert oracle.bf16_bits(top) == 0x7f7f
    assert oracle.bf16_bits((2 - 2.0 ** -8) * 2.0 ** 127) == 0x7f80
    assert oracle.bf16_bits(np.nextafter((2 - 2.0 ** -8) * 2.0 ** 127, 0)) == 0x7f7f


def test_round_to_matches_torch_for_fp32_representable_values():
    """For values exact in fp32, one-step rounding equals torch's fp32->bf16 cast."""
    rng = np.random.default_rng(15)
    x = rng.standard_normal(20000).astype(np.float32).astype(np.float64)
    got = oracle.round_to(x, "bf16")
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------------------
# cache write and block copy
# ---------------------------------------------------------------------------
def test_reshape_and_cache_matches_indexed_assignment():
    rng = np.random.default_rng(16)
    NB, Hkv, bs, D, T = 12, 3, 16, 64, 20
    kc = rng.integers(0, 65535, (NB, Hkv, bs, D)).astype(np.uint16)
    vc = rng.integers(0, 65535, (NB, Hkv, bs, D)).astype(np.uint16)
    k = rng.integers(0, 65535, (T, Hkv, D)).astype(np.uint16)
    v = rng.integers(0, 65535, (T, Hkv, D)).astype(np.uint16)
    slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
    slots[[3, 11]] = -1
    ref_k, ref_v = kc.copy(), vc.copy()
    ok = slots >= 0
    # library scatter: view the cache as [NB*bs, Hkv, D] rows
    rk = ref_k.transpose(0, 2, 1, 3).reshape(NB * bs, Hkv, D)
    rv = ref_v.transpose(0, 2, 1, 3).reshape(NB * bs, Hkv, D)
    rk[slots[ok]] = k[ok]
    rv[slots[ok]] = v[ok]
    ref_k = rk.reshape(NB, bs, Hkv, D).transpose(0, 2, 1, 3)
    ref_v = rv.reshape(NB, bs, Hkv, D).transpose(0, 2, 1, 3)
    oracle.reshape_and_cache(k, v, kc, vc, slots, bs)
    assert np.array_equal(kc, ref_k) and np.array_equal(vc, ref_v)


def test_copy_blocks_matches_fancy_indexing():
    rng = np.random.default_rng(17)
    layers = [rng.integers(0, 65535, (10, 2, 16, 8)).astype(np.uint16) for _ in range(3)]
    mapping = np.array([[1, 7], [4, 2], [1, 9]], np.int64)
    ref = [c.copy() for c in layers]
    for c in ref:
        c[mapping[:, 1]] = c[mapping[:, 0]]
    oracle.copy_blocks(layers, mapping)
    for a, b in zip(layers, ref):
        assert np.array_equal(a, b)


# ---------------------------------------------------------------------------
# the pages' printed figures (closed forms) and the byte model the bench uses
# ---------------------------------------------------------------------------
def test_page_figures():
    g = json.load(open(os.path.join(HERE, "golden", "page_figures.json")))
    f = g["opt13b_kv_bytes_per_token"]
    per_token = 2 * f["model"]["layers"] * f["model"]["hidden"] * f["model"]["dtype_bytes"]
    assert per_token == f["value_bytes"]
    assert abs(per_token / 1024 - 800) < 1e-9          # "about 800 KB"
    # the workload byte model at OPT-13B shape (40 heads x 128 = 5120 hidden), one layer
    lay = wl.make_layout("opt13b_f16", num_seqs=2, context_lens=[1, 1])
    assert lay.kv_bytes() // 2 * f["model"]["layers"] == per_token
    p = g["pages_for_2048_tokens_at_128"]
    assert -(-p["tokens"] // p["page_size"]) == p["pages"]
    assert wl.CONFIGS["opt13b_f16"]["block_size"] == g["tokens_per_page_default"]["tokens"]


def test_swap_blocks_matches_fancy_indexing():
    rng = np.random.default_rng(18)
    src = [rng.integers(0, 65535, (9, 2, 16, 8)).astype(np.uint16) for _ in range(2)]
    dst = [rng.integers(0, 65535, (5, 2, 16, 8)).astype(np.uint16) for _ in range(2)]
    mapping = np.array([[8, 0], [3, 4], [0, 2]], np.int64)
    ref = [d.copy() for d in dst]
    for s_, r in zip(src, ref):
        r[mapping[:, 1]] = s_[mapping[:, 0]]
    oracle.swap_blocks(src, dst, mapping)
    for d, r in zip(dst, ref):
        assert np.array_equal(d, r)


# ---------------------------------------------------------------------------
# prefill / chunked prefill
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype,H,Hkv,D,bs,lens,nq", [
    ("bf16", 4, 4, 64, 16, [20, 37, 5], [20, 10, 1]),       # full prefill, a chunk, a decode step
    ("f16", 8, 2, 128, 16, [70, 16, 33], [33, 16, 7]),
    ("bf16", 8, 1, 64, 32, [100, 3], [64, 3]),
])
def test_prefill_matches_causal_sdpa(dtype, H, Hkv, D, bs, lens, nq):
    rng = np.random.default_rng(30)
    q_dec, Kc, Vc, kc, vc, _, tables = build_paged(rng, lens, H, Hkv, D, bs, dtype)
    tdt = wl.torch_dtype(dtype)
    qsl = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    qt = (torch.from_numpy(rng.standard_normal((int(qsl[-1]), H, D)))).to(tdt)
    q_raw = _raw_from_torch(qt, dtype)
    scale = 1.0 / math.sqrt(D)
    got = oracle.paged_prefill(q_raw, kc, vc, tables, np.array(lens, np.int32), qsl, scale, dtype, Hkv, bs)
    G = H // Hkv
    for s, (L, n) in enumerate(zip(lens, nq)):
        K = Kc[s].repeat_interleave(G, 0)
        V = Vc[s].repeat_interleave(G, 0)
        q = qt[qsl[s]:qsl[s + 1]].double().transpose(0, 1)            # [H, n, D]
        # query i at position L - n + i sees keys 0 .. L - n + i
        mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, attn_mask=mask, scale=scale)
        np.testing.assert_allclose(got[qsl[s]:qsl[s + 1]], ref.transpose(0, 1).numpy(), rtol=0, atol=1e-12)
        if n == L:   # a whole prompt is the textbook causal attention
            ref2 = torch.nn.functional.scaled_dot_product_attention(q, K, V, is_causal=True, scale=scale)
            np.testing.assert_allclose(got[qsl[s]:qsl[s + 1]], ref2.transpose(0, 1).numpy(), atol=1e-12)


def test_prefill_large_logits_match_causal_sdpa():
    """Logits of tens (the scale 8x the usual): the oracle's exponentials stay
    finite and it still equals causal SDPA in fp64, the definition the
    logit-jump GPU tests rely on."""
    rng = np.random.default_rng(32)
    lens, nq = [300, 150], [300, 60]
    H, Hkv, D, bs = 4, 2, 64, 16
    _, Kc, Vc, kc, vc, _, tables = build_paged(rng, lens, H, Hkv, D, bs, "bf16")
    qsl = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    qt = torch.from_numpy(rng.standard_normal((int(qsl[-1]), H, D))).to(torch.bfloat16)
    scale = 8.0 / math.sqrt(D)
    got = oracle.paged_prefill(_raw_from_torch(qt, "bf16"), kc, vc, tables, np.array(lens, np.int32), qsl,
                               scale, "bf16", Hkv, bs)
    assert np.isfinite(got).all()
    G = H // Hkv
    for s, (L, n) in enumerate(zip(lens, nq)):
        K, V = Kc[s].repeat_interleave(G, 0), Vc[s].repeat_interleave(G, 0)
        q = qt[qsl[s]:qsl[s + 1]].double().transpose(0, 1)
        mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, attn_mask=mask, scale=scale)
        np.testing.assert_allclose(got[qsl[s]:qsl[s + 1]], ref.transpose(0, 1).numpy(), rtol=0, atol=1e-11)


def test_prefill_last_query_equals_decode():
    """The last query of every sequence attends to the whole context: the decode definition."""
    rng = np.random.default_rng(31)
    lens, nq = [45, 16, 90], [5, 16, 1]
    _, Kc, Vc, kc, vc, _, tables = build_paged(rng, lens, 4, 2, 64, 16, "bf16")
    qsl = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    qt = torch.from_numpy(rng.standard_normal((int(qsl[-1]), 4, 64))).to(torch.bfloat16)
    q_raw = _raw_from_torch(qt, "bf16")
    L = np.array(lens, np.int32)
    pre = oracle.paged_prefill(q_raw, kc, vc, tables, L, qsl, 0.125, "bf16", 2, 16)
    last = q_raw[qsl[1:] - 1]
    dec = oracle.paged_attention(last, kc, vc, tables, L, 0.125, "bf16", 2, 16)
    assert np.array_equal(pre[qsl[1:] - 1], dec)
