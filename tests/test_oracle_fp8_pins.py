"""Pins of the oracle's FP8 (E4M3) cache arithmetic (CPU only): widening of
all 256 codes against torch's float8_e4m3fn, rounding against a brute-force
nearest-even search (and torch inside the finite range), saturation, the
fp32 quotient of the cache write, and attention over an E4M3 cache against
torch SDPA on the dequantised contiguous K/V."""
import math

import numpy as np
import pytest
import torch

import oracle


def _table():
    codes = np.arange(256, dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    return codes, vals


def test_decode_all_codes_matches_torch():
    codes, vals = _table()
    got = np.array([oracle.e4m3_to_double(c) for c in codes])
    nan = np.isnan(vals)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2      # 0x7f and 0xff
    assert np.array_equal(got[~nan], vals[~nan])
    assert got[0x7e] == 448.0 and got[1] == 2.0 ** -9


def test_rounding_is_nearest_even_with_saturation():
    codes, vals = _table()
    keep = np.isfinite(vals) & (codes < 0x80)
    pc, pv = codes[keep], vals[keep]
    order = np.argsort(pv)
    pc, pv = pc[order], pv[order]
    rng = np.random.default_rng(20)
    xs = np.concatenate([np.exp2(rng.uniform(-12, 9.5, 3000)), (pv[:-1] + pv[1:]) / 2, pv,
                         [0.0, 2.0 ** -10, 3 * 2.0 ** -11, 447.9, 448.0, 455.0, 464.0, 1e6]])
    for x in xs:
        if x >= 448.0:
            want = 0x7e                                  # saturate
        else:
            i = np.searchsorted(pv, x)
            cands = [j for j in (i - 1, i) if 0 <= j < len(pv)]
            d = [abs(pv[j] - x) for j in cands]
            best = [cands[k] for k in range(len(cands)) if d[k] == min(d)]
            if len(best) > 1:
                best = [j for j in best if pc[j] % 2 == 0]
            want = int(pc[best[0]])
        assert oracle.e4m3_bits(x) == want, (x, oracle.e4m3_bits(x), want)
        assert oracle.e4m3_bits(-x) == want | 0x80
    assert oracle.e4m3_bits(float("nan")) == 0x7f


def test_rounding_matches_torch_in_range():
    rng = np.random.default_rng(21)
    x = np.concatenate([rng.standard_normal(20000) * 40, rng.uniform(-448, 448, 5000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_bits(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_quantize_divides_in_fp32():
    rng = np.random.default_rng(22)
    for _ in range(2000):
        x = float(np.float32(rng.standard_normal() * 10))
        sc = float(np.float32(rng.uniform(0.01, 3)))
        want = oracle.e4m3_bits(float(np.float32(x) / np.float32(sc)))
        assert oracle.quantize_e4m3(x, sc) == want


def test_fp8_attention_matches_sdpa_on_dequantised_kv():
    rng = np.random.default_rng(23)
    S, H, Hkv, D, bs = 3, 8, 2, 128, 16
    lens = [40, 1, 77]
    k_scale, v_scale = 0.05, 0.03
    nblk = [-(-L // bs) for L in lens]
    NB = sum(nblk) + 2
    ids = rng.permutation(NB)
    tables = np.full((S, max(nblk)), -1, np.int32)
    kc = np.full((NB, Hkv, bs, D), 0x7f, np.uint8)                  # NaN codes outside the context
    vc = kc.copy()
    q = torch.from_numpy(rng.standard_normal((S, H, D))).to(torch.bfloat16)
    outs = []
    pos = 0
    for s, L in enumerate(lens):
        tables[s, :nblk[s]] = ids[pos:pos + nblk[s]]
        pos += nblk[s]
        Kc = rng.integers(0, 256, (Hkv, L, D)).astype(np.uint8)
        Vc = rng.integers(0, 256, (Hkv, L, D)).astype(np.uint8)
        Kc[(Kc & 0x7f) == 0x7f] = 0x10                               # no NaN codes inside
        Vc[(Vc & 0x7f) == 0x7f] = 0x11
        for t in range(L):
            kc[tables[s, t // bs], :, t % bs] = Kc[:, t]
            vc[tables[s, t // bs], :, t % bs] = Vc[:, t]
        K = torch.from_numpy(Kc).view(torch.float8_e4m3fn).double() * k_scale
        V = torch.from_numpy(Vc).view(torch.float8_e4m3fn).double() * v_scale
        K = K.repeat_interleave(H // Hkv, 0)
        V = V.repeat_interleave(H // Hkv, 0)
        o = torch.nn.functional.scaled_dot_product_attention(q[s].double()[:, None, :], K, V, scale=0.1)
        outs.append(o[:, 0, :].numpy())
    got = oracle.paged_attention_fp8(q.view(torch.int16).numpy().view(np.uint16), "bf16", kc, vc,
                                     k_scale, v_scale, tables, np.array(lens, np.int32), 0.1, Hkv, bs)
    np.testing.assert_allclose(got, np.stack(outs), rtol=0, atol=1e-12)


def test_fp8_cache_write_matches_elementwise_quantisation():
    rng = np.random.default_rng(24)
    T, Hkv, D, bs, NB = 5, 2, 64, 16, 4
    k = torch.from_numpy(rng.standard_normal((T, Hkv, D)) * 3).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((T, Hkv, D)) * 3).to(torch.bfloat16)
    kc = np.zeros((NB, Hkv, bs, D), np.uint8)
    vc = np.zeros_like(kc)
    slots = np.array([3, 17, -1, 63, 40], np.int64)
    oracle.reshape_and_cache_fp8(k.view(torch.int16).numpy().view(np.uint16),
                                 v.view(torch.int16).numpy().view(np.uint16), "bf16", kc, vc, slots,
                                 bs, 0.02, 0.5)
    kf, vf = k.float().numpy(), v.float().numpy()
    for i, sl in enumerate(slots):
        if sl < 0:
            continue
        for g in range(Hkv):
            want_k = [oracle.e4m3_bits(float(np.float32(x) / np.float32(0.02))) for x in kf[i, g]]
            want_v = [oracle.e4m3_bits(float(np.float32(x) / np.float32(0.5))) for x in vf[i, g]]
            assert list(kc[sl // bs, g, sl % bs]) == want_k
            assert list(vc[sl // bs, g, sl % bs]) == want_v
    assert (kc[2 // bs, :, 2 % bs] == 0).all()          # untouched slot
