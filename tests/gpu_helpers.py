"""Shared pieces of the GPU parity tests: run a decode step through the C ABI
and through the CPU oracle on the same seeded inputs, then compare."""
import numpy as np
import torch

import oracle
import paged_kv_cache_480_b200 as pkv
from paged_kv_cache_480_b200 import workloads as wl


def raw(t, dtype):
    """Raw storage-format numpy array of a tensor (copied to the host)."""
    t = t.detach().contiguous().cpu()
    if dtype == "f32":
        return t.numpy().copy()
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def gpu_step(lay, ten, partition_size=0, write_new=True):
    """reshape_and_cache of the new tokens, then decode; returns (out, error bits)."""
    dev = ten["q"].device
    bt = torch.from_numpy(lay.block_tables).to(dev)
    cl = torch.from_numpy(lay.context_lens).to(dev)
    if write_new:
        sm = torch.from_numpy(lay.slot_mapping).to(dev)
        pkv.reshape_and_cache(ten["k_new"], ten["v_new"], ten["k_cache"], ten["v_cache"], sm)
    out = torch.full_like(ten["q"], float("nan"))
    pkv.paged_attention_decode(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, lay.scale,
                               max_context_len=max(lay.max_context_len, 1),
                               partition_size=partition_size)
    return out, pkv.read_device_errors()


def oracle_step(lay, host, write_new=True):
    """The same step on the host copies (modified in place); returns fp64 output."""
    if write_new:
        oracle.reshape_and_cache(host["k_new"], host["v_new"], host["k_cache"], host["v_cache"],
                                 lay.slot_mapping, lay.block_size)
    return oracle.paged_attention(host["q"], host["k_cache"], host["v_cache"], lay.block_tables,
                                  lay.context_lens, lay.scale, lay.dtype, lay.num_kv_heads,
                                  lay.block_size)


def same_bits(a, b):
    """Bit-for-bit equality (NaN patterns included)."""
    a, b = np.ascontiguousarray(a), np.ascontiguousarray(b)
    return a.shape == b.shape and np.array_equal(a.view(np.uint8), b.view(np.uint8))


def host_copy(ten, dtype):
    return {k: raw(v, dtype) for k, v in ten.items()}


def compare(out_gpu, ref, dtype, rel_bar=None):
    """Apply the parity bar; returns a dict of error statistics.

    fp32: |gpu - ref| <= 1e-5 |ref| + 1e-6 elementwise and max|gpu - ref| /
    max|ref| <= 1e-5.  fp16/bf16: max-abs <= 1e-2 and mean-abs <= 1e-3 (plus
    an optional normwise relative bar).
    """
    got = oracle.decode(raw(out_gpu, dtype), dtype)
    assert got.shape == ref.shape
    assert np.isfinite(got).all(), "non-finite output"
    err = np.abs(got - ref)
    stats = dict(max_abs=float(err.max()), mean_abs=float(err.mean()),
                 rel=float(err.max() / max(np.abs(ref).max(), 1e-30)))
    if dtype == "f32":
        assert (err <= 1e-5 * np.abs(ref) + 1e-6).all(), stats
        assert stats["rel"] <= 1e-5, stats
    else:
        assert stats["max_abs"] <= 1e-2, stats
        assert stats["mean_abs"] <= 1e-3, stats
        if rel_bar is not None:
            assert stats["rel"] <= rel_bar, stats
    return stats


SCALED_REL = 2.0 ** -7


def compare_scaled(out_gpu, ref, dtype):
    """The bar for outputs that reach |v| ~ 4 (one key dominating a row):
    fp32 as in compare; fp16/bf16 |gpu - ref| <= 1e-2 + 2^-7 |ref| per element
    and mean-abs <= 1e-3.  bf16's spacing on [4, 8) is 2^-5, so rounding the
    output alone costs up to 2^-8 |ref|, above the absolute 1e-2 there;
    rounding each softmax weight to the element type (relative 2^-8) moves
    the output by at most 2^-8 times the weighted spread of V around it,
    which the 1e-2 term covers for unit-variance V.  Two such roundings:
    2^-7 |ref| + 1e-2."""
    got = oracle.decode(raw(out_gpu, dtype), dtype)
    assert got.shape == ref.shape
    assert np.isfinite(got).all(), "non-finite output"
    err = np.abs(got - ref)
    if dtype == "f32":
        return compare(out_gpu, ref, dtype)
    stats = dict(max_abs=float(err.max()), mean_abs=float(err.mean()), max_ref=float(np.abs(ref).max()),
                 worst_ratio=float((err / (1e-2 + SCALED_REL * np.abs(ref))).max()))
    assert (err <= 1e-2 + SCALED_REL * np.abs(ref)).all(), stats
    assert stats["mean_abs"] <= 1e-3, stats
    return stats


def check_step(lay, device="cuda", partition_size=0, rel_bar=None):
    """Full parity check of one decode step: caches bit-exact, output within the bar."""
    ten = wl.make_tensors(lay, device=device)
    host = host_copy(ten, lay.dtype)
    out, err = gpu_step(lay, ten, partition_size)
    assert err == 0, f"device check bits {err}"
    ref = oracle_step(lay, host)
    assert same_bits(raw(ten["k_cache"], lay.dtype), host["k_cache"]), "k_cache differs"
    assert same_bits(raw(ten["v_cache"], lay.dtype), host["v_cache"]), "v_cache differs"
    return compare(out, ref, lay.dtype, rel_bar), out, ten
