"""CPU oracle for paged decode attention, cache write and copy-on-write.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product library never calls it, and it imports nothing from the product
package: the only thing the two sides share is the seeded inputs.

The arithmetic lives in ``paged_attention_oracle.c`` (plain C, fp64); this
module only marshals numpy arrays into it.  Storage formats are passed as
raw arrays: fp32 as ``float32``, fp16 as ``float16`` or ``uint16`` bits and
bf16 as ``uint16`` bits (the upper half of an IEEE binary32).

Pins (tests/test_oracle_*.py) tie every function to something other than
itself: torch's scaled_dot_product_attention on contiguous K/V, closed forms
(one token, two tokens, equal keys), invariants (physical-block
permutation, weights summing to one), the pages' printed sizes, numpy's
fp16 rounding and a brute-force nearest-value search for bf16 rounding.
The block-manager model in ``block_manager_model.py`` is pinned by
brute-force replay invariants.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32, F16, BF16 = 0, 1, 2
DTYPE_CODES = {"f32": F32, "f16": F16, "bf16": BF16}
ELEM_BYTES = {F32: 4, F16: 2, BF16: 2}

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.orc_paged_attention.argtypes = [P, P, P, P, I, P, I, P, I, I, I, I, I, D, I]
        lib.orc_attention_weights.argtypes = [P, P, P, P, I, P, I, P, I, I, I, I, I, I, D]
        lib.orc_partition_stats.argtypes = [P, P, P, P, P, P, I, P, I, P, I, I, I, I, I, D, I, I, I]
        lib.orc_lse_merge.argtypes = [P, P, P, P, I64, I, I]
        lib.orc_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, I, I64, I64]
        lib.orc_copy_blocks.argtypes = [P, I, P, I, I64]
        lib.orc_swap_blocks.argtypes = [P, P, I, P, I, I64]
        lib.orc_round.argtypes = [P, P, I, I64]
        lib.orc_paged_prefill.argtypes = [P, P, P, P, I, P, I, P, P, I, I, I, I, I, D, I]
        lib.orc_paged_attention_ex.argtypes = [P, P, I, P, P, I, D, D, P, I, P, I, I, I, I, I, D, I]
        lib.orc_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_to_double.restype = D
        lib.orc_double_to_e4m3.argtypes = [D]
        lib.orc_double_to_e4m3.restype = ctypes.c_uint8
        lib.orc_quantize_e4m3.argtypes = [D, ctypes.c_float]
        lib.orc_quantize_e4m3.restype = ctypes.c_uint8
        lib.orc_reshape_and_cache_e4m3.argtypes = [P, P, I, P, P, P, I, I, I, I, I64, I64,
                                                   ctypes.c_float, ctypes.c_float]
        lib.orc_load.argtypes = [P, I, I64]
        lib.orc_load.restype = D
        lib.orc_double_to_f16.argtypes = [D]
        lib.orc_double_to_f16.restype = ctypes.c_uint16
        lib.orc_double_to_bf16.argtypes = [D]
        lib.orc_double_to_bf16.restype = ctypes.c_uint16
        _lib = lib
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def _raw(a, code):
    """Contiguous raw view of a storage-format array."""
    a = np.ascontiguousarray(a)
    want = {F32: (np.float32,), F16: (np.float16, np.uint16, np.int16), BF16: (np.uint16, np.int16)}[code]
    if a.dtype.type not in want:
        raise TypeError(f"array of dtype {a.dtype} does not hold format code {code}")
    return a


def default_threads():
    return len(os.sched_getaffinity(0))


def paged_attention(q, k_cache, v_cache, block_tables, context_lens, scale, dtype, num_kv_heads,
                    block_size, nthreads=None):
    """fp64 decode attention through the block table.  Returns [S, H, D] float64.

    q: [S, H, D]; k_cache, v_cache: [NB, Hkv, bs, D]; block_tables: int32
    [S, MB]; context_lens: int32 [S].  ``dtype`` is "f32", "f16" or "bf16".
    """
    code = DTYPE_CODES[dtype]
    q, kc, vc = _raw(q, code), _raw(k_cache, code), _raw(v_cache, code)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, H, D = q.shape
    assert kc.shape[1] == num_kv_heads and kc.shape[2] == block_size and kc.shape[3] == D
    out = np.zeros((S, H, D), np.float64)
    _load().orc_paged_attention(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), code, _ptr(bt), bt.shape[1],
                                _ptr(cl), S, H, num_kv_heads, D, block_size, float(scale),
                                nthreads or default_threads())
    return out


def attention_weights(q, k_cache, v_cache, block_tables, context_lens, scale, dtype, num_kv_heads,
                      block_size, s, h):
    """Softmax weights of row (s, h): float64 [context_lens[s]]."""
    code = DTYPE_CODES[dtype]
    q, kc, vc = _raw(q, code), _raw(k_cache, code), _raw(v_cache, code)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, H, D = q.shape
    w = np.zeros(max(int(cl[s]), 1), np.float64)
    _load().orc_attention_weights(_ptr(w), _ptr(q), _ptr(kc), _ptr(vc), code, _ptr(bt), bt.shape[1],
                                  _ptr(cl), s, h, H, num_kv_heads, D, block_size, float(scale))
    return w[: int(cl[s])]


def partition_stats(q, k_cache, v_cache, block_tables, context_lens, scale, dtype, num_kv_heads,
                    block_size, partition_size, num_partitions, nthreads=None):
    """Per-partition (acc, m, l): acc [S, H, P, D], m and l [S, H, P], all float64."""
    code = DTYPE_CODES[dtype]
    q, kc, vc = _raw(q, code), _raw(k_cache, code), _raw(v_cache, code)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, H, D = q.shape
    P = num_partitions
    acc = np.zeros((S, H, P, D), np.float64)
    m = np.zeros((S, H, P), np.float64)
    l = np.zeros((S, H, P), np.float64)
    _load().orc_partition_stats(_ptr(acc), _ptr(m), _ptr(l), _ptr(q), _ptr(kc), _ptr(vc), code,
                                _ptr(bt), bt.shape[1], _ptr(cl), S, H, num_kv_heads, D, block_size,
                                float(scale), partition_size, P, nthreads or default_threads())
    return acc, m, l


def lse_merge(acc, m, l):
    """Merge partition statistics: acc [..., P, D], m, l [..., P] -> [..., D]."""
    acc = np.ascontiguousarray(acc, dtype=np.float64)
    m = np.ascontiguousarray(m, dtype=np.float64)
    l = np.ascontiguousarray(l, dtype=np.float64)
    P, D = acc.shape[-2], acc.shape[-1]
    lead = acc.shape[:-2]
    rows = int(np.prod(lead)) if lead else 1
    out = np.zeros(lead + (D,), np.float64)
    _load().orc_lse_merge(_ptr(out), _ptr(acc), _ptr(m), _ptr(l), rows, P, D)
    return out


def round_to(x, dtype):
    """Round fp64 values to a storage format in one RNE step; returns raw array."""
    code = DTYPE_CODES[dtype]
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.float32 if code == F32 else np.uint16)
    _load().orc_round(_ptr(x), _ptr(out), code, x.size)
    return out


def decode(raw, dtype):
    """Widen a raw storage-format array to float64 (exact)."""
    code = DTYPE_CODES[dtype]
    raw = _raw(raw, code)
    if code == F32:
        return raw.astype(np.float64)
    if code == F16:
        return raw.view(np.uint16).view(np.float16).astype(np.float64)
    return (raw.view(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f16_bits(x):
    return _load().orc_double_to_f16(float(x))


def bf16_bits(x):
    return _load().orc_double_to_bf16(float(x))


def reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, block_size):
    """Host scatter of new K/V rows into the caches, in place.

    k, v: [T, Hkv, D] raw storage arrays (contiguous); caches: [NB, Hkv, bs, D].
    """
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    T, Hkv, D = k.shape
    eb = k.dtype.itemsize
    _load().orc_reshape_and_cache(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(sm), T, Hkv,
                                  D, block_size, eb, Hkv * D, Hkv * D)


def copy_blocks(caches, block_mapping):
    """In-place block copies for every cache array in ``caches`` ([NB, ...] each)."""
    bm = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    if len(caches) == 0 or bm.shape[0] == 0:
        return
    block_bytes = caches[0][0].nbytes
    for c in caches:
        assert c.flags.c_contiguous and c[0].nbytes == block_bytes
    arr = (ctypes.c_void_p * len(caches))(*[c.ctypes.data for c in caches])
    _load().orc_copy_blocks(arr, len(caches), _ptr(bm), bm.shape[0], block_bytes)


def swap_blocks(src_pools, dst_pools, block_mapping):
    """dst_pools[c][dst] = src_pools[c][src] for every (src, dst) pair, in place."""
    bm = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    if len(src_pools) == 0 or bm.shape[0] == 0:
        return
    block_bytes = src_pools[0][0].nbytes
    for a in list(src_pools) + list(dst_pools):
        assert a.flags.c_contiguous and a[0].nbytes == block_bytes
    n = len(src_pools)
    sa = (ctypes.c_void_p * n)(*[a.ctypes.data for a in src_pools])
    da = (ctypes.c_void_p * n)(*[a.ctypes.data for a in dst_pools])
    _load().orc_swap_blocks(sa, da, n, _ptr(bm), bm.shape[0], block_bytes)


def e4m3_to_double(code):
    return _load().orc_e4m3_to_double(int(code))


def e4m3_bits(x):
    return _load().orc_double_to_e4m3(float(x))


def quantize_e4m3(x, scale):
    """The cache code of x: e4m3(fp32(x) / fp32(scale))."""
    return _load().orc_quantize_e4m3(float(x), ctypes.c_float(scale))


def paged_attention_fp8(q, qdtype, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                        scale, num_kv_heads, block_size, nthreads=None):
    """fp64 decode attention over E4M3 caches (uint8 codes) times their scales."""
    qc = DTYPE_CODES[qdtype]
    q = _raw(q, qc)
    kc = np.ascontiguousarray(k_cache, dtype=np.uint8)
    vc = np.ascontiguousarray(v_cache, dtype=np.uint8)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, H, D = q.shape
    out = np.zeros((S, H, D), np.float64)
    _load().orc_paged_attention_ex(_ptr(out), _ptr(q), qc, _ptr(kc), _ptr(vc), 3, float(k_scale),
                                   float(v_scale), _ptr(bt), bt.shape[1], _ptr(cl), S, H,
                                   num_kv_heads, D, block_size, float(scale),
                                   nthreads or default_threads())
    return out


def reshape_and_cache_fp8(k, v, src_dtype, k_cache, v_cache, slot_mapping, block_size, k_scale,
                          v_scale):
    """Host quantising scatter into uint8 E4M3 caches, in place."""
    sc = DTYPE_CODES[src_dtype]
    k = _raw(k, sc)
    v = _raw(v, sc)
    assert k_cache.dtype == np.uint8 and k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    T, Hkv, D = k.shape
    _load().orc_reshape_and_cache_e4m3(_ptr(k), _ptr(v), sc, _ptr(k_cache), _ptr(v_cache), _ptr(sm),
                                       T, Hkv, D, block_size, Hkv * D, Hkv * D,
                                       ctypes.c_float(k_scale), ctypes.c_float(v_scale))


def paged_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale, dtype,
                  num_kv_heads, block_size, nthreads=None):
    """fp64 causal prefill attention: q [T, H, D] packed by sequence
    (query_start_loc int32 [S+1]); the last n_s tokens of each sequence's
    context are its queries.  Returns [T, H, D] float64."""
    code = DTYPE_CODES[dtype]
    q, kc, vc = _raw(q, code), _raw(k_cache, code), _raw(v_cache, code)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
    T, H, D = q.shape
    assert qsl[-1] == T
    out = np.zeros((T, H, D), np.float64)
    _load().orc_paged_prefill(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), code, _ptr(bt), bt.shape[1],
                              _ptr(cl), _ptr(qsl), len(cl), H, num_kv_heads, D, block_size,
                              float(scale), nthreads or default_threads())
    return out
