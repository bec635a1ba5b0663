"""The C-ABI library: it loads, exports every declared entry point, and
rejects bad arguments on the host before any GPU work (CPU only)."""
import ctypes
import os
import re

import numpy as np
import pytest

from paged_kv_cache_480_b200 import binding
from paged_kv_cache_480_b200 import build as pkv_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    pkv_build.build()
    return binding.load_library()


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)
    keywords = {"if", "sizeof", "defined"}
    return sorted(set(n for n in names if n not in keywords))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "paged_attention_decode" in names and "copy_blocks" in names and "reshape_and_cache" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_python_names_cover_the_entry_points():
    """Every public name of the package resolves, and every C entry point that
    computes has a Python function of the same name."""
    import paged_kv_cache_480_b200 as pkv
    for n in pkv.__all__:
        assert getattr(pkv, n) is not None, n
    for n in declared_functions():
        if n.startswith(("paged_attention", "reshape_and_cache", "copy_blocks", "swap_blocks")) \
                and n != "paged_attention_workspace_init":
            assert n in pkv.__all__, f"{n} has no Python name"


def test_status_strings(lib):
    assert lib.pkv_status_string(0) == b"ok"
    assert b"sm_100a" in lib.pkv_version()


def test_partition_and_workspace_sizes(lib):
    # library choice: a per-call size in [8, 16] blocks (in [16, 32] for G >= 4);
    # the call reports the lower end, which sizes the workspace
    assert lib.paged_attention_partition_size(40, 40, 16, 2048, 0) == 128
    assert lib.paged_attention_partition_size(64, 8, 16, 32768, 0) == 256
    assert lib.paged_attention_partition_size(32, 32, 32, 4096, 0) == 256
    assert lib.paged_attention_partition_size(32, 32, 16, 4096, 48) == 48
    assert lib.paged_attention_partition_size(32, 32, 16, 4096, 40) == 0      # not a block multiple
    assert lib.paged_attention_partition_size(32, 32, 16, 4096, 1024) == 0    # > 32 blocks
    small = lib.paged_attention_workspace_size(64, 40, 40, 128, 16, 200, 1, 0)
    big = lib.paged_attention_workspace_size(64, 40, 40, 128, 16, 2048, 1, 0)
    assert 0 < small < big
    # partials: S * parts * H * (D floats + an (m, l) pair), parts at the smallest size
    assert big >= 64 * 16 * 40 * (128 * 4 + 8)
    assert lib.paged_attention_workspace_size(64, 40, 7, 128, 16, 2048, 1, 0) == 0   # G not integral
    # any integral group: G = 12 (slices of 8 + 4 heads) and MQA (G = 64) need the same
    # partials per query head as MHA
    assert lib.paged_attention_workspace_size(64, 48, 4, 128, 16, 2048, 1, 0) >= 64 * 8 * 48 * (128 * 4 + 8)
    assert lib.paged_attention_workspace_size(64, 64, 1, 128, 16, 2048, 1, 0) >= 64 * 8 * 64 * (128 * 4 + 8)
    assert lib.paged_attention_workspace_size(64, 40, 40, 96, 16, 2048, 1, 0) == 0   # head_size 96


def _decode(lib, **kw):
    args = dict(out=16, q=16, k=16, v=16, bt=16, cl=16, scale=0.1, hkv=4, bs=16, s=2, h=4, d=64, nb=8,
                mb=4, ctx=64, dtype=2, ps=0, ws=16, wsb=1 << 20)
    args.update(kw)
    P = ctypes.c_void_p
    return lib.paged_attention_decode(
        P(args["out"]), P(args["q"]), P(args["k"]), P(args["v"]), P(args["bt"]), P(args["cl"]),
        args["scale"], args["hkv"], args["bs"], args["s"], args["h"], args["d"], args["nb"], args["mb"],
        args["ctx"], args["dtype"], args["ps"], P(args["ws"]), args["wsb"], None)


def test_decode_rejects_bad_arguments_before_launch(lib):
    # (pointers are fake; every call below fails validation before any CUDA call)
    assert _decode(lib, out=0) == 1                 # null pointer
    assert _decode(lib, d=96) == 2                  # head size
    assert _decode(lib, bs=8) == 2                  # block size
    assert _decode(lib, h=6, hkv=4) == 2            # heads not a multiple
    assert _decode(lib, dtype=5) == 2               # dtype
    assert _decode(lib, q=8) == 1                   # misaligned q
    assert _decode(lib, ctx=100) == 1               # context beyond the table (4 blocks x 16)
    assert _decode(lib, ps=40) == 1                 # partition not a block multiple
    assert _decode(lib, ws=0) == 6                  # no workspace
    assert _decode(lib, wsb=64) == 6                # workspace too small
    assert _decode(lib, scale=float("nan")) == 1


def test_cache_ops_reject_bad_arguments(lib):
    P = ctypes.c_void_p
    # reshape_and_cache: misaligned key, token stride too small, bad dtype
    assert lib.reshape_and_cache(P(8), P(16), P(16), P(16), P(16), 4, 2, 64, 16, 8, 128, 128, 2, None) == 1
    assert lib.reshape_and_cache(P(16), P(16), P(16), P(16), P(16), 4, 2, 64, 16, 8, 64, 128, 2, None) == 1
    assert lib.reshape_and_cache(P(16), P(16), P(16), P(16), P(16), 4, 2, 64, 16, 8, 128, 128, 9, None) == 2
    assert lib.reshape_and_cache(None, None, None, None, None, 0, 2, 64, 16, 8, 128, 128, 2, None) == 0
    # copy_blocks: block bytes not a multiple of 16, too many layers, null caches
    arr = (ctypes.c_void_p * 1)(16)
    assert lib.copy_blocks(arr, arr, 1, P(16), 2, 8, 1000, None) == 1
    assert lib.copy_blocks(arr, arr, 300, P(16), 2, 8, 1024, None) == 1
    null = (ctypes.c_void_p * 1)(0)
    assert lib.copy_blocks(null, null, 1, P(16), 2, 8, 1024, None) == 1
    assert lib.copy_blocks(arr, arr, 1, P(16), 0, 8, 1024, None) == 0   # nothing to copy


def _prefill(lib, **kw):
    args = dict(out=16, q=16, k=16, v=16, bt=16, cl=16, qsl=16, scale=0.1, t=40, s=2, h=4, hkv=4, d=64,
                bs=16, nb=8, mb=4, mq=32, dtype=2)
    args.update(kw)
    P = ctypes.c_void_p
    return lib.paged_attention_prefill(
        P(args["out"]), P(args["q"]), P(args["k"]), P(args["v"]), P(args["bt"]), P(args["cl"]),
        P(args["qsl"]), args["scale"], args["t"], args["s"], args["h"], args["hkv"], args["d"], args["bs"],
        args["nb"], args["mb"], args["mq"], args["dtype"], None)


def test_prefill_rejects_bad_arguments_before_launch(lib):
    assert _prefill(lib, out=0) == 1                 # null pointer
    assert _prefill(lib, qsl=0) == 1
    assert _prefill(lib, dtype=0) == 2               # f32: no tensor-core kernel
    assert _prefill(lib, d=96) == 2                  # head size
    assert _prefill(lib, bs=8) == 2                  # block size
    assert _prefill(lib, h=256, hkv=1) == 2          # G = 256: a query tile holds at most 128 rows
    assert _prefill(lib, q=8) == 1                   # misaligned q
    assert _prefill(lib, qsl=18) == 1                # misaligned int32 array
    assert _prefill(lib, mq=41) == 1                 # bound above the token count
    assert _prefill(lib, mq=0) == 1                  # tokens but no queries bound
    assert _prefill(lib, scale=float("nan")) == 1
    assert _prefill(lib, scale=-0.1) == 1
    assert _prefill(lib, scale=0.0) == 1
    assert _prefill(lib, nb=1 << 27, hkv=4) == 2     # pool rows beyond 2^31
    assert _prefill(lib, t=0, mq=0) == 0             # nothing to do


def test_wait_limit_setting(lib):
    assert lib.pkv_set_wait_limit(0) == 0
    assert lib.pkv_set_wait_limit(1 << 33) == 1      # beyond 32 bits
    assert lib.pkv_set_wait_limit(-1) == 0           # back to the default
