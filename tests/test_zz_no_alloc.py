"""paged_attention_decode_noalloc: the decode step for callers that cannot
allocate device memory (for example a plug-in whose host framework owns all
device memory, or a loop that cannot pay cudaMalloc's synchronisation).

It is called through the C ABI and checked against the regular entry point
(which takes a caller-allocated workspace) on the same inputs, twice in a
row: the fixed scratch keeps the first call's contents, and the second call
must not be disturbed by them.  This file is collected last on purpose.
"""
import pytest
import torch

import paged_kv_cache_480_b200 as pkv
from paged_kv_cache_480_b200 import binding
from paged_kv_cache_480_b200 import workloads as wl
from gpu_helpers import compare, host_copy, oracle_step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_480_b200 import build
    build.build()
    pkv.load_library()


def _inputs():
    # split contexts (up to 8 partitions of 256 tokens), so the scratch holds partials
    lay = wl.custom_layout("bf16", 32, 32, 128, 16, [2000, 1, 257, 1300, 16, 900, 0, 1999], seed=77)
    ten = wl.make_tensors(lay, device="cuda", pending_new_token=False)
    bt = torch.from_numpy(lay.block_tables).cuda()
    cl = torch.from_numpy(lay.context_lens).cuda()
    return lay, ten, bt, cl


def test_noalloc_matches_workspace_entry_point_twice():
    lay, ten, bt, cl = _inputs()
    args = (ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, lay.scale)
    ref = torch.empty_like(ten["q"])
    pkv.paged_attention_decode(ref, *args, max_context_len=lay.max_context_len)
    outs = []
    for _ in range(2):
        out = torch.full_like(ten["q"], float("nan"))
        binding.paged_attention_decode_noalloc(out, *args, max_context_len=lay.max_context_len)
        outs.append(out)
    torch.cuda.synchronize()
    assert pkv.read_device_errors() == 0
    ref_oracle = oracle_step(lay, host_copy(ten, "bf16"), write_new=False)
    compare(ref, ref_oracle, "bf16")
    for out in outs:
        diff = (out.float() - ref.float()).abs()
        assert torch.isfinite(out).all()
        assert diff.max().item() <= 1e-2 and diff.mean().item() <= 1e-3
        compare(out, ref_oracle, "bf16")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lay, ten, bt, cl = _inputs()
    out = torch.zeros_like(ten["q"])
    # a bound of 32768 tokens needs far more than 16 MiB of partials
    big = torch.zeros((lay.num_seqs, 2048), dtype=torch.int32, device="cuda")
    with pytest.raises(binding.PagedKVError) as e:
        binding.paged_attention_decode_noalloc(out, ten["q"], ten["k_cache"], ten["v_cache"], big, cl,
                                               lay.scale, max_context_len=32768)
    assert e.value.status == 6
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0      # nothing was launched
