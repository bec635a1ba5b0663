"""Host-side logic of bench.py on CPU: the multi-rank reduction (world size 2
over gloo, as torchrun runs it on GPUs with NCCL), the whole-job aggregate,
the byte model, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from paged_kv_cache_480_b200 import workloads as wl  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(times[rank], world, "cpu")
        out[rank] = ms
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_world_size_2_gloo():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    times = [3.25, 7.5]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 7.5          # every rank sees the slowest rank's time


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(4.0, 1, "cpu") == 4.0


def test_whole_job_value_scales_with_replicas():
    one = bench.whole_job_value(1e9, 1.0, 1)
    assert one == pytest.approx(1000.0)                 # 1 GB per ms = 1000 GB/s
    assert bench.whole_job_value(1e9, 1.0, 8) == pytest.approx(8 * one)


def test_decode_byte_model():
    lay = wl.custom_layout("bf16", 8, 2, 128, 16, [0, 1, 17, 100], seed=1)
    lens = np.array([0, 1, 17, 100])
    kv = lens.sum() * 2 * 128 * 2 * 2
    qo = 2 * 4 * 8 * 128 * 2
    tables = (-(-lens // 16)).sum() * 4
    assert bench.decode_bytes(lay) == kv + qo + tables + 4 * 4
    assert bench.cache_write_bytes(lay) == 4 * (4 * 2 * 128 * 2 + 8)


def test_reference_arm_json_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_mha_f32", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("{")][-1]
    d = json.loads(line)
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "tiny_mha_f32"


def test_reference_arm_other_ranks_do_nothing():
    class A:
        workload = "tiny_mha_f32"
    assert bench.run_reference(A(), rank=1, world=2) is None


def test_tensor_peak_follows_the_sampled_clock():
    burst, kind, b2 = bench.tensor_peak({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0})
    assert "burst" in kind and burst == b2
    sus, kind, b3 = bench.tensor_peak({"sm_mhz": 1300.0, "sm_max_mhz": 1965.0})
    assert "sustained" in kind and sus <= b3
    assert "burst" in bench.tensor_peak(None)[1]


def test_prefill_flop_model():
    """Causal pairs: every query i of n at position L - n + i sees L - n + i + 1 keys."""
    lay = wl.make_prefill_layout(context_lens=[5, 300, 7], query_lens=[5, 17, 1], dtype="bf16",
                                 num_heads=4, num_kv_heads=2, head_size=64, block_size=16)
    brute = sum(L - n + i + 1 for L, n in [(5, 5), (300, 17), (7, 1)] for i in range(n))
    assert wl.prefill_pairs(lay) == brute
    assert bench.prefill_flops(lay) == 4 * 64 * 4 * brute
    slots = bench.prefill_slots(lay)
    assert len(slots) == 23
    # the slot of sequence 1's last query is its last context position
    L, bs = 300, 16
    assert slots[5 + 16] == lay.block_tables[1, (L - 1) // bs] * bs + (L - 1) % bs


def test_default_steps_depend_on_the_arm(monkeypatch):
    """No --steps: 200 timed steps on the GPU arms (so that a 0.25 ms decode
    step still leaves many clock samples inside the timed region), 20 for the
    CPU reference arm; an explicit --steps is kept as given."""
    cases = [([], 200), (["--impl", "reference"], 20), (["--measure", "prefill"], 200),
             (["--steps", "7"], 7), (["--impl", "reference", "--steps", "3"], 3)]
    for argv, steps in cases:
        monkeypatch.setattr(sys, "argv", ["bench.py"] + argv)
        assert bench.parse().steps == steps, argv


def test_clock_summary_median_and_reasons():
    clk = bench.ClockSampler(0)
    clk.samples = [(1965.0, []), (1900.0, ["sw_power_cap"]), (1965.0, [])]
    clk.max_mhz = 1965.0
    s = clk.summary()
    assert s["sm_mhz"] == 1965.0 and s["samples"] == 3 and s["reasons"] == ["sw_power_cap"]
    empty = bench.ClockSampler(0).summary()
    assert empty["samples"] == 0 and empty["sm_mhz"] is None
