"""Benchmark of the paged decode hot path on B200.

One step = one pass of the whole hot path over one batch: copy-on-write block
copies (when the workload forks), the cache write of each sequence's new
token, and paged decode attention (plus its log-sum-exp merge when contexts
are split).  Inputs are seeded and synthetic, resident in HBM when timing
starts; the K/V of a step (4.3 GB for the default workload, the 7B-shaped
layer of 256 sequences) is far larger than the 126 MB L2, so no explicit
flush is needed.  The same line also reports, under "targets", the decode
call of the long-context GQA and MQA workloads timed the same way.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the CPU oracle as the reference arm)

Prints one JSON line (rank 0).  Multi-GPU runs are independent replicas, one
process per GPU (torchrun); time is the max over ranks.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attn: achieved HBM GB/s (% of B200 peak), µs/step, seqs/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 200 on the GPU, so that the clock samples taken during the "
                         "timed region are many even for a 0.25 ms step; 20 for the CPU reference arm)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama7b_bf16")
    ap.add_argument("--block-size", type=int, default=None)
    ap.add_argument("--partition-size", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--measure", default="decode", choices=["decode", "swap", "prefill", "cache_ops"],
                    help="swap: swap_blocks between the GPU pool and a pinned host pool; "
                         "prefill: cache write + causal prefill attention (--workload "
                         "prefill_llama7b_bf16 or chunked_gqa_bf16); cache_ops: reshape_and_cache and "
                         "copy_blocks alone, GB/s of bytes read + written")
    ap.add_argument("--kv-cache", default="auto", choices=["auto", "fp8"],
                    help="fp8: E4M3 cache written by reshape_and_cache_fp8kv, read by the fp8 decode")
    ap.add_argument("--fused", action="store_true",
                    help="cache write fused into the decode (paged_attention_decode_append)")
    ap.add_argument("--no-targets", action="store_true",
                    help="skip the decode calls of the long-context GQA / MQA workloads")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = 20 if args.impl == "reference" else 200
    return args


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


FALLBACK_BF16_TFLOPS = 1590.0


FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def tensor_peak(clocks=None):
    """Dense bf16 tensor throughput (TFLOP/s) measured by cuBLAS: the burst
    figure, or the sustained one (seconds of back-to-back GEMMs under the
    power cap) when the SM clock sampled during the timed region sat below
    90% of its maximum, i.e. the kernel ran power-capped like that loop."""
    burst, sustained, kind = FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            burst, kind = float(d["bf16_tflops"]), "measured"
            sustained = float(d.get("bf16_tflops_sustained", burst))
    capped = bool(clocks and clocks.get("sm_mhz") and clocks.get("sm_max_mhz")
                  and clocks["sm_mhz"] < 0.9 * clocks["sm_max_mhz"])
    if capped:
        return sustained, f"{kind} cuBLAS bf16 sustained (SM clock {clocks['sm_mhz']:.0f} MHz under load)", burst
    return burst, f"{kind} cuBLAS bf16 burst", burst


# ---------------------------------------------------------------------------
# workload and byte model
# ---------------------------------------------------------------------------
def decode_bytes(lay, cache_bytes=None):
    """Algorithmic bytes of one decode call: K+V of every context token, q
    and out, the block-table entries read and the context lengths.
    cache_bytes: bytes per cache element (default: the model's dtype)."""
    from paged_kv_cache_480_b200.workloads import DTYPE_BYTES
    dt = DTYPE_BYTES[lay.dtype]
    cb = dt if cache_bytes is None else cache_bytes
    lens = lay.context_lens.astype(np.int64)
    kv = int(lens.sum()) * lay.num_kv_heads * lay.head_size * cb * 2
    qo = 2 * lay.num_seqs * lay.num_heads * lay.head_size * dt
    tables = int((-(-lens // lay.block_size)).sum()) * 4
    return kv + qo + tables + 4 * lay.num_seqs


def cache_write_bytes(lay, cache_bytes=None):
    """reshape_and_cache of one token per sequence: read k, v; write them; read slots."""
    from paged_kv_cache_480_b200.workloads import DTYPE_BYTES
    dt = DTYPE_BYTES[lay.dtype]
    cb = dt if cache_bytes is None else cache_bytes
    n = lay.num_kv_heads * lay.head_size
    return lay.num_seqs * (2 * n * dt + 2 * n * cb + 8)


FP8_SCALES = (1.0 / 64, 1.0 / 64)


def build_workload(name, block_size, device, fp8=False):
    from paged_kv_cache_480_b200 import workloads as wl
    if name == "cow_bf16":
        if fp8:
            raise SystemExit("--kv-cache fp8 runs the decode workloads only")
        return build_cow_state(device)
    lay = wl.make_layout(name, block_size=block_size)
    if fp8:
        ten = wl.make_tensors_fp8(lay, device=device, k_scale=FP8_SCALES[0], v_scale=FP8_SCALES[1])
    else:
        ten = wl.make_tensors(lay, device=device)
    return lay, ten, None


def build_cow_state(device):
    """The parallel-sampling workload at its first generation step: prompts
    prefilled and forked, so the step's first own token of every writing
    sample triggers copy-on-write of the shared partial block."""
    import torch
    import paged_kv_cache_480_b200 as pkv
    from paged_kv_cache_480_b200 import workloads as wl
    sc = wl.make_cow_scenario()
    NB, Hkv, bs, D = sc.num_blocks, sc.num_kv_heads, sc.block_size, sc.head_size
    bm = pkv.BlockManager(NB, bs, free_order=np.random.default_rng(sc.seed + 1).permutation(NB))
    kc = torch.full((NB, Hkv, bs, D), float("nan"), dtype=torch.bfloat16, device=device)
    vc = torch.full_like(kc, float("nan"))
    pk, pv = wl.cow_prefix_kv(sc, device)
    pos = 0
    for p in range(sc.num_prompts):
        root, L = p * sc.samples, int(sc.prefix_lens[p])
        bm.allocate(root, L)
        t = np.arange(L)
        slots = bm.block_table(root)[t // bs].astype(np.int64) * bs + t % bs
        pkv.reshape_and_cache(pk[pos:pos + L], pv[pos:pos + L], kc, vc, torch.from_numpy(slots).to(device))
        pos += L
        for j in range(1, sc.samples):
            bm.fork(root, root + j)
    seqs = np.arange(sc.num_seqs)
    slots, pairs = bm.append_slots(seqs)     # every sample writes one token this step
    lens = (sc.prefix_lens[:, None] + np.ones_like(sc.own_tokens)).reshape(-1).astype(np.int32)
    MB = int(-(-lens.max() // bs))
    tables, glens = bm.fill_tables(seqs, MB)
    assert np.array_equal(glens, lens)
    lay = wl.Layout(name="cow_bf16", dtype="bf16", num_seqs=sc.num_seqs, num_heads=sc.num_heads,
                    num_kv_heads=Hkv, head_size=D, block_size=bs, num_blocks=NB, scale=sc.scale,
                    value_scale=1.0, context_lens=lens, block_tables=tables, slot_mapping=slots,
                    seed=sc.seed, extra=dict(cow_pairs=pairs))
    gen = torch.Generator(device=device).manual_seed(sc.seed)
    k_new = torch.randn((sc.num_seqs, Hkv, D), generator=gen, device=device).to(torch.bfloat16)
    v_new = torch.randn((sc.num_seqs, Hkv, D), generator=gen, device=device).to(torch.bfloat16)
    ten = dict(q=wl.cow_queries(sc, device), k_cache=kc, v_cache=vc, k_new=k_new, v_new=v_new)
    return lay, ten, pairs


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, polled through
    NVML every 0.25 ms on a background thread while the timed region runs
    (it only reads; no setting is changed; a decode step is ~0.25 ms, so a
    20-step region still gets ~20 samples).  Samples are kept only between
    mark_start() and mark_end(), i.e. under load."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, device_index):
        import threading
        self.samples, self.max_mhz, self.error = [], None, None
        self._stop = threading.Event()
        self._on = threading.Event()
        self._thread = None
        self.device_index = device_index

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
        for i in range(pynvml.nvmlDeviceGetCount()):
            h = pynvml.nvmlDeviceGetHandleByIndex(i)
            u = pynvml.nvmlDeviceGetUUID(h)
            u = u.decode() if isinstance(u, bytes) else u
            if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                return h
        return pynvml.nvmlDeviceGetHandleByIndex(self.device_index)

    def _run(self):
        import pynvml
        try:
            h = self._handle()
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            masks = {k: getattr(pynvml, v) for k, v in self.REASONS.items() if hasattr(pynvml, v)}
            while not self._stop.is_set():
                if self._on.is_set():
                    mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((float(mhz), [k for k, m in masks.items() if bits & m]))
                self._stop.wait(0.00025)
        except Exception as e:              # NVML missing: report no samples
            self.error = str(e)[:120]

    def __enter__(self):
        import threading
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def mark_start(self):
        self._on.set()

    def mark_end(self):
        self._on.clear()

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml", "error": self.error}
        reasons = sorted({r for _, rs in self.samples for r in rs})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml, 0.25 ms polling"}


def kernel_source_sha():
    h = hashlib.sha256()
    for f in ("decode_kernel.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_480_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def prefill_source_sha():
    h = hashlib.sha256()
    for f in ("prefill_kernel.cuh", "prefill.cu", "tc05.cuh", "tc_softmax.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_480_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_prefill_traffic(workload):
    """DRAM bytes per prefill launch from the committed ncu capture, if it
    still matches the kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "prefill_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        e = json.load(f).get(workload)
    if not e or e.get("source_sha") != prefill_source_sha():
        return None
    return e.get("bytes_per_call")


def profiled_traffic(workload, block_size, fp8=False):
    """DRAM bytes per decode call from a committed ncu summary, if it still
    matches the kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    key = f"{workload}/bs{block_size}" + ("/fp8" if fp8 else "")
    e = d.get(key)
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return e.get("bytes_per_call")


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(lay, host, budget_s, max_seqs=None, threads=None, fp8=False):
    """Time the oracle on leading sequences of the workload (bounded), repeating
    until ~budget_s of work; returns (GB/s, seconds, bytes, seqs, threads).
    fp8: the caches hold E4M3 codes (FP8_SCALES) and the oracle's FP8 decode runs."""
    import oracle
    S = lay.num_seqs if max_seqs is None else min(max_seqs, lay.num_seqs)
    sub = lambda a: a[:S]
    threads = threads or oracle.default_threads()
    from paged_kv_cache_480_b200 import workloads as wl
    sublay = wl.Layout(**{**lay.__dict__, "num_seqs": S, "context_lens": sub(lay.context_lens),
                          "block_tables": sub(lay.block_tables), "slot_mapping": sub(lay.slot_mapping)})
    nbytes = decode_bytes(sublay, 1 if fp8 else None)
    total_t, total_b, reps = 0.0, 0, 0
    while total_t < budget_s or reps == 0:
        t0 = time.perf_counter()
        if fp8:
            oracle.paged_attention_fp8(host["q"][:S], lay.dtype, host["k_cache"], host["v_cache"], *FP8_SCALES,
                                       sublay.block_tables, sublay.context_lens, lay.scale, lay.num_kv_heads,
                                       lay.block_size, nthreads=threads)
        else:
            oracle.paged_attention(host["q"][:S], host["k_cache"], host["v_cache"], sublay.block_tables,
                                   sublay.context_lens, lay.scale, lay.dtype, lay.num_kv_heads,
                                   lay.block_size, nthreads=threads)
        total_t += time.perf_counter() - t0
        total_b += nbytes
        reps += 1
        if total_t > 2 * budget_s:
            break
    return total_b / total_t / 1e9, total_t, total_b, S * reps, threads


def host_arrays(ten, dtype):
    import torch
    out = {}
    for k in ("q", "k_cache", "v_cache"):
        t = ten[k].contiguous().cpu()
        if t.dtype == torch.uint8:                  # E4M3 codes
            out[k] = t.numpy()
        else:
            out[k] = t.numpy() if dtype == "f32" else t.view(torch.int16).numpy().view(np.uint16)
    return out


# ---------------------------------------------------------------------------
# the arms
# ---------------------------------------------------------------------------
def run_reference(args, rank, world):
    """The CPU oracle, as it stands, timed on this host's cores (rank 0 only)."""
    if rank != 0:
        return None
    from paged_kv_cache_480_b200 import workloads as wl
    name = args.workload
    if name == "cow_bf16":
        return {"impl": "reference", "unavailable": "the oracle reference arm runs the decode workloads only"}
    lay = wl.make_layout(name, block_size=args.block_size)
    ten = wl.make_tensors(lay, device="cpu", pending_new_token=False)
    host = host_arrays(ten, lay.dtype)
    # bounded sample per step: enough sequences for ~1-3 s of oracle work
    probe_gbs, _, _, _, _ = oracle_sample(lay, host, 0.0, max_seqs=max(1, lay.num_seqs // 16))
    per_step = max(1, min(lay.num_seqs, int(2.0 * probe_gbs * 1e9 / max(decode_bytes(lay) / lay.num_seqs, 1))))
    for _ in range(args.warmup):
        oracle_sample(lay, host, 0.0, max_seqs=per_step)
    times, nbytes = [], 0
    for _ in range(args.steps):
        gbs, t, b, seqs, threads = oracle_sample(lay, host, 0.0, max_seqs=per_step)
        times.append(t)
        nbytes = b
    ms = 1e3 * sum(times) / len(times)
    value = nbytes / (sum(times) / len(times)) / 1e9
    sample = f"{per_step} of {lay.num_seqs} sequences (all heads) per step"
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": name, "block_size": lay.block_size,
                                            "sample": sample},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def max_over_ranks(ms, world, device):
    """The slowest rank's time (ms): every rank takes part in one all-reduce."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(step_bytes, ms_step, world):
    """Aggregate throughput (GB/s) of `world` replicas each moving step_bytes per step."""
    return world * step_bytes / (ms_step * 1e-3) / 1e9


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import paged_kv_cache_480_b200 as pkv

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    pkv.load_library()
    fp8 = args.kv_cache == "fp8"
    if fp8 and args.fused:
        raise SystemExit("--fused works with caches of the model's dtype")
    cb = 1 if fp8 else None
    lay, ten, pairs = build_workload(args.workload, args.block_size, device, fp8)
    S, H, Hkv, D, bs = lay.num_seqs, lay.num_heads, lay.num_kv_heads, lay.head_size, lay.block_size
    max_ctx = lay.max_context_len
    bt = torch.from_numpy(lay.block_tables).to(device)
    cl = torch.from_numpy(lay.context_lens).to(device)
    sm = torch.from_numpy(lay.slot_mapping).to(device)
    pairs_d = torch.from_numpy(np.ascontiguousarray(pairs)).to(device) if pairs is not None and len(pairs) else None
    out = torch.empty_like(ten["q"])
    code = {"f32": 0, "f16": 1, "bf16": 2}[lay.dtype]
    ps = args.partition_size
    need = pkv.paged_attention_workspace_size(S, H, Hkv, D, bs, max_ctx, code, ps)
    ws = torch.zeros(need, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    nparts = pkv.paged_attention_partition_size(H, Hkv, bs, max_ctx, ps)
    split = max_ctx > nparts
    launches_per_step = (1 if args.fused else 2) + (1 if split else 0) + (1 if pairs_d is not None else 0)

    ev = []

    def step(record=False):
        if pairs_d is not None:
            pkv.copy_blocks([ten["k_cache"]], [ten["v_cache"]], pairs_d, stream=stream)
        if fp8:
            pkv.reshape_and_cache_fp8kv(ten["k_new"], ten["v_new"], ten["k_cache"], ten["v_cache"], sm,
                                        *FP8_SCALES, stream=stream)
        elif not args.fused:
            pkv.reshape_and_cache(ten["k_new"], ten["v_new"], ten["k_cache"], ten["v_cache"], sm,
                                  stream=stream)
        if record:
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
        if fp8:
            pkv.paged_attention_decode_fp8kv(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl,
                                             lay.scale, *FP8_SCALES, max_context_len=max_ctx,
                                             partition_size=ps, workspace=ws, stream=stream)
        elif args.fused:
            pkv.paged_attention_decode_append(out, ten["q"], ten["k_new"], ten["v_new"], ten["k_cache"],
                                              ten["v_cache"], sm, bt, cl, lay.scale,
                                              max_context_len=max_ctx, partition_size=ps,
                                              workspace=ws, stream=stream)
        else:
            pkv.paged_attention_decode(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, lay.scale,
                                       max_context_len=max_ctx, partition_size=ps, workspace=ws,
                                       stream=stream)
        if record:
            b.record(stream)
            ev.append((a, b))

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(device)
    assert pkv.read_device_errors() == 0
    if world > 1:
        dist.barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        time.sleep(0.05)
        torch.cuda.synchronize(device)
        clk.mark_start()
        start.record(stream)
        for _ in range(args.steps):
            step(record=True)
        end.record(stream)
        torch.cuda.synchronize(device)
        clk.mark_end()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(start.elapsed_time(end), world, device)
    dec_ms = [a.elapsed_time(b) for a, b in ev]
    errors = pkv.read_device_errors()

    step_bytes = decode_bytes(lay, cb) + cache_write_bytes(lay, cb)
    if pairs_d is not None:
        step_bytes += 2 * len(pairs) * 2 * Hkv * bs * D * 2
    ms_step = ms_total / args.steps
    value = whole_job_value(step_bytes, ms_step, world)

    result = None
    if rank == 0:
        peak, peak_kind = peaks()
        dec_avg = sum(dec_ms) / len(dec_ms)
        achieved = decode_bytes(lay, cb) / (dec_avg * 1e-3) / 1e9
        kname = "paged_attention_decode_append (fused cache write + decode" if args.fused else \
            "paged_attention_decode_fp8kv (decode" if fp8 else "paged_attention_decode (decode"
        roof = {"kernel": kname + (" + lse merge)" if split else ")"),
                "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": peak_kind,
                "frac_of_nominal_8TBs": achieved / NOMINAL_HBM_GBS,
                "traffic": profiled_traffic(lay.name, bs, fp8),
                "algorithmic_bytes": decode_bytes(lay, cb),
                "avg_call_us": dec_avg * 1e3}
        result = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
                  "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                  "us_per_step": ms_step * 1e3, "seqs_per_s": world * S / (ms_step * 1e-3),
                  "pct_of_peak": 100 * value / world / peak,
                  "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                  "dtype": lay.dtype + ("/fp8-e4m3 cache" if fp8 else ""), "data": "synthetic",
                  "config": {"workload": lay.name, "num_seqs": S, "num_heads": H,
                             "num_kv_heads": Hkv, "head_size": D, "block_size": bs,
                             "num_blocks": lay.num_blocks, "max_context_len": max_ctx,
                             "mean_context_len": float(lay.context_lens.mean()),
                             "partition_size": nparts, "split_context": split,
                             "cow_pairs": 0 if pairs is None else int(len(pairs)),
                             "step_bytes": step_bytes, "fused_cache_write": bool(args.fused),
                             "kv_cache": "fp8-e4m3" if fp8 else lay.dtype,
                             "l2": f"inputs larger than L2: {lay.kv_bytes() / 1e9:.2f} GB of K/V per step",
                             "parallelism": f"replicas x{world}"},
                  "roofline": roof, "gpu_launches": launches_per_step * args.steps,
                  "clocks": clk.summary(), "device_errors": errors}
        if not args.no_e2e:
            result["e2e"] = run_e2e(args, lay, ten, pairs, device, ws, step_bytes, fp8)
        if not args.no_cpu_baseline and world == 1:
            host = host_arrays(ten, lay.dtype)
            what = "fp64 oracle (FP8 decode)" if fp8 else "fp64 oracle"
            gbs, t, b, seqs, threads = oracle_sample(lay, host, 10.0,
                                                     max_seqs=max(1, lay.num_seqs // 8), fp8=fp8)
            gbs1, t1, _, seqs1, _ = oracle_sample(lay, host, 5.0, max_seqs=max(1, lay.num_seqs // 32),
                                                  threads=1, fp8=fp8)
            result["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                      "sample": f"{what} over the first {max(1, lay.num_seqs // 8)} "
                                                f"sequences, repeated: {seqs} sequence-passes in {t:.1f} s",
                                      "value_1core": gbs1,
                                      "sample_1core": f"first {max(1, lay.num_seqs // 32)} sequences on one "
                                                      f"thread: {seqs1} sequence-passes in {t1:.1f} s"}
        if not args.no_targets and not args.fused:
            del ten, out, ws
            torch.cuda.empty_cache()
            result["targets"] = decode_targets(args, device, local_rank, fp8,
                                               exclude=lay.name if args.partition_size == 0 else None)
    return result


TARGET_WORKLOADS = ("gqa_long_bf16", "mqa_long_bf16")


def decode_targets(args, device, local_rank, fp8, exclude=None):
    """The decode call of the long-context workloads (GQA: 64 query heads
    over 8 KV heads; MQA: 64 over 1; 16 sequences of 16K-32K tokens), each
    timed like the main line's: one reshape_and_cache + decode per step, CUDA
    events around the decode call on its stream, args.steps calls after
    args.warmup, SM clocks sampled meanwhile."""
    import torch
    import paged_kv_cache_480_b200 as pkv
    from paged_kv_cache_480_b200 import workloads as wl
    peak, peak_kind = peaks()
    cb = 1 if fp8 else None
    res = {}
    for name in TARGET_WORKLOADS:
        if name == exclude:
            continue
        lay, ten, _ = build_workload(name, None, device, fp8)
        S, H, Hkv, D, bs = lay.num_seqs, lay.num_heads, lay.num_kv_heads, lay.head_size, lay.block_size
        max_ctx = lay.max_context_len
        bt = torch.from_numpy(lay.block_tables).to(device)
        cl = torch.from_numpy(lay.context_lens).to(device)
        sm = torch.from_numpy(lay.slot_mapping).to(device)
        out = torch.empty_like(ten["q"])
        need = pkv.paged_attention_workspace_size(S, H, Hkv, D, bs, max_ctx, {"f32": 0, "f16": 1, "bf16": 2}[lay.dtype])
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
        stream = torch.cuda.current_stream(device)
        ev = []

        def step(record=False):
            if fp8:
                pkv.reshape_and_cache_fp8kv(ten["k_new"], ten["v_new"], ten["k_cache"], ten["v_cache"], sm,
                                            *FP8_SCALES, stream=stream)
            else:
                pkv.reshape_and_cache(ten["k_new"], ten["v_new"], ten["k_cache"], ten["v_cache"], sm, stream=stream)
            if record:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
            if fp8:
                pkv.paged_attention_decode_fp8kv(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, lay.scale,
                                                 *FP8_SCALES, max_context_len=max_ctx, workspace=ws, stream=stream)
            else:
                pkv.paged_attention_decode(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, lay.scale,
                                           max_context_len=max_ctx, workspace=ws, stream=stream)
            if record:
                b.record(stream)
                ev.append((a, b))

        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize(device)
        with ClockSampler(local_rank) as clk:
            time.sleep(0.05)
            clk.mark_start()
            for _ in range(args.steps):
                step(record=True)
            torch.cuda.synchronize(device)
            clk.mark_end()
        errors = pkv.read_device_errors()
        dec = sum(a.elapsed_time(b) for a, b in ev) / len(ev)
        nbytes = decode_bytes(lay, cb)
        gbs = nbytes / (dec * 1e-3) / 1e9
        res[name] = {"avg_call_us": dec * 1e3, "achieved": gbs, "unit": "GB/s", "peak": peak, "peak_kind": peak_kind,
                     "frac": gbs / peak, "frac_of_nominal_8TBs": gbs / NOMINAL_HBM_GBS,
                     "algorithmic_bytes": nbytes, "seqs_per_s": S / (dec * 1e-3),
                     "shape": f"{S} seqs, {H} q heads / {Hkv} KV heads, D {D}, bs {bs}, "
                              f"mean context {float(lay.context_lens.mean()):.0f}",
                     "kv_cache": "fp8-e4m3" if fp8 else lay.dtype, "calls": len(ev),
                     "clocks": clk.summary(), "device_errors": errors}
        del ten, out, ws
        torch.cuda.empty_cache()
    return res


def run_e2e(args, lay, ten, pairs, device, ws, step_bytes, fp8=False):
    """Same step through the C ABI with the step's inputs in pinned host
    memory.  The inputs (q, new K/V, slots, tables, lengths, CoW pairs) sit
    in one pinned staging buffer and go to the device in one copy; the
    output comes back in one copy; both are inside the timed region every
    step.  The step (copy, library calls, copy back) is captured once in a
    CUDA graph and replayed per step, as a serving loop would; the eager
    version (one Python call sequence per step) is reported beside it."""
    import torch
    import paged_kv_cache_480_b200 as pkv
    parts = [("q", ten["q"]), ("k", ten["k_new"]), ("v", ten["v_new"]),
             ("sm", torch.from_numpy(lay.slot_mapping)), ("bt", torch.from_numpy(lay.block_tables)),
             ("cl", torch.from_numpy(lay.context_lens))]
    if pairs is not None and len(pairs):
        parts.append(("pairs", torch.from_numpy(np.ascontiguousarray(pairs))))
    offs, total = {}, 0
    for name, t in parts:
        offs[name] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_buf = torch.empty(total, dtype=torch.uint8).pin_memory()
    d_buf = torch.empty(total, dtype=torch.uint8, device=device)

    def view(buf, name, t):
        n = t.numel() * t.element_size()
        return buf[offs[name]:offs[name] + n].view(t.dtype).view(t.shape)

    for name, t in parts:
        view(h_buf, name, t).copy_(t.detach().cpu())
    d = {name: view(d_buf, name, t) for name, t in parts}
    out = torch.empty_like(ten["q"])
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    max_ctx = lay.max_context_len
    h2d = sum(t.numel() * t.element_size() for _, t in parts)
    d2h = h_out.numel() * h_out.element_size()

    def body(stream):
        d_buf.copy_(h_buf, non_blocking=True)
        if "pairs" in d:
            pkv.copy_blocks([ten["k_cache"]], [ten["v_cache"]], d["pairs"], stream=stream)
        if fp8:
            pkv.reshape_and_cache_fp8kv(d["k"], d["v"], ten["k_cache"], ten["v_cache"], d["sm"], *FP8_SCALES,
                                        stream=stream)
            pkv.paged_attention_decode_fp8kv(out, d["q"], ten["k_cache"], ten["v_cache"], d["bt"], d["cl"],
                                             lay.scale, *FP8_SCALES, max_context_len=max_ctx, workspace=ws,
                                             stream=stream)
        elif args.fused:
            pkv.paged_attention_decode_append(out, d["q"], d["k"], d["v"], ten["k_cache"], ten["v_cache"],
                                              d["sm"], d["bt"], d["cl"], lay.scale,
                                              max_context_len=max_ctx, workspace=ws, stream=stream)
        else:
            pkv.reshape_and_cache(d["k"], d["v"], ten["k_cache"], ten["v_cache"], d["sm"], stream=stream)
            pkv.paged_attention_decode(out, d["q"], ten["k_cache"], ten["v_cache"], d["bt"], d["cl"],
                                       lay.scale, max_context_len=max_ctx, workspace=ws, stream=stream)
        h_out.copy_(out, non_blocking=True)

    n_steps = max(args.steps, 200)

    def timed(run, sync):
        """Median wall time of one step (host sync every step; the median
        keeps host scheduling jitter out of a ~0.3 ms step)."""
        for _ in range(3):
            run()
            sync()
        times = []
        for _ in range(n_steps):
            t0 = time.perf_counter()
            run()
            sync()
            times.append(time.perf_counter() - t0)
        return statistics.median(times)

    stream = torch.cuda.current_stream(device)
    eager = timed(lambda: body(stream), stream.synchronize)
    result = {"value": step_bytes / eager / 1e9, "unit": "GB/s", "us_per_step": eager * 1e6,
              "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "mode": "eager",
              "timing": f"median of {n_steps} wall-clock steps, each ending in a host sync"}
    try:
        cap = torch.cuda.Stream(device)
        cap.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(cap):
            body(cap)                       # warm the capture stream
            cap.synchronize()
            with torch.cuda.graph(graph, stream=cap):
                body(cap)
        stream.wait_stream(cap)
        replay = timed(graph.replay, torch.cuda.synchronize)
        assert pkv.read_device_errors() == 0
        result.update({"value": step_bytes / replay / 1e9, "us_per_step": replay * 1e6,
                       "mode": "cuda graph of the step, replayed per step",
                       "eager_value": step_bytes / eager / 1e9, "eager_us_per_step": eager * 1e6})
        del graph
    except Exception as e:                  # capture unavailable: keep the eager number
        result["graph_error"] = str(e)[:200]
    return result


# ---------------------------------------------------------------------------
# prefill: cache write of the chunk's K/V + causal prefill attention
# ---------------------------------------------------------------------------
PREFILL_METRIC = "paged prefill attn: achieved TFLOP/s (causal pairs x 4 x head_size x heads)"


def prefill_flops(lay):
    from paged_kv_cache_480_b200 import workloads as wl
    return 4 * lay.head_size * lay.num_heads * wl.prefill_pairs(lay)


def prefill_slots(lay):
    """Cache slots of every sequence's query tokens (positions L - n .. L - 1)."""
    bs = lay.block_size
    out = []
    for s, (L, n) in enumerate(zip(lay.context_lens, lay.extra["query_lens"])):
        pos = np.arange(int(L) - int(n), int(L))
        out.append(lay.block_tables[s, pos // bs].astype(np.int64) * bs + pos % bs)
    return np.concatenate(out) if out else np.zeros(0, np.int64)


def prefill_workload(name, device):
    from paged_kv_cache_480_b200 import workloads as wl
    if name not in wl.PREFILL_CONFIGS:
        name = "prefill_llama7b_bf16"
    lay = wl.make_prefill_layout(name)
    ten = wl.make_prefill_tensors(lay, device=device)
    slots = prefill_slots(lay)
    # the chunk's own K/V as the step writes them: the values already at those
    # slots, so repeated steps leave the cache unchanged
    sl = torch_from(slots, device)
    nb, hkv, bs, d = ten["k_cache"].shape
    flat_k = ten["k_cache"].permute(0, 2, 1, 3).reshape(nb * bs, hkv, d)
    flat_v = ten["v_cache"].permute(0, 2, 1, 3).reshape(nb * bs, hkv, d)
    ten["k_new"] = flat_k[sl].contiguous()
    ten["v_new"] = flat_v[sl].contiguous()
    ten["slots"] = sl
    return lay, ten


def torch_from(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def prefill_oracle_sample(lay, host, budget_s, nseq):
    """Oracle prefill over the first nseq sequences (all heads), repeated to
    ~budget_s; returns (TFLOP/s, seconds, flops, passes, threads)."""
    import oracle
    from paged_kv_cache_480_b200 import workloads as wl
    qsl = lay.extra["query_start_loc"]
    sub = wl.Layout(**{**lay.__dict__, "num_seqs": nseq, "context_lens": lay.context_lens[:nseq],
                       "block_tables": lay.block_tables[:nseq], "slot_mapping": lay.slot_mapping[:nseq],
                       "extra": {"query_lens": lay.extra["query_lens"][:nseq],
                                 "query_start_loc": qsl[:nseq + 1]}})
    flops = prefill_flops(sub)
    threads = oracle.default_threads()
    q = host["q"][:int(qsl[nseq])]
    total_t, reps = 0.0, 0
    while total_t < budget_s or reps == 0:
        t0 = time.perf_counter()
        oracle.paged_prefill(q, host["k_cache"], host["v_cache"], sub.block_tables, sub.context_lens,
                             qsl[:nseq + 1], lay.scale, lay.dtype, lay.num_kv_heads, lay.block_size,
                             nthreads=threads)
        total_t += time.perf_counter() - t0
        reps += 1
    return flops * reps / total_t / 1e12, total_t, flops * reps, reps, threads


def run_prefill(args, rank, world, local_rank):
    import torch
    import paged_kv_cache_480_b200 as pkv
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    pkv.load_library()
    lay, ten = prefill_workload(args.workload, device)
    bt = torch_from(lay.block_tables, device)
    cl = torch_from(lay.context_lens, device)
    qsl = torch_from(lay.extra["query_start_loc"], device)
    mq = int(lay.extra["query_lens"].max())
    T = int(lay.extra["query_start_loc"][-1])
    out = torch.empty_like(ten["q"])
    stream = torch.cuda.current_stream(device)
    ev = []

    def step(record=False):
        pkv.reshape_and_cache(ten["k_new"], ten["v_new"], ten["k_cache"], ten["v_cache"], ten["slots"],
                              stream=stream)
        if record:
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
        pkv.paged_attention_prefill(out, ten["q"], ten["k_cache"], ten["v_cache"], bt, cl, qsl, lay.scale,
                                    max_query_len=mq, stream=stream)
        if record:
            b.record(stream)
            ev.append((a, b))

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(device)
    assert pkv.read_device_errors() == 0
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        time.sleep(0.05)
        torch.cuda.synchronize(device)
        clk.mark_start()
        start.record(stream)
        for _ in range(args.steps):
            step(record=True)
        end.record(stream)
        torch.cuda.synchronize(device)
        clk.mark_end()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    ms_total = max_over_ranks(start.elapsed_time(end), world, device)
    errors = pkv.read_device_errors()
    flops = prefill_flops(lay)
    ms_step = ms_total / args.steps
    if rank != 0:
        return None
    clocks = clk.summary()
    peak, peak_kind, burst = tensor_peak(clocks)
    k_ms = [a.elapsed_time(b) for a, b in ev]
    k_avg = sum(k_ms) / len(k_ms)
    achieved = flops / (k_avg * 1e-3) / 1e12
    kv_bytes = lay.kv_bytes()
    result = {"metric": PREFILL_METRIC, "value": world * flops / (ms_step * 1e-3) / 1e12, "unit": "TFLOP/s",
              "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
              "tokens_per_s": world * T / (ms_step * 1e-3), "higher_is_better": True, "scaling": "weak",
              "vs_baseline": None, "dtype": lay.dtype, "data": "synthetic",
              "config": {"workload": lay.name, "num_seqs": lay.num_seqs, "query_tokens": T,
                         "num_heads": lay.num_heads, "num_kv_heads": lay.num_kv_heads,
                         "head_size": lay.head_size, "block_size": lay.block_size,
                         "num_blocks": lay.num_blocks, "max_context_len": lay.max_context_len,
                         "max_query_len": mq, "causal_pairs": int(flops // (4 * lay.head_size * lay.num_heads)),
                         "flops_per_step": flops,
                         "l2": f"inputs larger than L2: {kv_bytes / 1e9:.2f} GB of K/V in the cache",
                         "parallelism": f"replicas x{world}"},
              "roofline": {"kernel": "paged_attention_prefill", "bound": "tensor", "achieved": achieved,
                           "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "peak_kind": peak_kind,
                           "frac_of_burst": achieved / burst, "traffic": profiled_prefill_traffic(lay.name),
                           "traffic_note": "DRAM bytes per launch, one-pass ncu capture with a cold L2",
                           "algorithmic_flops": flops,
                           "avg_call_us": k_avg * 1e3},
              "gpu_launches": 2 * args.steps, "clocks": clocks, "device_errors": errors}
    if not args.no_e2e:
        result["e2e"] = run_prefill_e2e(args, lay, ten, device, flops)
    if not args.no_cpu_baseline and world == 1:
        host = host_arrays(ten, lay.dtype)
        tf, t, f, reps, threads = prefill_oracle_sample(lay, host, 10.0, 1)
        result["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                  "sample": f"fp64 oracle prefill of the first sequence (all heads), "
                                            f"{reps} passes in {t:.1f} s"}
    return result


def run_prefill_e2e(args, lay, ten, device, flops):
    """The prefill step through the C ABI with its inputs (q, the chunk's
    K/V, slots, tables, lengths, query offsets) in pinned host memory, one
    copy in and the output out every step; a CUDA graph of the step replayed."""
    import torch
    import paged_kv_cache_480_b200 as pkv
    parts = [("q", ten["q"]), ("k", ten["k_new"]), ("v", ten["v_new"]), ("sm", ten["slots"]),
             ("bt", torch.from_numpy(lay.block_tables)), ("cl", torch.from_numpy(lay.context_lens)),
             ("qsl", torch.from_numpy(lay.extra["query_start_loc"]))]
    offs, total = {}, 0
    for name, t in parts:
        offs[name] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_buf = torch.empty(total, dtype=torch.uint8).pin_memory()
    d_buf = torch.empty(total, dtype=torch.uint8, device=device)

    def view(buf, name, t):
        n = t.numel() * t.element_size()
        return buf[offs[name]:offs[name] + n].view(t.dtype).view(t.shape)

    for name, t in parts:
        view(h_buf, name, t).copy_(t.detach().cpu())
    d = {name: view(d_buf, name, t) for name, t in parts}
    out = torch.empty_like(ten["q"])
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    mq = int(lay.extra["query_lens"].max())
    h2d = sum(t.numel() * t.element_size() for _, t in parts)
    d2h = h_out.numel() * h_out.element_size()

    def body(stream):
        d_buf.copy_(h_buf, non_blocking=True)
        pkv.reshape_and_cache(d["k"], d["v"], ten["k_cache"], ten["v_cache"], d["sm"], stream=stream)
        pkv.paged_attention_prefill(out, d["q"], ten["k_cache"], ten["v_cache"], d["bt"], d["cl"], d["qsl"],
                                    lay.scale, max_query_len=mq, stream=stream)
        h_out.copy_(out, non_blocking=True)

    n_steps = max(args.steps, 50)

    def timed(run, sync):
        for _ in range(3):
            run()
            sync()
        times = []
        for _ in range(n_steps):
            t0 = time.perf_counter()
            run()
            sync()
            times.append(time.perf_counter() - t0)
        return statistics.median(times)

    stream = torch.cuda.current_stream(device)
    eager = timed(lambda: body(stream), stream.synchronize)
    result = {"value": flops / eager / 1e12, "unit": "TFLOP/s", "us_per_step": eager * 1e6,
              "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "mode": "eager",
              "timing": f"median of {n_steps} wall-clock steps, each ending in a host sync"}
    try:
        cap = torch.cuda.Stream(device)
        cap.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(cap):
            body(cap)
            cap.synchronize()
            with torch.cuda.graph(graph, stream=cap):
                body(cap)
        stream.wait_stream(cap)
        replay = timed(graph.replay, torch.cuda.synchronize)
        assert pkv.read_device_errors() == 0
        result.update({"value": flops / replay / 1e12, "us_per_step": replay * 1e6,
                       "mode": "cuda graph of the step, replayed per step",
                       "eager_value": flops / eager / 1e12, "eager_us_per_step": eager * 1e6})
        del graph
    except Exception as e:
        result["graph_error"] = str(e)[:200]
    return result


def run_prefill_reference(args, rank, world):
    """The oracle prefill, as it stands, on this host's cores (rank 0 only)."""
    if rank != 0:
        return None
    from paged_kv_cache_480_b200 import workloads as wl
    name = args.workload if args.workload in wl.PREFILL_CONFIGS else "prefill_llama7b_bf16"
    lay = wl.make_prefill_layout(name)
    ten = wl.make_prefill_tensors(lay, device="cpu")
    host = host_arrays(ten, lay.dtype)
    for _ in range(args.warmup):
        prefill_oracle_sample(lay, host, 0.0, 1)
    times, flops = [], 0
    for _ in range(args.steps):
        tf, t, f, reps, threads = prefill_oracle_sample(lay, host, 0.0, 1)
        times.append(t)
        flops = f
    avg = sum(times) / len(times)
    value = flops / avg / 1e12
    sample = "the first sequence of the workload (all heads) per step"
    return {"impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": avg * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": name, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_cache_ops(args, rank, world, local_rank):
    """reshape_and_cache and copy_blocks timed alone, in GB/s of the bytes
    they read and write (algorithmic: K and V rows and slots; source and
    destination blocks).  L2 is flushed before every timed call (a 256 MB
    write), each call timed with its own CUDA events."""
    import torch
    import paged_kv_cache_480_b200 as pkv
    from paged_kv_cache_480_b200 import workloads as wl
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    pkv.load_library()
    stream = torch.cuda.current_stream(device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def timed(fn, reps=20):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e-3)
        return statistics.median(ts)

    lines = []

    def line(metric, nbytes, t, cfg):
        lines.append({"metric": metric, "value": nbytes / t / 1e9, "unit": "GB/s", "n_gpus": world,
                      "steps": 20, "warmup": 3, "ms_per_step": t * 1e3, "higher_is_better": True,
                      "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                      "config": {"workload": cfg, "bytes": nbytes, "l2": "flushed before every call"},
                      "roofline": {"bound": "hbm", "achieved": nbytes / t / 1e9, "peak": peaks()[0],
                                   "unit": "GB/s", "frac": nbytes / t / 1e9 / peaks()[0],
                                   "peak_kind": peaks()[1]},
                      "gpu_launches": 20})

    # reshape_and_cache: one decode step of the 7B-shaped workload, and a prefill's chunk
    lay = wl.make_layout("llama7b_bf16")
    ten = wl.make_tensors(lay, device=device)
    sm = torch.from_numpy(lay.slot_mapping).to(device)
    row = lay.num_kv_heads * lay.head_size * 2
    t = timed(lambda: pkv.reshape_and_cache(ten["k_new"], ten["v_new"], ten["k_cache"], ten["v_cache"], sm,
                                            stream=stream))
    line("reshape_and_cache GB/s (read + write)", lay.num_seqs * (4 * row + 8), t,
         f"llama7b_bf16 decode step: {lay.num_seqs} tokens x 32 heads x 128")
    del ten
    play, pten = prefill_workload("prefill_llama7b_bf16", device)
    T = int(play.extra["query_start_loc"][-1])
    t = timed(lambda: pkv.reshape_and_cache(pten["k_new"], pten["v_new"], pten["k_cache"], pten["v_cache"],
                                            pten["slots"], stream=stream), reps=10)
    line("reshape_and_cache GB/s (read + write)", T * (4 * row + 8), t,
         f"prefill_llama7b_bf16 chunk write: {T} tokens x 32 heads x 128")
    del pten
    # copy_blocks: the first fork step of the parallel-sampling workload
    lay, ten, pairs = build_cow_state(device)
    pd = torch.from_numpy(np.ascontiguousarray(pairs)).to(device)
    blk = lay.num_kv_heads * lay.block_size * lay.head_size * 2
    t = timed(lambda: pkv.copy_blocks([ten["k_cache"]], [ten["v_cache"]], pd, stream=stream))
    line("copy_blocks GB/s (read + write)", len(pairs) * 2 * 2 * blk, t,
         f"cow_bf16 first fork step: {len(pairs)} pairs x (K, V) x {blk // 1024} KB")
    assert pkv.read_device_errors() == 0
    return lines


def run_swap(args, rank, world, local_rank):
    """swap_blocks throughput, device <-> pinned host, against a contiguous
    pinned copy of the same size measured in the same run (the host link's
    ceiling).  Pools shaped like the OPT-13B layer (40 heads x 16 x 128 fp16 =
    160 KB per block per cache), K and V, 512 scattered blocks each way."""
    import torch
    import paged_kv_cache_480_b200 as pkv
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    shape = (40, 16, 128)
    NBd, NBh, n = 2048, 1024, 512
    kd = torch.randn((NBd,) + shape, device=device).half()
    vd = torch.randn((NBd,) + shape, device=device).half()
    kh = torch.empty((NBh,) + shape, dtype=torch.float16).pin_memory()
    vh = torch.empty_like(kh).pin_memory()
    rng = np.random.default_rng(480)
    out_map = torch.from_numpy(np.stack([rng.choice(NBd, n, replace=False),
                                         rng.choice(NBh, n, replace=False)], 1).astype(np.int64)).to(device)
    in_map = torch.from_numpy(np.stack([rng.choice(NBh, n, replace=False),
                                        rng.choice(NBd, n, replace=False)], 1).astype(np.int64)).to(device)
    nbytes = 2 * n * kd[0].numel() * 2
    stream = torch.cuda.current_stream(device)

    def timed(fn):
        for _ in range(max(args.warmup, 3)):
            fn()
        torch.cuda.synchronize(device)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(device)
        return a.elapsed_time(b) / args.steps * 1e-3

    t_out = timed(lambda: pkv.swap_blocks([kd, vd], [kh, vh], out_map, stream=stream))
    t_in = timed(lambda: pkv.swap_blocks([kh, vh], [kd, vd], in_map, stream=stream))
    big_h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    big_d = torch.empty(nbytes, dtype=torch.uint8, device=device)
    t_h2d = timed(lambda: big_d.copy_(big_h, non_blocking=True))
    t_d2h = timed(lambda: big_h.copy_(big_d, non_blocking=True))
    assert pkv.read_device_errors() == 0
    res = []
    for name, t, tp in (("device->host", t_out, t_d2h), ("host->device", t_in, t_h2d)):
        ach, peak = nbytes / t / 1e9, nbytes / tp / 1e9
        res.append({"metric": f"swap_blocks {name} GB/s", "value": ach, "unit": "GB/s", "n_gpus": world,
                    "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
                    "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
                    "data": "synthetic",
                    "config": {"workload": "swap 512 scattered blocks x (K, V) of 160 KB", "bytes": nbytes},
                    "roofline": {"bound": "host link", "achieved": ach, "peak": peak, "unit": "GB/s",
                                 "frac": ach / peak,
                                 "peak_kind": "contiguous pinned copy of the same bytes, this run"},
                    "gpu_launches": args.steps})
    return res


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_prefill_reference(args, rank, world) if args.measure == "prefill" else \
            run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.measure in ("swap", "cache_ops"):
            fn = run_swap if args.measure == "swap" else run_cache_ops
            for line in fn(args, rank, world, local_rank):
                if rank == 0:
                    print(json.dumps(line), flush=True)
            return
        if args.measure == "prefill":
            res = run_prefill(args, rank, world, local_rank)
        else:
            res = run_ours(args, rank, world, local_rank)
        if res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
