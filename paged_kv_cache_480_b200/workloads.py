"""Seeded synthetic decode workloads shaped like the pages' configurations.

This module holds none of the method's arithmetic: it draws random values,
length mixes and physical block ids, and builds block tables by plain
free-list bookkeeping.  Both the CUDA path and the CPU oracle consume what it
produces; neither is used here.

Five named workloads (base seed 480 + index):

  tiny_mha_f32   4 seqs, 4 heads, head 64, block 16, pool 64; lengths U{1..100};
                 ids drawn without replacement; q/K/V N(0,1); scale 1/8.
  opt13b_f16     64 seqs, 40 heads, head 128, block 16; lengths U{256..2048};
                 pool 1.1x the blocks in use, shuffled ids; q/K/V N(0,1)/sqrt(128).
  llama7b_bf16   256 seqs, 32 heads, head 128, block 16 or 32; lengths
                 clip(round(exp(ln 700 + 0.8 z)), 16, 4096); pool 90% occupied
                 after random allocate/free churn; q/K/V N(0,1).
  gqa_long_bf16  16 seqs, 64 query heads over 8 KV heads, head 128, block 16;
                 lengths U{16384..32768}; pool 1.1x, shuffled; q/K/V N(0,1).
  cow_bf16       64 prompts x 8 samples, 32 heads, head 128, block 16; prompt
                 prefix 1024 - r, r ~ U{1..15} (so its last block is partly
                 filled and shared); each sample then generates U{0..256}
                 tokens of its own (a scenario, see make_cow_scenario).

One more shape beyond those five, for multi-query attention (every query
head shares one KV head):

  mqa_long_bf16  gqa_long_bf16's sequences and lengths with 64 query heads
                 over a single KV head (seed 480 + 7).

Every slot of the pool that holds no context token is filled with NaN, so a
kernel that reads past a sequence's length or into a free block shows it.
The new token of a decode step (position context_len - 1) is not in the
pool: the step writes it with reshape_and_cache first.
"""
from collections import deque
from dataclasses import dataclass, field
import math

import numpy as np

BASE_SEED = 480

CONFIGS = {
    "tiny_mha_f32": dict(index=0, num_seqs=4, num_heads=4, num_kv_heads=4, head_size=64,
                         block_size=16, dtype="f32"),
    "opt13b_f16": dict(index=1, num_seqs=64, num_heads=40, num_kv_heads=40, head_size=128,
                       block_size=16, dtype="f16"),
    "llama7b_bf16": dict(index=2, num_seqs=256, num_heads=32, num_kv_heads=32, head_size=128,
                         block_size=16, dtype="bf16"),
    "gqa_long_bf16": dict(index=3, num_seqs=16, num_heads=64, num_kv_heads=8, head_size=128,
                          block_size=16, dtype="bf16"),
    "cow_bf16": dict(index=4, num_seqs=512, num_heads=32, num_kv_heads=32, head_size=128,
                     block_size=16, dtype="bf16"),
    "mqa_long_bf16": dict(index=7, num_seqs=16, num_heads=64, num_kv_heads=1, head_size=128,
                          block_size=16, dtype="bf16"),
}

DTYPE_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


@dataclass
class Layout:
    """Integer structure of one decode step (host numpy arrays)."""
    name: str
    dtype: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_size: int
    block_size: int
    num_blocks: int
    scale: float
    value_scale: float          # q/K/V are N(0,1) * value_scale
    context_lens: np.ndarray    # int32 [S]; includes the step's new token
    block_tables: np.ndarray    # int32 [S, MB]; unused entries are -1
    slot_mapping: np.ndarray    # int64 [S]; slot of position context_len - 1 (-1 if empty)
    seed: int
    extra: dict = field(default_factory=dict)

    @property
    def max_blocks_per_seq(self):
        return self.block_tables.shape[1]

    @property
    def max_context_len(self):
        return int(self.context_lens.max()) if self.num_seqs else 0

    def kv_bytes(self):
        """K+V bytes of all context tokens of one layer."""
        return int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads * self.head_size \
            * DTYPE_BYTES[self.dtype] * 2


def _tables_from_ids(context_lens, block_size, ids):
    """Hand out physical ids in order to the sequences' logical blocks."""
    nblk = [-(-int(L) // block_size) for L in context_lens]
    mb = max(1, max(nblk) if nblk else 1)
    tables = np.full((len(context_lens), mb), -1, np.int32)
    pos = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = ids[pos:pos + n]
        pos += n
    return tables


def _slots(context_lens, tables, block_size):
    slots = np.full(len(context_lens), -1, np.int64)
    for s, L in enumerate(context_lens):
        if L > 0:
            t = int(L) - 1
            slots[s] = int(tables[s, t // block_size]) * block_size + t % block_size
    return slots


def churned_free_order(rng, num_blocks, ops, max_alloc=64):
    """Free-list order after random allocate/free churn of decoy requests."""
    free = deque(int(b) for b in rng.permutation(num_blocks))
    live = []
    for _ in range(ops):
        if live and (rng.random() < 0.5 or len(free) < max_alloc):
            blocks = live.pop(int(rng.integers(len(live))))
            free.extend(blocks)
        else:
            n = int(rng.integers(1, max_alloc + 1))
            live.append([free.popleft() for _ in range(n)])
    order = [int(i) for i in rng.permutation(len(live))]
    for i in order:
        free.extend(live[i])
    return list(free)


def make_layout(name, block_size=None, seed=None, num_seqs=None, max_context=None,
                context_lens=None):
    """Build the integer layout of a named workload.

    ``num_seqs`` and ``max_context`` shrink a workload for quick checks
    (lengths are clipped to ``max_context``); ``context_lens`` overrides the
    drawn lengths entirely.
    """
    cfg = dict(CONFIGS[name])
    idx = cfg.pop("index")
    if block_size is not None:
        cfg["block_size"] = block_size
    if num_seqs is not None:
        cfg["num_seqs"] = num_seqs
    seed = BASE_SEED + idx if seed is None else seed
    rng = np.random.default_rng(seed)
    S, bs, D = cfg["num_seqs"], cfg["block_size"], cfg["head_size"]
    scale = 1.0 / math.sqrt(D)
    value_scale = 1.0 / math.sqrt(D) if name == "opt13b_f16" else 1.0

    if context_lens is not None:
        lens = np.asarray(context_lens, np.int64)
        S = cfg["num_seqs"] = len(lens)
    elif name == "tiny_mha_f32":
        lens = rng.integers(1, 101, S)
    elif name == "opt13b_f16":
        lens = rng.integers(256, 2049, S)
    elif name == "llama7b_bf16":
        lens = np.clip(np.round(np.exp(math.log(700.0) + 0.8 * rng.standard_normal(S))), 16, 4096)
    elif name in ("gqa_long_bf16", "mqa_long_bf16"):
        lens = rng.integers(16384, 32769, S)
    elif name == "cow_bf16":
        raise ValueError("cow_bf16 is a scenario: use make_cow_scenario")
    else:
        raise KeyError(name)
    lens = lens.astype(np.int64)
    if max_context is not None:
        lens = np.minimum(lens, max_context)
    lens = lens.astype(np.int32)
    used = int(sum(-(-int(L) // bs) for L in lens))

    if name == "tiny_mha_f32" and num_seqs is None and context_lens is None:
        nb = 64
        ids = rng.choice(nb, size=used, replace=False)
    elif name == "llama7b_bf16":
        nb = max(int(math.ceil(used / 0.9)), used + 1)
        order = churned_free_order(rng, nb, ops=4 * S, max_alloc=min(64, max(1, nb - used)))
        ids = np.asarray(order[:used], np.int64)
    else:
        nb = max(int(math.ceil(1.1 * used)), used + 1)
        ids = rng.permutation(nb)[:used]
    tables = _tables_from_ids(lens, bs, ids)
    return Layout(name=name, dtype=cfg["dtype"], num_seqs=S, num_heads=cfg["num_heads"],
                  num_kv_heads=cfg["num_kv_heads"], head_size=D, block_size=bs, num_blocks=nb,
                  scale=scale, value_scale=value_scale, context_lens=lens, block_tables=tables,
                  slot_mapping=_slots(lens, tables, bs), seed=seed)


def custom_layout(dtype, num_heads, num_kv_heads, head_size, block_size, context_lens, seed,
                  pool_factor=1.5, name="custom", value_scale=1.0):
    """Layout with given lengths and shuffled ids from a pool pool_factor x larger."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(context_lens, np.int32)
    used = int(sum(-(-int(L) // block_size) for L in lens))
    nb = max(int(math.ceil(pool_factor * used)), used + 1)
    ids = rng.permutation(nb)[:used]
    tables = _tables_from_ids(lens, block_size, ids)
    return Layout(name=name, dtype=dtype, num_seqs=len(lens), num_heads=num_heads,
                  num_kv_heads=num_kv_heads, head_size=head_size, block_size=block_size,
                  num_blocks=nb, scale=1.0 / math.sqrt(head_size), value_scale=value_scale,
                  context_lens=lens, block_tables=tables,
                  slot_mapping=_slots(lens, tables, block_size), seed=seed)


# ---------------------------------------------------------------------------
# Tensor values (torch is used as the random-number source and for storage).
# ---------------------------------------------------------------------------
_TORCH_DTYPES = None


def torch_dtype(dtype):
    import torch
    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype]


def _randn(gen, shape, device, value_scale, dtype, chunk=1 << 26):
    """N(0,1)*value_scale drawn in fp32 and rounded once (RNE) to dtype."""
    import torch
    out = torch.empty(shape, dtype=torch_dtype(dtype), device=device)
    flat = out.view(-1)
    for start in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - start)
        x = torch.randn(n, generator=gen, device=device, dtype=torch.float32)
        if value_scale != 1.0:
            x.mul_(value_scale)
        flat[start:start + n].copy_(x)
    return out


def valid_slot_mask(layout, include_new_token=False):
    """bool [NB, bs]: True where a context token lives (new token optional)."""
    mask = np.zeros((layout.num_blocks, layout.block_size), bool)
    bs = layout.block_size
    for s, L in enumerate(layout.context_lens):
        n = int(L) if include_new_token else max(int(L) - 1, 0)
        if n == 0:
            continue
        t = np.arange(n)
        mask[layout.block_tables[s, t // bs], t % bs] = True
    return mask


def make_tensors(layout, device="cpu", pending_new_token=True):
    """q [S,H,D], k_cache/v_cache [NB,Hkv,bs,D], k_new/v_new [S,Hkv,D] on device.

    Slots without a context token hold NaN.  With pending_new_token the
    slot of each sequence's last position is NaN too and the values to
    write there are k_new/v_new; otherwise they are already in the pool.
    """
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(layout.seed * 1000 + 7)
    S, H, Hkv, D = layout.num_seqs, layout.num_heads, layout.num_kv_heads, layout.head_size
    NB, bs = layout.num_blocks, layout.block_size
    vs = layout.value_scale
    q = _randn(gen, (S, H, D), device, vs, layout.dtype)
    k_cache = _randn(gen, (NB, Hkv, bs, D), device, vs, layout.dtype)
    v_cache = _randn(gen, (NB, Hkv, bs, D), device, vs, layout.dtype)
    k_new = _randn(gen, (S, Hkv, D), device, vs, layout.dtype)
    v_new = _randn(gen, (S, Hkv, D), device, vs, layout.dtype)
    mask = valid_slot_mask(layout, include_new_token=not pending_new_token)
    invalid = torch.from_numpy(~mask).to(device)
    nan = float("nan")
    k_cache.masked_fill_(invalid[:, None, :, None], nan)
    v_cache.masked_fill_(invalid[:, None, :, None], nan)
    return dict(q=q, k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new)


def make_tensors_fp8(layout, device="cpu", k_scale=1.0 / 64, v_scale=1.0 / 64, pending_new_token=True):
    """Tensors for an FP8 E4M3 cache: q, k_new, v_new in the layout's dtype;
    k_cache / v_cache uint8 codes of the same N(0,1) draws divided by the
    scales (rounded by torch's float8_e4m3fn cast, values well inside the
    finite range); slots without a context token hold the NaN code 0x7f."""
    import torch
    ten = make_tensors(layout, device=device, pending_new_token=pending_new_token)
    out = dict(q=ten["q"], k_new=ten["k_new"], v_new=ten["v_new"])
    for name, sc in (("k_cache", k_scale), ("v_cache", v_scale)):
        x = ten[name].float()
        nan = torch.isnan(x)
        codes = (x.nan_to_num(0.0) / sc).to(torch.float8_e4m3fn).view(torch.uint8)
        codes[nan] = 0x7f
        out[name] = codes
        del x
    return out


# ---------------------------------------------------------------------------
# Parallel sampling with copy-on-write (cow_bf16).
# ---------------------------------------------------------------------------
@dataclass
class CowScenario:
    dtype: str
    num_prompts: int
    samples: int
    num_heads: int
    num_kv_heads: int
    head_size: int
    block_size: int
    num_blocks: int
    prefix_lens: np.ndarray     # int32 [P]
    own_tokens: np.ndarray      # int32 [P, samples]; tokens each sample adds after the fork
    scale: float
    seed: int

    @property
    def num_seqs(self):
        return self.num_prompts * self.samples

    def final_lens(self):
        return (self.prefix_lens[:, None] + self.own_tokens).reshape(-1).astype(np.int32)

    def max_steps(self):
        return int(self.own_tokens.max()) if self.own_tokens.size else 0

    def active(self, step):
        """Sequence ids (prompt * samples + j) that append a token at this step."""
        return np.nonzero(self.own_tokens.reshape(-1) > step)[0].astype(np.int64)


def make_cow_scenario(seed=None, num_prompts=64, samples=8, prefix=1024, r_max=15, own_max=256,
                      num_heads=32, head_size=128, block_size=16, dtype="bf16"):
    """Prompts share a prefix of prefix - r tokens (r ~ U{1..r_max}; r_max=0
    keeps it at exactly prefix); each sample then adds U{0..own_max} tokens."""
    seed = BASE_SEED + 4 if seed is None else seed
    rng = np.random.default_rng(seed)
    r = rng.integers(1, r_max + 1, num_prompts) if r_max > 0 else np.zeros(num_prompts, np.int64)
    prefix_lens = (prefix - r).astype(np.int32)
    own = rng.integers(0, own_max + 1, (num_prompts, samples)).astype(np.int32)
    bs = block_size
    shared = sum(-(-int(p) // bs) for p in prefix_lens)
    per_sample = sum(-(-(int(p) + int(o)) // bs) for p, row in zip(prefix_lens, own) for o in row)
    num_blocks = shared + per_sample + 16   # enough for every copy and new block
    return CowScenario(dtype=dtype, num_prompts=num_prompts, samples=samples, num_heads=num_heads,
                       num_kv_heads=num_heads, head_size=head_size, block_size=bs,
                       num_blocks=num_blocks, prefix_lens=prefix_lens, own_tokens=own,
                       scale=1.0 / math.sqrt(head_size), seed=seed)


def cow_prefix_kv(sc, device="cpu"):
    """K/V rows of every prompt's prefix, concatenated: [sum prefix, Hkv, D]."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(sc.seed * 1000 + 11)
    T = int(sc.prefix_lens.sum())
    k = _randn(gen, (T, sc.num_kv_heads, sc.head_size), device, 1.0, sc.dtype)
    v = _randn(gen, (T, sc.num_kv_heads, sc.head_size), device, 1.0, sc.dtype)
    return k, v


def cow_step_kv(sc, step, device="cpu"):
    """K/V rows appended at one generation step by the active sequences."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(sc.seed * 1000 + 13 + 7919 * step)
    n = len(sc.active(step))
    k = _randn(gen, (n, sc.num_kv_heads, sc.head_size), device, 1.0, sc.dtype)
    v = _randn(gen, (n, sc.num_kv_heads, sc.head_size), device, 1.0, sc.dtype)
    return k, v


def cow_queries(sc, device="cpu"):
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(sc.seed * 1000 + 17)
    return _randn(gen, (sc.num_seqs, sc.num_heads, sc.head_size), device, 1.0, sc.dtype)


# ---------------------------------------------------------------------------
# Prefill / chunked prefill.
# ---------------------------------------------------------------------------
PREFILL_CONFIGS = {
    # whole prompts of a Llama-2-7B-shaped layer (32 heads, head 128): n = L
    "prefill_llama7b_bf16": dict(index=5, num_seqs=16, num_heads=32, num_kv_heads=32, head_size=128,
                                 block_size=16, dtype="bf16"),
    # the last 512-token chunk of long prompts, 64 query heads over 8 KV heads
    "chunked_gqa_bf16": dict(index=6, num_seqs=16, num_heads=64, num_kv_heads=8, head_size=128,
                             block_size=16, dtype="bf16"),
}


def make_prefill_layout(name=None, seed=None, num_seqs=None, max_context=None, context_lens=None,
                        query_lens=None, dtype=None, num_heads=None, num_kv_heads=None, head_size=None,
                        block_size=None, chunk=512):
    """Integer structure of one prefill call.

    prefill_llama7b_bf16: lengths U{512..2048}, every token a query (n = L).
    chunked_gqa_bf16: contexts U{4096..16384}, the last min(chunk, L)
    tokens are the queries (earlier chunks already in the cache).
    Without a name, context_lens / query_lens and the shape arguments give
    the call directly.  The pool is 1.1x the blocks in use, ids shuffled.
    ``extra['query_lens']`` holds n per sequence and
    ``extra['query_start_loc']`` their prefix sums (int32 [S + 1]).
    """
    if name is not None:
        cfg = dict(PREFILL_CONFIGS[name])
        idx = cfg.pop("index")
        seed = BASE_SEED + idx if seed is None else seed
    else:
        cfg = dict(num_seqs=len(context_lens), num_heads=num_heads, num_kv_heads=num_kv_heads,
                   head_size=head_size, block_size=block_size, dtype=dtype)
        seed = BASE_SEED if seed is None else seed
    for k, v in dict(num_seqs=num_seqs, num_heads=num_heads, num_kv_heads=num_kv_heads,
                     head_size=head_size, block_size=block_size, dtype=dtype).items():
        if v is not None:
            cfg[k] = v
    rng = np.random.default_rng(seed)
    S, bs, D = cfg["num_seqs"], cfg["block_size"], cfg["head_size"]
    if context_lens is not None:
        lens = np.asarray(context_lens, np.int64)
        S = len(lens)
    elif name == "prefill_llama7b_bf16":
        lens = rng.integers(512, 2049, S)
    elif name == "chunked_gqa_bf16":
        lens = rng.integers(4096, 16385, S)
    else:
        raise ValueError("context_lens is required without a named workload")
    if max_context is not None:
        lens = np.minimum(lens, max_context)
    lens = lens.astype(np.int32)
    if query_lens is not None:
        nq = np.asarray(query_lens, np.int32)
    elif name == "chunked_gqa_bf16":
        nq = np.minimum(lens, chunk).astype(np.int32)
    else:
        nq = lens.copy()
    if len(nq) != S or np.any(nq < 0) or np.any(nq > lens):
        raise ValueError("query_lens must satisfy 0 <= n <= context_len per sequence")
    used = int(sum(-(-int(L) // bs) for L in lens))
    nb = max(int(math.ceil(1.1 * used)), used + 1)
    ids = rng.permutation(nb)[:used]
    tables = _tables_from_ids(lens, bs, ids)
    qsl = np.concatenate([[0], np.cumsum(nq.astype(np.int64))]).astype(np.int32)
    return Layout(name=name or "custom_prefill", dtype=cfg["dtype"], num_seqs=S,
                  num_heads=cfg["num_heads"], num_kv_heads=cfg["num_kv_heads"], head_size=D,
                  block_size=bs, num_blocks=nb, scale=1.0 / math.sqrt(D), value_scale=1.0,
                  context_lens=lens, block_tables=tables, slot_mapping=_slots(lens, tables, bs),
                  seed=seed, extra=dict(query_lens=nq, query_start_loc=qsl))


def make_prefill_tensors(layout, device="cpu"):
    """q [T,H,D] and k_cache/v_cache [NB,Hkv,bs,D] with every context token
    (queries' own keys included) already in the pool; other slots NaN."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(layout.seed * 1000 + 19)
    T = int(layout.extra["query_start_loc"][-1])
    H, Hkv, D = layout.num_heads, layout.num_kv_heads, layout.head_size
    NB, bs = layout.num_blocks, layout.block_size
    vs = layout.value_scale
    q = _randn(gen, (T, H, D), device, vs, layout.dtype)
    k_cache = _randn(gen, (NB, Hkv, bs, D), device, vs, layout.dtype)
    v_cache = _randn(gen, (NB, Hkv, bs, D), device, vs, layout.dtype)
    invalid = torch.from_numpy(~valid_slot_mask(layout, include_new_token=True)).to(device)
    k_cache.masked_fill_(invalid[:, None, :, None], float("nan"))
    v_cache.masked_fill_(invalid[:, None, :, None], float("nan"))
    return dict(q=q, k_cache=k_cache, v_cache=v_cache)


def prefill_pairs(layout):
    """(query, key) pairs the causal mask keeps: sum over queries of L - n + i + 1."""
    total = 0
    for L, n in zip(layout.context_lens.astype(np.int64), layout.extra["query_lens"].astype(np.int64)):
        total += n * (L - n) + n * (n + 1) // 2
    return int(total)
