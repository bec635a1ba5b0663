"""Host model of the tensor-core decode's work split and of the merge's slot
lookup (decode_tc_kernel.cuh, merge_kernel.cuh), on the CPU.

The kernel gives each of C persistent CTAs a contiguous range of equal cost
over the units (sequence, KV head, slice of up to 128 query heads), a unit
costing UNIT_COST plus its key tiles of 128; each CTA writes one partial per
half for every unit it touches, in slot 2 * (cta + unit) + half.  The model
below restates that arithmetic and checks the invariants the kernel relies
on: every key tile is processed exactly once, no slot is written twice or
lies past the workspace, and the merge's lookup finds exactly the slots that
were written for each unit.  The GPU parity tests check the kernel itself.
"""
import numpy as np
import pytest

from paged_kv_cache_480_b200 import workloads as wl

UNIT_COST = 2      # kTcUnitCost
CTAS = 148         # kDecodeTcCtas


def split(lens, num_heads, num_kv_heads, C=CTAS, unit_cost=UNIT_COST):
    S = len(lens)
    G = num_heads // num_kv_heads
    slices = (G + 127) // 128
    NU = num_kv_heads * slices
    tiles = [(L + 127) // 128 for L in lens]
    w = [unit_cost + t if t > 0 else 0 for t in tiles]
    W = np.concatenate([[0], np.cumsum(w)]).astype(np.int64)
    V = int(W[-1]) * NU
    slots_cap = 2 * (C + S * NU)
    covered, written, cost = {}, set(), []
    for c in range(C):
        v0, v1 = V * c // C, V * (c + 1) // C
        found = [s for s in range(S) if w[s] > 0 and W[s] * NU <= v0 < W[s + 1] * NU]
        if v1 <= v0 or not found:
            cost.append(0)
            continue
        s = found[0]
        o = v0 - W[s] * NU
        u = o // w[s]
        t = max(0, o - u * w[s] - unit_cost)
        left = v1 - (W[s] * NU + u * w[s] + unit_cost)   # cost from the unit's first tile to the end
        done = nseg = 0
        while True:
            while t >= tiles[s]:
                if tiles[s] > 0:
                    left -= tiles[s] + unit_cost
                t = 0
                u += 1
                if u == NU:
                    u, s = 0, s + 1
                    if s == S:
                        break
            if s == S or t >= left:
                break
            n = min(tiles[s] - t, left - t)
            for k in range(t, t + n):
                covered[(s, u, k)] = covered.get((s, u, k), 0) + 1
            for x in (0, 1):
                slot = 2 * (c + s * NU + u) + x
                assert slot < slots_cap
                assert (s, u, slot) not in written
                written.add((s, u, slot))
            t += n
            done += n
            nseg += 1
        cost.append(done + unit_cost * nseg)
    for s in range(S):
        for u in range(NU):
            for k in range(tiles[s]):
                assert covered.get((s, u, k), 0) == 1, (s, u, k)
    # the merge: the CTAs whose range meets unit u's tiles, from the prefix sums W
    read = set()
    for s in range(S):
        ws = int(W[s + 1] - W[s])
        Ts = ws - unit_cost if ws > 0 else 0
        assert Ts == tiles[s]
        if Ts == 0:
            continue
        for u in range(NU):
            a = int(W[s]) * NU + u * ws + unit_cost
            cf, cl = ((a + 1) * C - 1) // V, ((a + Ts) * C - 1) // V
            assert 2 * (cl - cf + 1) <= 2 * C
            for cc in range(cf, cl + 1):
                if (cc + 1) * V // C > cc * V // C:
                    for x in (0, 1):
                        read.add((s, u, 2 * (cc + s * NU + u) + x))
    assert read == written
    return cost


EDGE = [0, 1, 15, 16, 17, 127, 128, 129, 255, 256, 257, 511, 512, 513, 1000, 33]


@pytest.mark.parametrize("heads,kv_heads", [(32, 2), (64, 1), (256, 1), (130, 1), (128, 4)])
@pytest.mark.parametrize("unit_cost", [0, 2])
def test_edge_lengths(heads, kv_heads, unit_cost):
    split(EDGE, heads, kv_heads, unit_cost=unit_cost)


@pytest.mark.parametrize("C", [1, 2, 3, 7, 148])
def test_few_ctas_and_empty_sequences(C):
    split([700, 1300, 90, 1, 0, 513], 32, 2, C=C)
    split([0, 0, 300, 0, 0, 1, 0], 32, 2, C=C)
    split([0, 0], 64, 4, C=C)
    split([1], 64, 1, C=C)


def test_many_short_sequences():
    split([129] * 400, 16, 1)
    split([5000] * 200, 32, 2)


def test_mqa_workload_is_balanced():
    """On the MQA workload the ranges cost the same to within one tile, and
    a unit boundary no longer lands two units' fixed costs on one CTA."""
    lay = wl.make_layout("mqa_long_bf16")
    cost = split([int(L) for L in lay.context_lens], lay.num_heads, lay.num_kv_heads)
    assert max(cost) - min(cost) <= UNIT_COST + 1
