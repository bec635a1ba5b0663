"""The C++ block manager against the reference model (CPU only).

With the same initial free-list order both follow one policy, so every
slot, copy-on-write pair, table, reference count and utilisation must agree
exactly; the model itself is pinned by the content replay in
test_block_manager_model.py.
"""
import numpy as np
import pytest

from oracle.block_manager_model import BlockManagerModel, OutOfBlocks as ModelOOB
from paged_kv_cache_480_b200 import binding
from paged_kv_cache_480_b200 import build as pkv_build


@pytest.fixture(scope="module", autouse=True)
def _built():
    pkv_build.build()


def compare(bm, model, live):
    assert bm.num_free() == model.num_free()
    for seq in live:
        assert list(bm.block_table(seq)) == model.tables[seq]
        assert bm.seq_len(seq) == model.lens[seq]
    for b in range(model.num_blocks):
        assert bm.ref_count(b) == model.ref[b]
    assert bm.utilisation() == pytest.approx(model.utilisation(), abs=1e-12)


@pytest.mark.parametrize("seed", range(5))
def test_random_ops_match_model_exactly(seed):
    rng = np.random.default_rng(100 + seed)
    nb, bs = 80, 16
    order = rng.permutation(nb)
    bm = binding.BlockManager(nb, bs, free_order=order)
    model = BlockManagerModel(nb, bs, free_order=order)
    live, nxt = [], 0
    for step in range(500):
        op = rng.random()
        if op < 0.15 or not live:
            n = int(rng.integers(0, 60))
            try:
                model.allocate(nxt, n)
                bm.allocate(nxt, n)
                live.append(nxt)
            except ModelOOB:
                with pytest.raises(binding.OutOfBlocks):
                    bm.allocate(nxt, n)
            nxt += 1
        elif op < 0.3:
            parent = live[int(rng.integers(len(live)))]
            model.fork(parent, nxt)
            bm.fork(parent, nxt)
            live.append(nxt)
            nxt += 1
        elif op < 0.4:
            seq = live.pop(int(rng.integers(len(live))))
            model.free_seq(seq)
            bm.free(seq)
        else:
            seq = live[int(rng.integers(len(live)))]
            try:
                want = model.append_slot(seq)
            except ModelOOB:
                with pytest.raises(binding.OutOfBlocks):
                    bm.append_slot(seq)
            else:
                assert bm.append_slot(seq) == want
        if step % 25 == 0:
            compare(bm, model, live)
    compare(bm, model, live)


def test_batch_append_and_fill_tables():
    bm = binding.BlockManager(64, 16)
    model = BlockManagerModel(64, 16)
    for b in (bm, model):
        b.allocate(0, 20)
        b.fork(0, 1)
        b.fork(0, 2)
    slots, pairs = bm.append_slots([1, 2, 0])
    want = [model.append_slot(s) for s in (1, 2, 0)]
    assert list(slots) == [w[0] for w in want]
    assert [tuple(p) for p in pairs] == [w[1] for w in want if w[1] is not None]
    tables, lens = bm.fill_tables([0, 1, 2], 4)
    for i, s in enumerate((0, 1, 2)):
        t = model.tables[s]
        assert list(tables[i, :len(t)]) == t and (tables[i, len(t):] == -1).all()
        assert lens[i] == model.lens[s]


def test_errors():
    bm = binding.BlockManager(4, 16)
    with pytest.raises(binding.PagedKVError):
        bm.fork(7, 8)                       # unknown parent
    bm.allocate(0, 10)
    with pytest.raises(binding.PagedKVError):
        bm.allocate(0, 10)                  # duplicate id
    with pytest.raises(binding.OutOfBlocks):
        bm.allocate(1, 64)                  # 4 blocks needed, 3 free
    assert bm.num_free() == 3
    with pytest.raises(binding.PagedKVError):
        binding.BlockManager(4, 16, free_order=[0, 1, 1, 2])   # not a permutation


def test_swap_out_and_in_match_model_exactly():
    rng = np.random.default_rng(9)
    g_order, h_order = rng.permutation(50), rng.permutation(18)
    gpu, host = binding.BlockManager(50, 16, g_order), binding.BlockManager(18, 16, h_order)
    mg, mh = BlockManagerModel(50, 16, g_order), BlockManagerModel(18, 16, h_order)
    for bm, model in ((gpu, mg),):
        for s, n in ((0, 70), (1, 33), (2, 100)):
            bm.allocate(s, n)
            model.allocate(s, n)
        bm.fork(0, 3)
        model.fork(0, 3)
        assert bm.append_slot(3) == model.append_slot(3)
    # swap out sequence 3 (shares 4 blocks with 0): private host copies
    pairs = gpu.swap_out(host, 3)
    want = mg.swap_out(3, mh)
    assert [tuple(p) for p in pairs] == want
    compare(gpu, mg, [0, 1, 2])
    compare(host, mh, [3])
    # all or nothing: sequences 2 (7 blocks) and 0 (5) fit in the 13 host blocks
    # left; sequence 1 (3 blocks) then finds 1 free and must fail, changing nothing
    for s in (2, 0):
        assert [tuple(p) for p in gpu.swap_out(host, s)] == mg.swap_out(s, mh)
    with pytest.raises(binding.OutOfBlocks):
        gpu.swap_out(host, 1)
    compare(gpu, mg, [1])
    compare(host, mh, [0, 2, 3])
    # swap back in
    assert [tuple(p) for p in host.swap_out(gpu, 3)] == mh.swap_out(3, mg)
    compare(gpu, mg, [1, 3])
    compare(host, mh, [0, 2])
