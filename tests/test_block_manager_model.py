"""Pins of the block-manager reference model (CPU only).

The decisive one is a brute-force content replay: every written token gets
a unique label, physical slots hold labels, copy-on-write copies them, and
reading any sequence through its table must give back exactly that
sequence's own history (shared prefix + its own tokens).  That is what
sharing with copy-on-write promises, whatever ids the allocator picks.
"""
import copy

import numpy as np
import pytest

from oracle.block_manager_model import BlockManagerModel, OutOfBlocks


class ContentSim:
    """Physical slot contents driven only by the model's slots and copies."""

    def __init__(self, bm):
        self.bm = bm
        self.slots = {}          # physical slot -> label
        self.history = {}        # seq -> list of labels
        self.next_label = 0

    def _label(self):
        self.next_label += 1
        return self.next_label

    def allocate(self, seq, n):
        blocks = self.bm.allocate(seq, n)
        labels = [self._label() for _ in range(n)]
        bs = self.bm.block_size
        for t, lab in enumerate(labels):
            self.slots[blocks[t // bs] * bs + t % bs] = lab
        self.history[seq] = labels

    def fork(self, parent, child):
        self.bm.fork(parent, child)
        self.history[child] = list(self.history[parent])

    def append(self, seq):
        slot, cow = self.bm.append_slot(seq)
        bs = self.bm.block_size
        if cow is not None:
            src, dst = cow
            for off in range(bs):
                if src * bs + off in self.slots:
                    self.slots[dst * bs + off] = self.slots[src * bs + off]
        lab = self._label()
        self.slots[slot] = lab
        self.history[seq].append(lab)
        return cow

    def free(self, seq):
        self.bm.free_seq(seq)
        del self.history[seq]

    def check(self):
        bs = self.bm.block_size
        for seq, hist in self.history.items():
            table = self.bm.tables[seq]
            got = [self.slots.get(table[t // bs] * bs + t % bs) for t in range(len(hist))]
            assert got == hist, seq
        self.bm.check_invariants()


@pytest.mark.parametrize("seed", range(6))
def test_random_replay_contents_and_invariants(seed):
    rng = np.random.default_rng(seed)
    bm = BlockManagerModel(96, 16, free_order=rng.permutation(96))
    sim = ContentSim(bm)
    live, next_id = [], 0
    for _ in range(600):
        op = rng.random()
        try:
            if op < 0.15 or not live:
                sim.allocate(next_id, int(rng.integers(0, 70)))
                live.append(next_id)
                next_id += 1
            elif op < 0.3:
                parent = live[int(rng.integers(len(live)))]
                sim.fork(parent, next_id)
                live.append(next_id)
                next_id += 1
            elif op < 0.4:
                seq = live.pop(int(rng.integers(len(live))))
                sim.free(seq)
            else:
                sim.append(live[int(rng.integers(len(live)))])
        except OutOfBlocks:
            pass
        sim.check()


def test_cow_fires_only_for_shared_partial_last_block():
    bm = BlockManagerModel(32, 16)
    bm.allocate(0, 20)              # 2 blocks, last holds 4 tokens
    bm.fork(0, 1)
    bm.fork(0, 2)
    slot, cow = bm.append_slot(1)   # shared + partial -> copy
    assert cow is not None and cow[0] == bm.tables[0][1] and cow[1] == bm.tables[1][1]
    assert slot == cow[1] * 16 + 4
    slot, cow = bm.append_slot(2)   # still shared with seq 0 -> copy
    assert cow is not None
    slot, cow = bm.append_slot(0)   # now sole owner -> in place
    assert cow is None and slot == bm.tables[0][1] * 16 + 4
    # a full shared last block never copies: a new block is opened
    bm2 = BlockManagerModel(8, 16)
    bm2.allocate(0, 32)
    bm2.fork(0, 1)
    slot, cow = bm2.append_slot(1)
    assert cow is None and bm2.tables[1][:2] == bm2.tables[0] and slot % 16 == 0
    assert bm2.ref[bm2.tables[0][0]] == 2


def test_out_of_blocks_changes_nothing():
    bm = BlockManagerModel(4, 16)
    bm.allocate(0, 40)              # 3 blocks
    bm.fork(0, 1)
    before = copy.deepcopy(bm.__dict__)
    with pytest.raises(OutOfBlocks):
        bm.allocate(2, 33)          # needs 3, one free
    assert bm.__dict__ == before
    bm.allocate(2, 16)              # the last free block
    before = copy.deepcopy(bm.__dict__)
    with pytest.raises(OutOfBlocks):
        bm.append_slot(1)           # shared partial block needs a copy: no block left
    assert bm.__dict__ == before


def test_sole_owner_append_needs_no_block():
    bm = BlockManagerModel(4, 16)
    bm.allocate(0, 40)
    bm.fork(0, 1)
    bm.append_slot(1)               # copies the partial block: pool now full
    assert bm.num_free() == 0
    slot, cow = bm.append_slot(0)   # seq 0 is now the only owner: writes in place
    assert cow is None
    with pytest.raises(OutOfBlocks):
        bm.allocate(2, 1)


def test_utilisation_bound_without_sharing():
    rng = np.random.default_rng(3)
    bm = BlockManagerModel(400, 16)
    lens = rng.integers(1, 300, 20)
    for s, L in enumerate(lens):
        bm.allocate(s, int(L))
    used = 400 - bm.num_free()
    assert bm.utilisation() == pytest.approx(lens.sum() / (used * 16))
    assert bm.utilisation() >= 1 - 15 * 20 / (used * 16)


def test_swap_out_and_in_keep_contents_and_are_all_or_nothing():
    rng = np.random.default_rng(7)
    gpu = BlockManagerModel(40, 16, free_order=rng.permutation(40))
    cpu = BlockManagerModel(10, 16)
    sim = ContentSim(gpu)
    sim.allocate(0, 70)
    sim.fork(0, 1)
    sim.append(1)                 # 71 tokens, last block copied on write
    sim.allocate(2, 100)          # 7 blocks
    pairs = gpu.swap_out(1, cpu)
    assert len(pairs) == 5 and 1 not in gpu.tables and cpu.lens[1] == 71
    host = {}
    for gb, cb in pairs:          # the copies the caller makes
        for off in range(16):
            if gb * 16 + off in sim.slots:
                host[cb * 16 + off] = sim.slots[gb * 16 + off]
    hist1 = sim.history.pop(1)
    gpu.check_invariants()
    cpu.check_invariants()
    sim.check()                   # the sequences left on the GPU are untouched
    # all or nothing: sequence 2 needs 7 host blocks, 5 are free
    before = copy.deepcopy((gpu.__dict__, cpu.__dict__))
    with pytest.raises(OutOfBlocks):
        gpu.swap_out(2, cpu)
    assert (gpu.__dict__, cpu.__dict__) == before
    # swap back in: fresh device blocks receive the host copies
    back = gpu.swap_in(1, cpu)
    assert len(back) == 5
    for cb, gb in back:
        for off in range(16):
            if cb * 16 + off in host:
                sim.slots[gb * 16 + off] = host[cb * 16 + off]
    sim.history[1] = hist1
    sim.check()                   # sequence 1 reads back exactly its history
    assert cpu.num_free() == 10 and 1 not in cpu.tables
    gpu.check_invariants()
    cpu.check_invariants()
