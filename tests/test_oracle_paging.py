"""Pins of the oracle's paging bookkeeping: page index, slots, free list, block tables (CPU only)."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import workloads as W
from oracle import paging


def check_page_index(golden, page_index=paging.page_index):
    for pos, bs, page in golden("page_index_worked_example.txt"):
        assert page_index(int(pos), int(bs)) == int(page)


def check_slots(golden, slot_of=paging.slot_of):
    row = [7, 2, 9]
    for pos, page, phys, off, slot in golden("slot_hand_example.txt"):
        assert paging.page_index(int(pos)) == int(page)
        assert row[int(page)] == int(phys)
        assert slot_of(row, int(pos)) == int(slot) == int(phys) * 16 + int(off)


def test_page_index_worked_example(golden):
    check_page_index(golden)


def test_slot_hand_examples(golden):
    check_slots(golden)


class _SetModel:
    """Order-free brute-force model of a block manager: a set of free ids and a refcount dict."""

    def __init__(self, n):
        self.free = set(range(n))
        self.ref = {}

    def alloc_ok(self):
        return bool(self.free)

    def take(self, b):
        assert b in self.free
        self.free.remove(b)
        self.ref[b] = 1

    def incref(self, b):
        if self.ref.get(b, 0) == 0:
            return False
        self.ref[b] += 1
        return True

    def decref(self, b):
        if self.ref.get(b, 0) == 0:
            return False
        self.ref[b] -= 1
        if self.ref[b] == 0:
            del self.ref[b]
            self.free.add(b)
        return True


@settings(max_examples=200, deadline=None)
@given(n=st.integers(1, 24), ops=st.lists(st.tuples(st.sampled_from("aifc"), st.integers(-2, 26)), max_size=120),
       seed=st.integers(0, 2**31 - 1))
def test_free_list_model_against_set_model(n, ops, seed):
    order = np.random.default_rng(seed).permutation(n).tolist()
    fl = paging.FreeListModel(n, order)
    ref = _SetModel(n)
    handed = []
    for op, b in ops:
        if op == "a":
            got = fl.alloc()
            if ref.alloc_ok():
                assert got is not None
                ref.take(got)
                handed.append(got)
            else:
                assert got is None
        elif op == "i":
            assert fl.incref(b) == ref.incref(b)
        elif op == "c":
            before = ref.ref.get(b, 0)
            got = fl.cow(b)
            if before == 0:
                assert got is None
            elif before == 1:
                assert got == (b, False)
            elif not ref.free:
                assert got is None
            else:  # the writer's reference moves to a fresh block that must receive a copy
                nb, copy = got
                assert copy and nb != b
                ref.take(nb)
                handed.append(nb)
                assert ref.decref(b)
        else:
            assert fl.free(b) == ref.decref(b)
        assert fl.num_free == len(ref.free)
        assert fl.num_free + len(ref.ref) == n
        for blk in range(n):
            assert fl.refcount(blk) == ref.ref.get(blk, 0) >= 0
    # Until something is freed (a copy-on-write also frees a reference), blocks come out in order.
    if all(op not in "fc" for op, _ in ops):
        assert handed == order[:len(handed)]


def test_freed_block_is_reused_first():
    fl = paging.FreeListModel(4, [2, 0, 3, 1])
    a, b = fl.alloc(), fl.alloc()
    assert (a, b) == (2, 0)
    assert fl.free(a)
    assert fl.alloc() == 2  # stack: last freed is handed out next
    assert fl.alloc() == 3


def test_block_tables_structure():
    for w in (W.TINY, W.LLAMA3_8B_GQA_SMALL, W.PREFIX_GQA_SMALL, W.LONG70B_FP8_SMALL):
        lens = W.context_lens(w).numpy()
        order = W.block_order(w).numpy()
        bt = paging.build_block_tables(lens, order, w.num_blocks, 16, w.shared_prefix_tokens)
        npre = w.shared_prefix_tokens // 16
        need = [-(-int(n) // 16) for n in lens]
        used = []
        for s, nb in enumerate(need):
            assert (bt[s, nb:] == -1).all()
            assert (bt[s, :nb] >= 0).all()
            assert np.array_equal(bt[s, :npre], bt[0, :npre])
            used.extend(bt[s, :nb].tolist() if s == 0 else bt[s, npre:nb].tolist())
        # Distinct physical blocks, handed out exactly in the free list's order.
        assert len(set(used)) == len(used) == sum(need) - npre * (len(lens) - 1)
        assert used == order[:len(used)].tolist()


def test_tiny_block_count():
    lens = W.context_lens(W.TINY).numpy()
    assert lens.tolist() == [1, 17, 33, 100]
    assert sum(-(-int(n) // 16) for n in lens) == 13
