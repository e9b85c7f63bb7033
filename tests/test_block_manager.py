"""Host logic of block allocation, fork and copy-on-write, and the oracle's
whole-block copy ("PagedAttention 与 Continuous Batching", §3.8 COW 与引用计数)."""
import json
import os

import numpy as np
import pytest

from paged_kv_cache_lens_b200 import workloads as wl
from paged_kv_cache_lens_b200.block_manager import BlockManager, OutOfBlocks

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_cow_trace_of_the_page():
    g = json.load(open(os.path.join(GOLDEN, "cow_trace.json")))
    # blocks 0, 1, 2 hold the prompt; the next free block is 7
    bm = BlockManager(16, free_order=[0, 1, 2, 7, 8, 9, 10, 11])
    prompt = bm.allocate_table(3 * 16 - 5)          # 43 tokens: 3 blocks, last one partial
    assert prompt == g["prompt_blocks"]
    tables = bm.fork(prompt, g["n_samples"])
    assert [bm.ref_count(b) for b in prompt] == g["ref_counts_after_fork"]
    fw = g["first_write"]
    slot, copy = bm.append_slot(tables[fw["sample"]], 43)
    assert copy == (fw["copied_block"], fw["new_block"])
    assert tables[fw["sample"]] == fw["table_after"]
    assert bm.ref_count(fw["copied_block"]) == fw["ref_count_of_copied_after"]
    assert slot == fw["new_block"] * 16 + 43 % 16
    # blocks 0 and 1 stay shared by all four samples
    assert bm.ref_count(0) == bm.ref_count(1) == 4


def test_every_sample_forks_until_the_last_holder_writes_in_place():
    """Samples 1 and 2 copy block 2 as sample 0 did; the fourth finds itself the
    only holder (ref_count 1) and appends in place, by the page's own rule
    (copy only while ref_count > 1)."""
    bm = BlockManager(16, free_order=[0, 1, 2, 7, 8, 9, 10])
    prompt = bm.allocate_table(43)
    tables = bm.fork(prompt, 4)
    copies = [bm.append_slot(t, 43)[1] for t in tables]
    assert copies[:3] == [(2, 7), (2, 8), (2, 9)] and copies[3] is None
    assert tables[3] == [0, 1, 2] and bm.ref_count(2) == 1


def test_full_last_block_gets_a_new_block_and_free_returns_blocks():
    bm = BlockManager(4)
    t = bm.allocate_table(32)                        # exactly two full blocks
    slot, copy = bm.append_slot(t, 32)
    assert copy is None and len(t) == 3 and slot == t[2] * 16
    bm.free_table(t)
    assert sorted(bm.free) == [0, 1, 2, 3] and not bm.ref


def test_out_of_blocks():
    bm = BlockManager(2)
    bm.allocate_table(32)
    with pytest.raises(OutOfBlocks):
        bm.allocate()


def test_oracle_copy_blocks(oracle):
    rng = np.random.default_rng(3)
    kc = wl.randn_bits(rng, (10, 2, 16, 8), wl.BF16)
    vc = wl.randn_bits(rng, (10, 2, 16, 8), wl.BF16)
    k0, v0 = kc.copy(), vc.copy()
    oracle.copy_blocks(kc, vc, kc, vc, [[2, 7], [5, 1]])
    assert np.array_equal(kc[7], k0[2]) and np.array_equal(vc[1], v0[5])
    untouched = [b for b in range(10) if b not in (7, 1)]
    assert np.array_equal(kc[untouched], k0[untouched])
    # between two pools (swap out, then back in elsewhere)
    hk, hv = np.zeros((4, 2, 16, 8), np.uint16), np.zeros((4, 2, 16, 8), np.uint16)
    oracle.copy_blocks(hk, hv, kc, vc, [[3, 0], [4, 1]])
    assert np.array_equal(hk[:2], kc[3:5]) and np.array_equal(hv[:2], vc[3:5])
    with pytest.raises(ValueError):
        oracle.copy_blocks(hk, hv, kc, vc, [[3, 4]])


def test_a_table_that_does_not_fit_takes_no_block():
    bm = BlockManager(3)
    bm.allocate_table(20)                             # 2 blocks
    with pytest.raises(OutOfBlocks):
        bm.allocate_table(40)                         # 3 needed, 1 free
    assert list(bm.free) == [2] and bm.ref_count(2) == 0


def test_misuse_is_refused_with_the_counts_unchanged():
    bm = BlockManager(8)
    t = bm.allocate_table(40)                         # blocks 0, 1, 2
    with pytest.raises(ValueError):
        bm.release(5)                                 # never allocated
    with pytest.raises(ValueError):
        bm.fork(t, 0)
    with pytest.raises(ValueError):
        bm.fork(t + [6], 2)                           # block 6 is not held
    with pytest.raises(ValueError):
        bm.free_table([0, 0, 1])                      # block 0 held once, listed twice
    assert [bm.ref_count(b) for b in range(8)] == [1, 1, 1, 0, 0, 0, 0, 0]
    with pytest.raises(ValueError):
        bm.append_slot(t, 49)                         # the sequence holds at most 48 tokens
    with pytest.raises(ValueError):
        bm.append_slot(t, -1)
    assert t == [0, 1, 2] and len(bm.free) == 5
    slot, copy = bm.append_slot(t, 48)                # the next token opens block 3
    assert copy is None and t == [0, 1, 2, 3] and slot == 48


@pytest.mark.parametrize("order", [[0, 1, 1], [0, 5], [-1, 2]])
def test_free_order_must_name_distinct_pool_blocks(order):
    with pytest.raises(ValueError):
        BlockManager(4, free_order=order)


def test_random_fork_append_free_keeps_the_pool_consistent():
    """Seeded random traffic of new sequences, forks, appends (with their
    copy-on-write) and frees: at every step each block is either free or held,
    never both, and its count equals the number of table entries naming it."""
    rng = np.random.default_rng(5)
    bm = BlockManager(64, block_size=4)
    seqs = []                                         # [table, tokens]
    for _ in range(3000):
        op = rng.integers(4)
        try:
            if op == 0 or not seqs:
                n = int(rng.integers(0, 13))
                seqs.append([bm.allocate_table(n), n])
            elif op == 1:
                i = int(rng.integers(len(seqs)))
                for t in bm.fork(seqs[i][0], int(rng.integers(1, 4)))[1:]:
                    seqs.append([t, seqs[i][1]])
            elif op == 2:
                s = seqs[int(rng.integers(len(seqs)))]
                bm.append_slot(s[0], s[1])
                s[1] += 1
            else:
                bm.free_table(seqs.pop(int(rng.integers(len(seqs))))[0])
        except OutOfBlocks:
            pass
        held = {}
        for t, n in seqs:
            assert len(t) == -(-n // 4)
            for b in t:
                held[b] = held.get(b, 0) + 1
        assert held == bm.ref
        assert not set(bm.free) & set(held) and len(bm.free) + len(held) == 64
