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
