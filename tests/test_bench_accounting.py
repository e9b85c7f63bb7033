"""The bench's byte and FLOP accounting against closed forms (CPU only)."""
import numpy as np

import bench
from paged_kv_cache_lens_b200 import workloads as wl


def test_mixed_step_chunk_flops_closed_form():
    """Four 512-row chunks over prior context P in {0, 1024, 2048, 3072}: row i
    of a chunk sees P + i + 1 keys, so a chunk holds 512 P + 512*513/2
    visible (row, key) pairs; each costs 4 D flops per query head."""
    W = wl.config(4)
    chunks = [r for r in range(W.num_seqs) if W.q_lens[r] > 1]
    pairs = sum(512 * p + 512 * 513 // 2 for p in (0, 1024, 2048, 3072))
    assert pairs == 3_671_040
    assert bench.chunk_flops(W, 0, chunks) == pairs * 32 * 4 * 128


def test_chunk_flops_with_window():
    """With a window of W keys, row i of a chunk over prior P sees min(P+i+1, W)."""
    W = wl.build_workload("cw", 3, [1, 100], [50, 300], 8, 2, 64)
    win = 64
    got = bench.chunk_flops(W, win, [1])
    want = sum(min(200 + i + 1, win) for i in range(100)) * 8 * 4 * 64
    assert got == want


def test_decode_bytes_closed_form():
    """Decode: every visible K/V element of every (request, KV head) once."""
    W = wl.build_workload("db", 4, [1, 1, 1], [17, 1, 300], 8, 2, 128)
    by = bench.algorithmic_bytes(W)
    assert by["kv"] == (17 + 1 + 300) * 2 * 2 * 128 * 2
    q = 3 * 8 * 128 * 2
    out = 3 * 8 * 128 * (4 if W.out_dtype == wl.F32 else 2)
    tbl = (2 + 1 + 19) * 4 + 3 * 4
    assert by["attention"] == by["kv"] + q + out + tbl


def test_window_bytes_count_visible_keys_only():
    W = wl.build_workload("wb", 5, [1, 1], [1000, 10], 8, 2, 128)
    per_tok = 2 * 2 * 128 * 2
    assert bench.algorithmic_bytes(W, 64)["kv_logical"] == (64 + 10) * per_tok
    assert np.array_equal(bench.visible_keys(W, 64), [64, 10])


def test_traffic_is_used_only_for_the_sources_it_was_taken_on(monkeypatch):
    """profiles/traffic.txt holds DRAM bytes keyed by the hash of the kernel
    sources a workload runs; another hash yields no traffic figure."""
    W2, W4 = wl.config(2, batch=4), wl.config(4, batch=8)
    assert bench.kernel_sha(W2) == bench.kernel_sha()          # decode kernel sources
    assert bench.kernel_sha(W4) != bench.kernel_sha(W2)        # plus the chunk kernel's
    table = {}
    for line in open(bench.os.path.join(bench.ROOT, "profiles", "traffic.txt")):
        if line.strip() and not line.startswith("#"):
            name, sha, nbytes = line.split()
            table[name] = (sha, int(nbytes))
    sha, nbytes = table[W2.name]
    monkeypatch.setattr(bench, "kernel_sha", lambda W=None: sha)
    assert bench.recorded_traffic(W2) == nbytes
    monkeypatch.setattr(bench, "kernel_sha", lambda W=None: "0" * 16)
    assert bench.recorded_traffic(W2) is None
