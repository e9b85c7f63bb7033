#!/usr/bin/env python3
"""Benchmark of the paged-attention hot path on B200.

One step = the whole path over one batch: write the step's new K/V rows into
the paged pool (pa_reshape_and_cache), then paged attention over every
sequence's cached context (pa_decode; pa_varlen for the mixed step).  The
default workload is the LLaMA-13B-shaped MHA decode: 64 sequences, context
lengths uniform in [128, 2048], 40 heads of dimension 128, bf16, 16-token
blocks in a 12000-block pool.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2..5] [--impl reference]

Rank 0 prints one JSON line.  Under torchrun every rank runs an independent
replica of the workload (the path has no exchange step), timed on the device
and reduced as the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_lens_b200 import workloads as wl  # noqa: E402

METRIC = "paged decode attention: achieved HBM GB/s (% of peak), sequence-steps/s/layer"
FALLBACK_HBM_GBS = 6650.0
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=2, choices=[2, 3, 4, 5])
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--op", default="step", choices=["step", "copy_blocks", "swap_blocks"],
                    help="step: the attention step (default); copy_blocks / swap_blocks: "
                         "whole-block copies on the GQA workload's pool geometry")
    ap.add_argument("--batch", type=int, default=None,
                    help="fewer requests, same distributions (profiling captures only)")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding window (keys per query) for the attention variant")
    ap.add_argument("--alibi", action="store_true", help="ALiBi slopes 2^(-8 i / H)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


NOMINAL_HBM_GBS = 8000.0     # B200 HBM3e, nominal (context beside the measured copy peak)


def read_probe_gbs(torch, pa, dev, stream, nbytes=2 << 30, iters=10) -> float:
    """Read-only HBM ceiling on this GPU: the library's read probe streaming a
    2 GiB buffer (16x the L2), CUDA events around `iters` launches."""
    buf = torch.ones(nbytes // 4, dtype=torch.int32, device=dev)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(3):
        pa.pa_hbm_read_probe(buf, sink, stream)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(iters):
        pa.pa_hbm_read_probe(buf, sink, stream)
    b.record(stream)
    torch.cuda.synchronize(dev)
    gbs = nbytes * iters / (a.elapsed_time(b) * 1e-3) / 1e9
    del buf
    return gbs


def chunk_flops(W, window: int, requests) -> int:
    """Algorithmic FLOPs of the given requests' attention: 4*D per visible
    (query row, query head, key) triple (QK^T and PV)."""
    total = 0
    for r in requests:
        ql, L = int(W.q_lens[r]), int(W.seqlens_k[r])
        pos = L - ql + np.arange(ql, dtype=np.int64)
        vis = pos + 1 if not window or window <= 0 else np.minimum(pos + 1, window)
        total += int(vis.sum())
    return total * W.num_q_heads * 4 * W.head_dim


def visible_keys(W, window: int) -> np.ndarray:
    """Keys each request's attention must read: all of them, or with a
    sliding window the last window + q_len - 1 (the span its rows see)."""
    L = W.seqlens_k.astype(np.int64)
    if window and window > 0:
        return np.minimum(L, window + W.q_lens.astype(np.int64) - 1)
    return L


def algorithmic_bytes(W, window: int = 0) -> dict:
    """Bytes the step must move at least once from HBM: every distinct visible
    K/V slot of every KV head (a block shared by several sequences counts
    once; it is read from L2 after that), the queries, the outputs, the
    block-table entries read, and the new rows written (read + write).
    'kv_logical' counts shared blocks once per sequence (the effective rate)."""
    kv_logical = W.kv_bytes_read()
    kv = W.unique_kv_bytes_read()
    if window and window > 0:
        per_tok = 2 * W.num_kv_heads * W.head_dim * W.kv_elem_bytes()
        kv_logical = int(visible_keys(W, window).sum()) * per_tok
        kv = min(kv, kv_logical)
    q = W.total_q * W.num_q_heads * W.head_dim * 2
    out = W.total_q * W.num_q_heads * W.head_dim * (4 if W.out_dtype == wl.F32 else 2)
    tbl = int((-(-W.seqlens_k.astype(np.int64) // W.block_size)).sum()) * 4 + W.num_seqs * 4
    new = int((W.new_slots >= 0).sum()) * W.num_kv_heads * W.head_dim * 2 * (
        2 + W.kv_elem_bytes()) + W.total_q * 8
    return {"kv": kv, "kv_logical": kv_logical, "attention": kv + q + out + tbl,
            "step": kv + q + out + tbl + new}


def workload_name(W) -> str:
    return wl.CONFIG_NAMES[int(W.name[6])] if W.name.startswith("config") else W.name


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons.  Sampling starts
    before the timed region; summary() keeps the samples stamped inside it
    (widened by the sampling period, so a short region still gets one)."""

    PERIOD_MS = 50

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix=f"pa_clocks_{device_index}_", suffix=".csv")
        os.close(fd)
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu=timestamp,{CLOCK_QUERY}",
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.5)
        except OSError:
            self.proc = None

    def mark_start(self):
        self.t0 = datetime.datetime.now()

    def mark_end(self):
        self.t1 = datetime.datetime.now()

    def stop(self):
        if self.proc is not None:
            time.sleep(2 * self.PERIOD_MS / 1000)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        pad = datetime.timedelta(milliseconds=2 * self.PERIOD_MS)
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                    float(parts[2])
                except ValueError:
                    continue
                if self.t0 - pad <= ts <= self.t1 + pad:
                    rows.append(parts[1:])
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        mx = [float(r[2]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------------------
# distributed plumbing (replicas only)
# --------------------------------------------------------------------------

def dist_setup(n_gpus):
    """One process per GPU (torchrun sets RANK / LOCAL_RANK / WORLD_SIZE): NCCL
    for the timing reduction when CUDA is there, gloo otherwise (CPU tests)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest replica's time: the job-level figure for weak scaling."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------
# the native arm
# --------------------------------------------------------------------------

def run_native(args):
    import torch
    from paged_kv_cache_lens_b200 import pa

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    W = wl.config(args.workload, batch=args.batch)
    TD = {wl.F16: torch.float16, wl.BF16: torch.bfloat16, wl.F32: torch.float32}

    def to_dev(a, dt):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(TD[dt])

    shape = (W.num_blocks, W.num_kv_heads, W.block_size, W.head_dim)
    if W.kv_dtype == wl.FP8_E4M3:
        kc = torch.zeros(shape, dtype=torch.uint8, device=dev)
        vc = torch.zeros(shape, dtype=torch.uint8, device=dev)
        ks = torch.from_numpy(W.k_scale).to(dev)
        vs = torch.from_numpy(W.v_scale).to(dev)
    else:
        kc = torch.zeros(shape, dtype=TD[W.kv_dtype], device=dev)
        vc = torch.zeros(shape, dtype=TD[W.kv_dtype], device=dev)
        ks = vs = None
    stream = torch.cuda.current_stream(dev)
    # cached context (setup, untimed)
    chunk = 1 << 18
    for s in range(0, len(W.prefill_slots), chunk):
        e = min(len(W.prefill_slots), s + chunk)
        pa.pa_reshape_and_cache(to_dev(W.prefill_k[s:e], W.src_dtype),
                                to_dev(W.prefill_v[s:e], W.src_dtype),
                                torch.from_numpy(W.prefill_slots[s:e]).to(dev), kc, vc, ks, vs)
    torch.cuda.synchronize(dev)

    # step inputs resident in HBM
    q = to_dev(W.q, W.q_dtype)
    nk, nv = to_dev(W.new_k, W.src_dtype), to_dev(W.new_v, W.src_dtype)
    slots = torch.from_numpy(W.new_slots).to(dev)
    bt = torch.from_numpy(W.block_tables).to(dev)
    sk = torch.from_numpy(W.seqlens_k).to(dev)
    cu = torch.from_numpy(W.cu_seqlens_q).to(dev)
    out = torch.empty((W.total_q, W.num_q_heads, W.head_dim), dtype=TD[W.out_dtype], device=dev)
    if W.decode:
        nws = pa.pa_decode_workspace_size(W.num_seqs, W.num_q_heads, W.head_dim,
                                          W.max_context_len, W.partition_size)
    else:
        nws = pa.pa_varlen_workspace_size(W.num_seqs, W.total_q, W.num_q_heads, W.head_dim,
                                          W.max_context_len)
    ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=dev)

    slopes = None
    if args.alibi:
        slopes = torch.tensor([2.0 ** (-8.0 * (i + 1) / W.num_q_heads)
                               for i in range(W.num_q_heads)], dtype=torch.float32, device=dev)

    def attend(q_, bt_, sk_, cu_, out_):
        if W.decode:
            pa.pa_decode(out_, q_, kc, vc, bt_, sk_, W.max_context_len, W.scale, ks, vs,
                         W.partition_size, ws, stream, window=args.window, alibi_slopes=slopes)
        else:
            pa.pa_varlen(out_, q_, cu_, sk_, W.max_q_len, W.max_context_len, kc, vc, bt_,
                         W.scale, ks, vs, ws, stream, window=args.window, alibi_slopes=slopes)

    def step():
        pa.pa_reshape_and_cache(nk, nv, slots, kc, vc, ks, vs, stream)
        attend(q, bt, sk, cu, out)

    max_parts = -(-W.max_context_len // (W.partition_size or 512))
    launches_per_step = 1 + 1 + (1 if max_parts > 1 else 0) + (0 if W.decode else 1)

    # ---- device-timed region: K whole steps, attention launches timed too
    ev_a = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.mark_start()
    t0.record(stream)
    for i in range(args.steps):
        pa.pa_reshape_and_cache(nk, nv, slots, kc, vc, ks, vs, stream)
        ev_a[i][0].record(stream)
        attend(q, bt, sk, cu, out)
        ev_a[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark_end()
    barrier(world)
    clocks.stop()
    ms_local = t0.elapsed_time(t1) / args.steps
    attn_ms = float(np.mean([a.elapsed_time(b) for a, b in ev_a]))
    ms = max_over_ranks(ms_local, world)
    attn_ms = max_over_ranks(attn_ms, world)
    assert pa.pa_device_error(stream) == 0

    # ---- end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e:
        pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()  # noqa: E731
        h_q = pin(W.q.view(np.int16))
        h_k, h_v = pin(W.new_k.view(np.int16)), pin(W.new_v.view(np.int16))
        h_slots, h_bt = pin(W.new_slots), pin(W.block_tables)
        h_sk, h_cu = pin(W.seqlens_k), pin(W.cu_seqlens_q)
        h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        d_q, d_k, d_v = torch.empty_like(q), torch.empty_like(nk), torch.empty_like(nv)
        d_slots, d_bt, d_sk, d_cu = (torch.empty_like(slots), torch.empty_like(bt),
                                     torch.empty_like(sk), torch.empty_like(cu))
        h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k, h_v, h_slots, h_bt, h_sk, h_cu))
        d2h = h_out.numel() * h_out.element_size()

        def e2e_step():
            d_q.view(torch.int16).copy_(h_q, non_blocking=True)
            d_k.view(torch.int16).copy_(h_k, non_blocking=True)
            d_v.view(torch.int16).copy_(h_v, non_blocking=True)
            d_slots.copy_(h_slots, non_blocking=True)
            d_bt.copy_(h_bt, non_blocking=True)
            d_sk.copy_(h_sk, non_blocking=True)
            d_cu.copy_(h_cu, non_blocking=True)
            pa.pa_reshape_and_cache(d_k, d_v, d_slots, kc, vc, ks, vs, stream)
            attend(d_q, d_bt, d_sk, d_cu, out)
            h_out.copy_(out, non_blocking=True)

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize(dev)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
        e2e = (e2e_ms, h2d, d2h)

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    # ---- context measured after the timed region: read-only HBM ceiling and,
    # for a mixed step, its decode rows and prefill chunks timed apart
    probe = read_probe_gbs(torch, pa, dev, stream)
    split = None
    if not W.decode:
        split = mixed_split(torch, pa, W, args, dev, stream, q, bt, sk, out, kc, vc, ks, vs,
                            slopes)

    by = algorithmic_bytes(W, args.window)
    peak, peak_kind = peaks()
    gbs = by["kv"] * world / (ms * 1e-3) / 1e9
    attn_gbs = by["attention"] / (attn_ms * 1e-3) / 1e9
    seq_steps = W.num_seqs * world / (ms * 1e-3)
    # the table holds captures of the full-size workloads without window or ALiBi
    plain = args.batch is None and not args.window and not args.alibi
    traffic = recorded_traffic(W) if plain else None
    line = {
        "metric": METRIC,
        "value": round(gbs, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.DTYPE_NAMES[W.kv_dtype],
        "data": "synthetic (seeded N(0,1) q/K/V, seeded block tables)",
        "seq_steps_per_s_per_layer": round(seq_steps, 1),
        "pct_of_hbm_peak": round(100 * gbs / peak, 2),
        "pct_of_nominal_hbm": round(100 * gbs / NOMINAL_HBM_GBS, 2),
        "config": {
            "workload": workload_name(W),
            "batch": W.num_seqs, "total_q": W.total_q, "q_heads": W.num_q_heads,
            "kv_heads": W.num_kv_heads, "head_dim": W.head_dim, "block_size": W.block_size,
            "num_blocks": W.num_blocks, "mean_context": round(float(W.seqlens_k.mean()), 1),
            "max_context": W.max_context_len, "partition_size": W.partition_size or "auto",
            "kv_bytes_per_step": by["kv"], "kv_bytes_logical": by["kv_logical"],
            "effective_gbs": round(by["kv_logical"] * world / (ms * 1e-3) / 1e9, 1),
            "l2": "inputs larger than L2 (KV read per step >> 126 MB); no flush",
            "parallelism": f"replicas x{world}",
            "window": args.window, "alibi": bool(args.alibi),
        },
        "roofline": {
            "bound": "hbm", "kernel": "pa_decode" if W.decode else "pa_varlen",
            "achieved": round(attn_gbs, 1), "peak": peak, "unit": "GB/s",
            "frac": round(attn_gbs / peak, 4), "traffic": traffic,
            "peak_source": f"{peak_kind} hbm_gbs", "attention_ms": round(attn_ms, 5),
            "algorithmic_bytes": by["attention"],
            "nominal_peak": NOMINAL_HBM_GBS,
            "frac_of_nominal": round(attn_gbs / NOMINAL_HBM_GBS, 4),
            "read_probe_gbs": round(probe, 1),
            "frac_of_read_probe": round(attn_gbs / probe, 4),
        },
        "clocks": clocks.summary(),
        "gpu_launches": launches_per_step * args.steps,
    }
    if split:
        line["split"] = split
    if e2e:
        e2e_ms, h2d, d2h = e2e
        line["e2e"] = {"value": round(by["kv"] * world / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": round(e2e_ms, 5)}
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(W, budget_s=12.0)
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def recorded_traffic(W):
    """DRAM bytes per attention launch from the committed ncu summary, if it
    was taken on this workload with the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 3 and parts[0] == W.name and not line.startswith("#"):
                    return int(parts[2]) if parts[1] == kernel_sha(W) else None
    except OSError:
        return None
    return None


def kernel_sha(W=None):
    """Hash of the kernel sources a workload's attention call runs: the decode
    kernel's, plus the chunk kernel's for a step with prefill chunks."""
    import hashlib
    h = hashlib.sha256()
    names = ["paged_attention.cu", "pa_device.cuh", "pa_launch.h"]
    if W is not None and not W.decode:
        names.append("paged_prefill.cu")
    for name in names:
        with open(os.path.join(ROOT, "paged_kv_cache_lens_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# --------------------------------------------------------------------------
# CPU oracle (baseline leg and the reference arm)
# --------------------------------------------------------------------------

def _oracle_sample(W, n_seqs, threads):
    """Run the oracle's step (cache write of the new rows + attention) over the
    first n_seqs requests; returns (seconds, kv bytes processed, requests)."""
    from oracle import pa_oracle
    rows = list(range(int(W.cu_seqlens_q[n_seqs])))
    reqs = n_seqs
    blocks = set()
    for r in range(reqs):
        n = -(-int(W.seqlens_k[r]) // W.block_size)
        blocks.update(int(b) for b in W.block_tables[r, :n])
    blocks = np.array(sorted(blocks), np.int64)
    shape = (W.num_blocks, W.num_kv_heads, W.block_size, W.head_dim)
    dt = np.uint8 if W.kv_dtype == wl.FP8_E4M3 else np.uint16
    kc, vc = np.empty(shape, dt), np.empty(shape, dt)
    keep = np.isin(W.prefill_slots // W.block_size, blocks)
    pa_oracle.reshape_and_cache(W.prefill_k[keep], W.prefill_v[keep], W.src_dtype,
                                W.prefill_slots[keep], kc, vc, W.block_size, W.kv_dtype,
                                W.k_scale, W.v_scale)
    nrows = len(rows)
    t = time.perf_counter()
    pa_oracle.reshape_and_cache(W.new_k[:nrows], W.new_v[:nrows], W.src_dtype,
                                W.new_slots[:nrows], kc, vc, W.block_size, W.kv_dtype,
                                W.k_scale, W.v_scale)
    cu = W.cu_seqlens_q[:reqs + 1]
    pa_oracle.paged_attention(W.q[:nrows], W.q_dtype, cu, W.seqlens_k[:reqs], kc, vc, W.kv_dtype,
                              W.block_tables[:reqs], W.scale, W.k_scale, W.v_scale,
                              num_threads=threads)
    dt_s = time.perf_counter() - t
    per_tok = 2 * W.num_kv_heads * W.head_dim * W.kv_elem_bytes()
    return dt_s, int(W.seqlens_k[:reqs].astype(np.int64).sum()) * per_tok, reqs


def mixed_split(torch, pa, W, args, dev, stream, q, bt, sk, out, kc, vc, ks, vs, slopes,
                iters=30):
    """A mixed step whose leading requests are single-row decodes and the rest
    prefill chunks: each part through pa_varlen on its own (same pools, same
    rows), CUDA events around each of `iters` calls with the L2 flushed before
    each by a 512 MiB read sweep (clean lines: no write-back lands inside the
    timed call), as the full step leaves it.  Decode rows report KV GB/s,
    chunks algorithmic TFLOP/s."""
    flush = torch.ones(128 << 20, dtype=torch.int32, device=dev)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    ql = W.q_lens
    nd = 0
    while nd < W.num_seqs and ql[nd] == 1:
        nd += 1
    if nd == 0 or nd == W.num_seqs or (ql[nd:] < 2).any():
        return None
    per_tok = 2 * W.num_kv_heads * W.head_dim * W.kv_elem_bytes()
    vis = visible_keys(W, args.window)
    res = {}
    for name, r0, r1 in (("decode_rows", 0, nd), ("chunks", nd, W.num_seqs)):
        q0, q1 = int(W.cu_seqlens_q[r0]), int(W.cu_seqlens_q[r1])
        cu_s = torch.from_numpy((W.cu_seqlens_q[r0:r1 + 1] - W.cu_seqlens_q[r0])
                                .astype(np.int32)).to(dev)
        nws = pa.pa_varlen_workspace_size(r1 - r0, q1 - q0, W.num_q_heads, W.head_dim,
                                          W.max_context_len)
        ws_s = torch.empty(max(nws, 256), dtype=torch.uint8, device=dev)
        mq = int(ql[r0:r1].max())

        def call():
            pa.pa_varlen(out[q0:q1], q[q0:q1], cu_s, sk[r0:r1], mq, W.max_context_len, kc, vc,
                         bt[r0:r1], W.scale, ks, vs, ws_s, stream, window=args.window,
                         alibi_slopes=slopes)

        for _ in range(3):
            call()
        torch.cuda.synchronize(dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(iters)]
        with torch.cuda.stream(stream):
            for a, b in evs:
                pa.pa_hbm_read_probe(flush, sink, stream)
                a.record(stream)
                call()
                b.record(stream)
        torch.cuda.synchronize(dev)
        ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
        part = {"requests": r1 - r0, "rows": q1 - q0, "ms": round(ms, 5), "l2": "flushed"}
        if name == "decode_rows":
            kv = int(vis[r0:r1].sum()) * per_tok
            part.update(kv_bytes=kv, kv_gbs=round(kv / (ms * 1e-3) / 1e9, 1))
        else:
            fl = chunk_flops(W, args.window, range(r0, r1))
            part.update(algorithmic_flops=fl, tflops=round(fl / (ms * 1e-3) / 1e12, 1))
        res[name] = part
    assert pa.pa_device_error(stream) == 0
    return res


def cpu_baseline(W, budget_s=12.0):
    """The oracle, as it stands, on this host's cores: a sample of the step
    (first n requests) grown towards budget_s, then repeated until the budget
    is spent."""
    threads = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    t, b, reqs = _oracle_sample(W, 1, threads)
    if t < budget_s and reqs < W.num_seqs:
        n = int(min(W.num_seqs, max(2, 0.5 * budget_s / max(t, 1e-3))))
        t, b, reqs = _oracle_sample(W, n, threads)
    total_t, total_b, reps = t, b, 1
    while total_t < budget_s:
        t, b, reqs = _oracle_sample(W, reqs, threads)
        total_t, total_b, reps = total_t + t, total_b + b, reps + 1
    # one core, on the first request alone, for ~2 s
    t1, b1, reps1 = 0.0, 0, 0
    while t1 < 2.0:
        t, b, _ = _oracle_sample(W, 1, 1)
        t1, b1, reps1 = t1 + t, b1 + b, reps1 + 1
    return {"value": round(total_b / total_t / 1e9, 4), "unit": "GB/s", "cores": threads,
            "single_core_value": round(b1 / t1 / 1e9, 4),
            "single_core_sample": f"request 0 x {reps1} repeats, {t1:.1f} s",
            "kind": "oracle",
            "sample": f"{reqs} of {W.num_seqs} requests of the step (cache write + attention, "
                      f"fp64) x {reps} repeats, {total_t:.1f} s",
            "seq_steps_per_s_per_layer": round(reqs * reps / total_t, 3)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    W = wl.config(args.workload)
    threads = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    # size one step's sample so that warmup + steps stay within a few minutes
    t1, _, _ = _oracle_sample(W, 1, threads)
    n = int(min(W.num_seqs, max(1, 3.0 / max(t1, 1e-3))))
    times, bytes_, reqs = [], 0, n
    for i in range(args.warmup + args.steps):
        t, b, reqs = _oracle_sample(W, n, threads)
        if i >= args.warmup:
            times.append(t)
            bytes_ = b
    s = float(np.mean(times)) if times else float("nan")
    value = bytes_ / s / 1e9
    line = {
        "metric": METRIC, "impl": "reference", "value": round(value, 4), "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(s * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(W), "batch": W.num_seqs,
                   "sample_requests_per_step": reqs},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle",
                         "sample": f"{reqs} of {W.num_seqs} requests per step (fp64 oracle)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_block_op(args):
    """Copy-on-write block copies inside the device pool, or swaps between the
    device pool and a pinned host pool, on Llama-3-8B-shaped blocks (8 KV
    heads x 16 tokens x 128 dims, bf16: 32 KiB per block per K or V)."""
    import torch
    from paged_kv_cache_lens_b200 import pa
    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    rng = np.random.default_rng(77)
    nb, hkv, bs, d = 16384, 8, 16, 128
    kc = torch.randn((nb, hkv, bs, d), dtype=torch.bfloat16, device=dev)
    vc = torch.randn_like(kc)
    block_bytes = hkv * bs * d * 2
    stream = torch.cuda.current_stream(dev)
    if args.op == "copy_blocks":
        n = 2048                                   # scattered (src, dst) pairs
        src = rng.choice(nb // 2, n, replace=False)
        dst = nb // 2 + rng.choice(nb // 2, n, replace=False)
        mapping = torch.from_numpy(np.stack([src, dst], 1).astype(np.int64)).to(dev)
        moved = 2 * 2 * n * block_bytes            # K and V, read + write
        run = lambda: pa.pa_copy_blocks(kc, vc, mapping, stream)  # noqa: E731
        name = "copy_blocks: HBM GB/s (read + write)"
        cfg = {"workload": "copy-on-write copies", "pairs": n, "block_bytes": block_bytes}
    else:
        n = 512                                    # one 8K-token sequence (page: 512 blocks)
        hk = torch.empty((n, hkv, bs, d), dtype=torch.bfloat16).pin_memory()
        hv = torch.empty_like(hk).pin_memory()
        pairs_out = np.stack([rng.choice(nb, n, replace=False), np.arange(n)], 1)
        moved = 2 * n * block_bytes                # K and V, one direction

        def run():
            pa.pa_swap_blocks(hk, hv, kc, vc, pairs_out, stream)
        name = "swap_blocks: device->host GB/s"
        cfg = {"workload": "swap out one 8K-token sequence (512 blocks)", "pairs": n,
               "block_bytes": block_bytes}
    for _ in range(max(args.warmup, 3)):
        run()
    torch.cuda.synchronize(dev)
    steps = min(args.steps, 200)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    t0.record(stream)
    for _ in range(steps):
        run()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world)
    assert pa.pa_device_error(stream) == 0
    if rank == 0:
        print(json.dumps({"metric": name, "value": round(moved * world / (ms * 1e-3) / 1e9, 1),
                          "unit": "GB/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
                          "ms_per_step": round(ms, 5), "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                          "data": "synthetic", "config": cfg, "gpu_launches":
                          steps if args.op == "copy_blocks" else 0}), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.op != "step":
        run_block_op(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
