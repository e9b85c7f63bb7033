#!/usr/bin/env python3
"""Benchmark of the paged-attention hot path on B200.

One step = the whole path over one batch: write the step's new K/V rows into
the paged pool (pa_reshape_and_cache), then paged attention over every
sequence's cached context (pa_decode; pa_varlen for the mixed step).  The
default (headline) workload is the Llama-3-8B-shaped GQA decode: 256
sequences, context lengths lognormal (median 1000) clipped to [32, 8192], 32
query heads over 8 KV heads of dimension 128, bf16, 16-token blocks, split-K
partitions of 512 tokens.  After it, the same line carries a compact record
of each other workload measured on the same contract ("configs"): the
LLaMA-13B MHA decode, the mixed prefill/decode step (with its decode rows and
prefill chunks timed apart) and the shared-prefix FP8 decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2..5] [--impl reference]

Rank 0 prints one JSON line.  Under torchrun every rank runs an independent
replica of the workload (the path has no exchange step), timed on the device
and reduced as the max over ranks.
"""
from __future__ import annotations

import argparse
import atexit
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
FALLBACK_BF16_TFLOPS = 1590.0
DEFAULT_WORKLOAD = 3
SUB_WORKLOADS = (2, 4, 5)
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD, choices=[2, 3, 4, 5])
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
    ap.add_argument("--no-sub", action="store_true",
                    help="skip the compact records of the other workloads")
    return ap.parse_args()


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
    (widened by the sampling period, so a short region still gets one).  At
    interpreter exit a sampler still running (a run that raised before
    stop()) is killed and the sample file removed."""

    PERIOD_MS = 50

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix=f"pa_clocks_{device_index}_", suffix=".csv")
        os.close(fd)
        self.t0 = self.t1 = None
        atexit.register(self._cleanup)

    def _cleanup(self):
        if self.proc is not None and self.proc.poll() is None:
            self.proc.kill()
            self.proc.wait()
        try:
            os.unlink(self.path)
        except OSError:
            pass

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

TD_NAMES = {wl.F16: "float16", wl.BF16: "bfloat16", wl.F32: "float32"}


def chunk_path(W) -> bool:
    """Whether pa_varlen sends this step's q_len >= 2 requests to the
    tensor-core chunk kernel (the library's rule: a power-of-two GQA group up
    to 128; a 16-bit pool with q of its type at head_dim 64, 128 or 256, or an
    E4M3 pool at head_dim 128)."""
    g = W.num_q_heads // W.num_kv_heads
    if W.decode or W.max_q_len < 2 or g < 1 or g > 128 or (g & (g - 1)):
        return False
    if W.kv_dtype == wl.FP8_E4M3:
        return W.head_dim == 128
    return W.q_dtype == W.kv_dtype and W.head_dim in (64, 128, 256)


class DeviceWorkload:
    """One workload resident on the GPU: the paged pools holding the cached
    context, the step's inputs, the output and the workspace; step() is one
    pass of the whole path (cache write of the new rows, then attention)."""

    def __init__(self, torch, pa, W, dev, window=0, alibi=False):
        self.torch, self.pa, self.W, self.dev = torch, pa, W, dev
        self.window = window
        TD = {k: getattr(torch, v) for k, v in TD_NAMES.items()}
        self.TD = TD
        shape = (W.num_blocks, W.num_kv_heads, W.block_size, W.head_dim)
        if W.kv_dtype == wl.FP8_E4M3:
            self.kc = torch.zeros(shape, dtype=torch.uint8, device=dev)
            self.vc = torch.zeros(shape, dtype=torch.uint8, device=dev)
            self.ks = torch.from_numpy(W.k_scale).to(dev)
            self.vs = torch.from_numpy(W.v_scale).to(dev)
        else:
            self.kc = torch.zeros(shape, dtype=TD[W.kv_dtype], device=dev)
            self.vc = torch.zeros(shape, dtype=TD[W.kv_dtype], device=dev)
            self.ks = self.vs = None
        self.stream = torch.cuda.current_stream(dev)
        # cached context (set-up, untimed)
        chunk = 1 << 18
        for s in range(0, len(W.prefill_slots), chunk):
            e = min(len(W.prefill_slots), s + chunk)
            pa.pa_reshape_and_cache(self.to_dev(W.prefill_k[s:e], W.src_dtype),
                                    self.to_dev(W.prefill_v[s:e], W.src_dtype),
                                    torch.from_numpy(W.prefill_slots[s:e]).to(dev),
                                    self.kc, self.vc, self.ks, self.vs)
        torch.cuda.synchronize(dev)
        # step inputs resident in HBM
        self.q = self.to_dev(W.q, W.q_dtype)
        self.nk = self.to_dev(W.new_k, W.src_dtype)
        self.nv = self.to_dev(W.new_v, W.src_dtype)
        self.slots = torch.from_numpy(W.new_slots).to(dev)
        self.bt = torch.from_numpy(W.block_tables).to(dev)
        self.sk = torch.from_numpy(W.seqlens_k).to(dev)
        self.cu = torch.from_numpy(W.cu_seqlens_q).to(dev)
        self.out = torch.empty((W.total_q, W.num_q_heads, W.head_dim), dtype=TD[W.out_dtype],
                               device=dev)
        if W.decode:
            nws = pa.pa_decode_workspace_size(W.num_seqs, W.num_q_heads, W.head_dim,
                                              W.max_context_len, W.partition_size)
        else:
            nws = pa.pa_varlen_workspace_size(W.num_seqs, W.total_q, W.num_q_heads,
                                              W.head_dim, W.max_context_len)
        self.partials = nws > 0 and (W.decode or self._varlen_partials())
        self.ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=dev)
        self.slopes = None
        if alibi:
            self.slopes = torch.tensor([2.0 ** (-8.0 * (i + 1) / W.num_q_heads)
                                        for i in range(W.num_q_heads)], dtype=torch.float32,
                                       device=dev)

    def _varlen_partials(self):
        W = self.W
        rows = max(W.num_seqs, W.total_q)
        ps = 512
        while ps > 128 and rows * W.num_q_heads * (-(-W.max_context_len // ps)) < 2048:
            ps //= 2
        return -(-W.max_context_len // ps) > 1

    def to_dev(self, a, dt):
        t = self.torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(self.dev)
        return t.view(self.TD[dt])

    def attend(self, q, bt, sk, cu, out, stream=None):
        W, pa = self.W, self.pa
        stream = self.stream if stream is None else stream
        if W.decode:
            pa.pa_decode(out, q, self.kc, self.vc, bt, sk, W.max_context_len, W.scale, self.ks,
                         self.vs, W.partition_size, self.ws, stream, window=self.window,
                         alibi_slopes=self.slopes)
        else:
            pa.pa_varlen(out, q, cu, sk, W.max_q_len, W.max_context_len, self.kc, self.vc, bt,
                         W.scale, self.ks, self.vs, self.ws, stream, window=self.window,
                         alibi_slopes=self.slopes)

    def write_new(self, nk, nv, slots, stream=None):
        self.pa.pa_reshape_and_cache(nk, nv, slots, self.kc, self.vc, self.ks, self.vs,
                                     self.stream if stream is None else stream)

    def step(self):
        self.write_new(self.nk, self.nv, self.slots)
        self.attend(self.q, self.bt, self.sk, self.cu, self.out)

    def launches_per_step(self) -> int:
        """Kernels of this library one step launches: the cache write, then
        attention (decode kernel; plus the work-list and chunk kernels for a
        step with prefill chunks, or the row-map kernel without them), plus
        the partition merge when some row spans several partitions."""
        W = self.W
        n = 1 + 1 + (1 if self.partials else 0)
        if not W.decode:
            n += 2 if chunk_path(W) else 1
        return n

    def time_steps(self, steps, warmup, world=1, clocks=None):
        """Device time of `steps` whole steps (CUDA events on the launching
        stream), and the mean duration of the attention call inside them."""
        torch = self.torch
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(warmup):
            self.step()
        barrier(world)
        torch.cuda.synchronize(self.dev)
        if clocks:
            clocks.mark_start()
        t0.record(self.stream)
        for i in range(steps):
            self.write_new(self.nk, self.nv, self.slots)
            ev[i][0].record(self.stream)
            self.attend(self.q, self.bt, self.sk, self.cu, self.out)
            ev[i][1].record(self.stream)
        t1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        if clocks:
            clocks.mark_end()
        barrier(world)
        ms = max_over_ranks(t0.elapsed_time(t1) / steps, world)
        attn = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in ev])), world)
        assert self.pa.pa_device_error(self.stream) == 0
        return ms, attn

    def time_e2e(self, steps, warmup, world=1):
        """The step through the public API from pinned host memory: every step
        copies its inputs (q, new K/V rows, slots, block tables, lengths,
        cu_seqlens) host -> device as one packed transfer and reads its output
        back device -> host.  Transfers run on a second stream, double
        buffered, so step i+1's inputs cross while step i computes."""
        torch, W = self.torch, self.W
        parts = [("q", W.q.view(np.uint8)), ("nk", W.new_k.view(np.uint8)),
                 ("nv", W.new_v.view(np.uint8)), ("slots", W.new_slots.view(np.uint8)),
                 ("bt", W.block_tables.view(np.uint8)), ("sk", W.seqlens_k.view(np.uint8)),
                 ("cu", W.cu_seqlens_q.view(np.uint8))]
        offs, n = {}, 0
        for name, a in parts:
            offs[name] = (n, a.nbytes)
            n += -(-a.nbytes // 256) * 256
        host = torch.empty(n, dtype=torch.uint8).pin_memory()
        hv = host.numpy()
        for name, a in parts:
            o, b = offs[name]
            hv[o:o + b] = np.ascontiguousarray(a).reshape(-1)
        h_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        dbuf = [torch.empty(n, dtype=torch.uint8, device=self.dev) for _ in range(2)]
        outs = [torch.empty_like(self.out) for _ in range(2)]

        def views(buf):
            def v(name, dt, shape):
                o, b = offs[name]
                return buf[o:o + b].view(dt).view(shape)
            TQ = self.TD[W.q_dtype]
            TS = self.TD[W.src_dtype]
            return (v("q", TQ, self.q.shape), v("nk", TS, self.nk.shape),
                    v("nv", TS, self.nv.shape), v("slots", torch.int64, self.slots.shape),
                    v("bt", torch.int32, self.bt.shape), v("sk", torch.int32, self.sk.shape),
                    v("cu", torch.int32, self.cu.shape))
        vw = [views(b) for b in dbuf]
        cs = torch.cuda.Stream(self.dev)
        E = lambda: torch.cuda.Event()  # noqa: E731
        ready, consumed, drained = [E(), E()], [E(), E()], [E(), E()]
        for e in consumed + drained:
            e.record(self.stream)

        def h2d(i):
            b = i % 2
            cs.wait_event(consumed[b])
            with torch.cuda.stream(cs):
                dbuf[b].copy_(host, non_blocking=True)
            ready[b].record(cs)

        def run(i):
            b = i % 2
            q, nk, nv, slots, bt, sk, cu = vw[b]
            self.stream.wait_event(ready[b])
            self.stream.wait_event(drained[b])
            self.write_new(nk, nv, slots)
            self.attend(q, bt, sk, cu, outs[b])
            consumed[b].record(self.stream)
            cs.wait_event(consumed[b])
            with torch.cuda.stream(cs):
                h_out.copy_(outs[b], non_blocking=True)
            drained[b].record(cs)

        def loop(k):
            h2d(0)
            for i in range(k):
                if i + 1 < k:
                    h2d(i + 1)
                run(i)

        loop(max(warmup, 1))
        torch.cuda.synchronize(self.dev)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        cs.wait_event(e0)
        loop(steps)
        self.stream.wait_event(drained[(steps - 1) % 2])
        e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
        h2d_bytes = sum(a.nbytes for _, a in parts)
        d2h_bytes = h_out.numel() * h_out.element_size()
        assert self.pa.pa_device_error(self.stream) == 0
        return ms, h2d_bytes, d2h_bytes

    def free(self):
        for k in list(vars(self)):
            if k not in ("torch", "pa", "W", "dev", "TD"):
                setattr(self, k, None)
        self.torch.cuda.empty_cache()


def peaks():
    """Roofline denominators: the measured copy bandwidth and bf16 dense
    rate of this machine's B200s (generated MEASURED_PEAKS.json), else the
    recipe's fallback figures."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        hbm = float(d["hbm_gbs"])
        bf16 = float(d.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
        return {"hbm": hbm, "bf16": bf16, "kind": "measured"}
    except (OSError, KeyError, ValueError, TypeError):
        return {"hbm": FALLBACK_HBM_GBS, "bf16": FALLBACK_BF16_TFLOPS, "kind": "fallback"}


def sub_record(torch, pa, c, dev, args, pk):
    """A compact record of reference workload c measured the same way as the
    headline (K timed steps after W warm-up steps, CUDA events)."""
    W = wl.config(c)
    d = DeviceWorkload(torch, pa, W, dev)
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    ms, attn_ms = d.time_steps(args.steps, args.warmup, 1, clocks)
    clocks.stop()
    by = algorithmic_bytes(W)
    attn_gbs = by["attention"] / (attn_ms * 1e-3) / 1e9
    rec = {"workload": workload_name(W), "ms_per_step": round(ms, 5),
           "attention_ms": round(attn_ms, 5), "algorithmic_bytes": by["attention"],
           "achieved_gbs": round(attn_gbs, 1), "frac": round(attn_gbs / pk["hbm"], 4),
           "traffic": recorded_traffic(W),
           "kv_gbs_per_step": round(by["kv"] / (ms * 1e-3) / 1e9, 1),
           "seq_steps_per_s_per_layer": round(W.num_seqs / (ms * 1e-3), 1),
           "clocks": clocks.summary()}
    if by["kv_logical"] != by["kv"]:
        rec["unique_kv_bytes"] = by["kv"]
        rec["logical_kv_bytes"] = by["kv_logical"]
        rec["logical_gbs"] = round(by["kv_logical"] / (attn_ms * 1e-3) / 1e9, 1)
        rec["note"] = "achieved/frac count distinct KV bytes (shared prefix once)"
    if not W.decode:
        split = mixed_split(torch, pa, W, args, dev, d.stream, d.q, d.bt, d.sk, d.out, d.kc,
                            d.vc, d.ks, d.vs, None)
        if split:
            split["decode_rows"]["frac"] = round(split["decode_rows"]["kv_gbs"] / pk["hbm"], 4)
            split["chunks"]["frac_of_bf16_peak"] = round(
                split["chunks"]["tflops"] / pk["bf16"], 4)
            rec["split"] = split
    d.free()
    return rec


def run_native(args):
    import torch
    from paged_kv_cache_lens_b200 import pa

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    W = wl.config(args.workload, batch=args.batch)
    d = DeviceWorkload(torch, pa, W, dev, args.window, args.alibi)
    stream = d.stream

    # ---- device-timed region: K whole steps, attention calls timed too
    clocks = ClockSampler(local)
    clocks.start()
    ms, attn_ms = d.time_steps(args.steps, args.warmup, world, clocks)
    clocks.stop()

    # ---- end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = d.time_e2e(args.steps, args.warmup, world)

    if rank != 0:
        d.free()
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    # ---- context measured after the timed region: read-only HBM ceiling and,
    # for a mixed step, its decode rows and prefill chunks timed apart
    probe = read_probe_gbs(torch, pa, dev, stream)
    pk = peaks()
    split = None
    if not W.decode:
        split = mixed_split(torch, pa, W, args, dev, stream, d.q, d.bt, d.sk, d.out, d.kc, d.vc,
                            d.ks, d.vs, d.slopes)
    launches = d.launches_per_step() * args.steps
    d.free()

    by = algorithmic_bytes(W, args.window)
    peak = pk["hbm"]
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
            "peak_source": f"{pk['kind']} hbm_gbs", "attention_ms": round(attn_ms, 5),
            "algorithmic_bytes": by["attention"],
            "nominal_peak": NOMINAL_HBM_GBS,
            "frac_of_nominal": round(attn_gbs / NOMINAL_HBM_GBS, 4),
            "read_probe_gbs": round(probe, 1),
            "frac_of_read_probe": round(attn_gbs / probe, 4),
        },
        "clocks": clocks.summary(),
        "gpu_launches": launches,
    }
    if split:
        split["decode_rows"]["frac"] = round(split["decode_rows"]["kv_gbs"] / peak, 4)
        split["chunks"]["frac_of_bf16_peak"] = round(split["chunks"]["tflops"] / pk["bf16"], 4)
        line["split"] = split
    if e2e:
        e2e_ms, h2d, d2h = e2e
        line["e2e"] = {"value": round(by["kv"] * world / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": round(e2e_ms, 5),
                       "transfers": "one packed pinned H2D + one D2H per step, on a second "
                                    "stream, double buffered"}
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(W, budget_s=12.0)
    # the other reference workloads, each on the same contract (not in `value`)
    if world == 1 and plain and not args.no_sub and args.workload == DEFAULT_WORKLOAD:
        line["configs"] = [sub_record(torch, pa, c, dev, args, pk) for c in SUB_WORKLOADS]
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
