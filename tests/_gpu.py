"""GPU-side helpers for the parity tests: move a Workload to the device and run
the hot path through the C ABI (via the ctypes binding)."""
import numpy as np
import torch

from paged_kv_cache_lens_b200 import pa
from paged_kv_cache_lens_b200 import workloads as wl

TORCH_DT = {wl.F16: torch.float16, wl.BF16: torch.bfloat16, wl.F32: torch.float32}
NAN_BITS = {wl.BF16: 0x7FC0, wl.F16: 0x7E00}


def bits_to_dev(a, dtype, dev="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.to(dev).view(TORCH_DT[dtype])


class DeviceStep:
    """Device copies of a workload's inputs, a NaN-filled pool, and the step."""

    def __init__(self, W, dev="cuda", out_dtype=None):
        self.W = W
        self.dev = dev
        shape = (W.num_blocks, W.num_kv_heads, W.block_size, W.head_dim)
        if W.kv_dtype == wl.FP8_E4M3:
            self.k_cache = torch.full(shape, 0x7F, dtype=torch.uint8, device=dev)
            self.v_cache = torch.full(shape, 0x7F, dtype=torch.uint8, device=dev)
            self.k_scale = torch.from_numpy(W.k_scale).to(dev)
            self.v_scale = torch.from_numpy(W.v_scale).to(dev)
        else:
            nan = NAN_BITS[W.kv_dtype]
            self.k_cache = torch.full(shape, nan, dtype=torch.int16, device=dev).view(
                TORCH_DT[W.kv_dtype])
            self.v_cache = torch.full(shape, nan, dtype=torch.int16, device=dev).view(
                TORCH_DT[W.kv_dtype])
            self.k_scale = self.v_scale = None
        self.q = bits_to_dev(W.q, W.q_dtype, dev)
        self.new_k = bits_to_dev(W.new_k, W.src_dtype, dev)
        self.new_v = bits_to_dev(W.new_v, W.src_dtype, dev)
        self.new_slots = torch.from_numpy(W.new_slots).to(dev)
        self.block_tables = torch.from_numpy(W.block_tables).to(dev)
        self.seqlens_k = torch.from_numpy(W.seqlens_k).to(dev)
        self.cu = torch.from_numpy(W.cu_seqlens_q).to(dev)
        self.out_dtype = W.out_dtype if out_dtype is None else out_dtype
        self.out = torch.empty((W.total_q, W.num_q_heads, W.head_dim),
                               dtype=TORCH_DT[self.out_dtype], device=dev)
        if W.decode:
            n = pa.pa_decode_workspace_size(W.num_seqs, W.num_q_heads, W.head_dim,
                                            W.max_context_len, W.partition_size)
        else:
            n = pa.pa_varlen_workspace_size(W.num_seqs, W.total_q, W.num_q_heads, W.head_dim,
                                            W.max_context_len)
        self.workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
        self.window = 0            # sliding window / ALiBi for pa_decode_ex / pa_varlen_ex
        self.alibi = None

    def fill_cache(self, chunk=1 << 18):
        """Write the cached context (outside any timed region), in pieces."""
        W = self.W
        for s in range(0, len(W.prefill_slots), chunk):
            e = min(len(W.prefill_slots), s + chunk)
            k = bits_to_dev(W.prefill_k[s:e], W.src_dtype, self.dev)
            v = bits_to_dev(W.prefill_v[s:e], W.src_dtype, self.dev)
            sl = torch.from_numpy(W.prefill_slots[s:e]).to(self.dev)
            pa.pa_reshape_and_cache(k, v, sl, self.k_cache, self.v_cache, self.k_scale,
                                    self.v_scale)
        torch.cuda.synchronize()

    def write_new(self):
        pa.pa_reshape_and_cache(self.new_k, self.new_v, self.new_slots, self.k_cache,
                                self.v_cache, self.k_scale, self.v_scale)

    def attend(self, partition_size=None):
        W = self.W
        if W.decode and partition_size is not None:
            n = pa.pa_decode_workspace_size(W.num_seqs, W.num_q_heads, W.head_dim,
                                            W.max_context_len, partition_size)
            if n > self.workspace.numel():
                self.workspace = torch.empty(n, dtype=torch.uint8, device=self.dev)
        if W.decode:
            pa.pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.block_tables,
                         self.seqlens_k, W.max_context_len, W.scale, self.k_scale, self.v_scale,
                         W.partition_size if partition_size is None else partition_size,
                         self.workspace, window=self.window, alibi_slopes=self.alibi)
        else:
            pa.pa_varlen(self.out, self.q, self.cu, self.seqlens_k, W.max_q_len,
                         W.max_context_len, self.k_cache, self.v_cache, self.block_tables,
                         W.scale, self.k_scale, self.v_scale, self.workspace,
                         window=self.window, alibi_slopes=self.alibi)

    def step(self, **kw):
        self.write_new()
        self.attend(**kw)

    def out_f64(self):
        return self.out.float().cpu().numpy().astype(np.float64)


def ulp(x, dtype):
    """Spacing of the output format at |x| (half an ulp is the rounding bound)."""
    ax = np.maximum(np.abs(x), 1e-30)
    e = np.floor(np.log2(ax))
    if dtype == wl.BF16:
        return np.exp2(np.maximum(e, -126) - 7)
    if dtype == wl.F16:
        return np.exp2(np.maximum(e, -14) - 10)
    return np.zeros_like(x)


def tolerance(W, want, out_dtype):
    base = 5e-2 if W.kv_dtype == wl.FP8_E4M3 else 2e-3
    return base + 0.5 * ulp(want, out_dtype)


def assert_close(got, want, W, out_dtype, what=""):
    tol = tolerance(W, want, out_dtype)
    err = np.abs(got - want)
    bad = ~(err <= tol)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {bad.sum()} of {bad.size} outside tolerance; max err {np.nanmax(err):.3e};"
            f" first {idx.tolist()} got {got[bad][:5]} want {want[bad][:5]}")
    return float(np.max(err)) if err.size else 0.0


def sampled_oracle_pools(oracle, W, rows):
    """Oracle pool holding the cached context of the requests owning `rows`
    (np.empty pool: only the touched pages are ever committed or read)."""
    reqs = sorted({int(np.searchsorted(W.cu_seqlens_q, r, side="right") - 1) for r in rows})
    blocks = set()
    for rq in reqs:
        n = -(-int(W.seqlens_k[rq]) // W.block_size)
        blocks.update(int(b) for b in W.block_tables[rq, :n])
    blocks = np.array(sorted(blocks), np.int64)
    shape = (W.num_blocks, W.num_kv_heads, W.block_size, W.head_dim)
    dt = np.uint8 if W.kv_dtype == wl.FP8_E4M3 else np.uint16
    kc, vc = np.empty(shape, dt), np.empty(shape, dt)
    for k, v, s in ((W.prefill_k, W.prefill_v, W.prefill_slots), (W.new_k, W.new_v, W.new_slots)):
        keep = np.isin(s // W.block_size, blocks) & (s >= 0)
        if keep.any():
            oracle.reshape_and_cache(k[keep], v[keep], W.src_dtype, s[keep], kc, vc, W.block_size,
                                     W.kv_dtype, W.k_scale, W.v_scale)
    return kc, vc
