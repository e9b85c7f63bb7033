"""The pins catch plausible mistakes: each case plants one mistake in a
temporary copy of the oracle's C source (on the CPU), rebuilds it, and checks
that at least one pin fails for the planted copy while the real oracle passes.
Every planted mistake keeps its reads and writes inside the arrays it is
given, so a planted copy returns wrong values rather than corrupting memory.
"""
import os

import numpy as np
import pytest
import torch

from oracle import pa_oracle
from oracle import pa_oracle_np as npo
from paged_kv_cache_lens_b200 import workloads as wl
from tests._helpers import oracle_attention, oracle_pools

SRC = os.path.join(os.path.dirname(pa_oracle.__file__), "pa_oracle.c")

MUTATIONS = {
    "drop_logit_scale": ("s[t] = J->scale * dot + slope", "s[t] = dot + slope"),
    "causal_off_by_one": ("int64_t last = kv_len - q_len + i;", "int64_t last = kv_len - q_len + i - 1;"),
    "top_left_causal": ("int64_t last = kv_len - q_len + i;", "int64_t last = i;"),
    "gqa_interleaved": ("int32_t h = hq / (J->num_q_heads / J->num_kv_heads);",
                        "int32_t h = hq % J->num_kv_heads;"),
    "values_from_key_cache": ("rc = cached(J, J->v_cache, J->v_scale, r, h, t, d, &v);",
                              "rc = cached(J, J->k_cache, J->k_scale, r, h, t, d, &v);"),
    "slot_offset_swapped": ("int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim + d;",
                            "int64_t dst = ((blk * num_kv_heads + h) * block_size + (block_size - 1 - off)) * head_dim + d;"),
    "fp8_ties_away": ("    return fmod(n, 2.0) == 0.0 ? n : n + 1.0;", "    return n + 1.0;"),
    "fp8_scale_multiplied": ("*v *= (double)sc[h];", "*v /= (double)sc[h];"),
    "window_off_by_one": ("first = last - J->window + 1;", "first = last - J->window;"),
    "alibi_sign": ("slope * (double)(t - last)", "slope * (double)(last - t)"),
    "table_row_stride": ("J->block_tables[(int64_t)r * J->max_blocks_per_seq + t / J->block_size]",
                         "J->block_tables[(int64_t)r * (J->max_blocks_per_seq - 1) + t / J->block_size]"),
    "gather_assumes_16_token_blocks": ("J->block_tables[(int64_t)r * J->max_blocks_per_seq + t / J->block_size]",
                                       "J->block_tables[(int64_t)r * J->max_blocks_per_seq + t / 16]"),
    "scatter_assumes_16_token_blocks": ("int64_t blk = slot / block_size;", "int64_t blk = slot / 16;"),
    "fp8_dequant_scale_of_head_0": ("*v *= (double)sc[h];", "*v *= (double)sc[0];"),
    "fp8_quant_scale_of_head_0": ("/ (double)k_scale[h]);", "/ (double)k_scale[0]);"),
    "query_of_head_0": ("(row * J->num_q_heads + hq) * (int64_t)D + d",
                        "(row * J->num_q_heads) * (int64_t)D + d"),
    "alibi_slope_of_kv_head": ("(double)J->alibi_slopes[hq]", "(double)J->alibi_slopes[h]"),
    "window_from_request_end": ("first = last - J->window + 1;", "first = kv_len - J->window;"),
    "copy_skips_last_pair": ("for (int64_t i = 0; i < num_pairs; ++i)",
                             "for (int64_t i = 0; i < num_pairs - 1; ++i)"),
    "copy_half_of_each_k_block": ("(size_t)block_bytes);", "(size_t)block_bytes / 2);"),
    "copy_v_from_k_pool": ("(const char *)src_v + s * block_bytes,", "(const char *)src_k + s * block_bytes,"),
}


def _sdpa(W, kc, vc):
    g = W.num_q_heads // W.num_kv_heads
    out = np.zeros((W.total_q, W.num_q_heads, W.head_dim))
    q = npo.to_f64(W.q, W.q_dtype)
    for r in range(W.num_seqs):
        r0, r1, L = int(W.cu_seqlens_q[r]), int(W.cu_seqlens_q[r + 1]), int(W.seqlens_k[r])
        t = np.arange(L)
        blk = W.block_tables[r, t // W.block_size]
        k = npo.to_f64(kc[blk, :, t % W.block_size, :], W.kv_dtype)
        v = npo.to_f64(vc[blk, :, t % W.block_size, :], W.kv_dtype)
        if W.kv_dtype == wl.FP8_E4M3:
            k = k * W.k_scale.astype(np.float64)[None, :, None]
            v = v * W.v_scale.astype(np.float64)[None, :, None]
        mask = t[None, :] <= (L - (r1 - r0) + np.arange(r1 - r0))[:, None]
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[r0:r1]).transpose(0, 1),
            torch.from_numpy(k).transpose(0, 1).repeat_interleave(g, 0),
            torch.from_numpy(v).transpose(0, 1).repeat_interleave(g, 0),
            attn_mask=torch.from_numpy(mask), scale=float(W.scale))
        out[r0:r1] = o.transpose(0, 1).numpy()
    return out


def _pins_pass(orc) -> bool:
    """A compact run of the pins: codec round trip and midpoints, the scatter
    against the NumPy twin, attention against float64 SDPA on a GQA varlen
    batch with bf16 and FP8 pools of 16-token blocks and a bf16 pool of
    8-token blocks, and whole-block copies within a pool and between two pools
    against plain array assignment."""
    try:
        for b in range(0x7E):
            if orc.e4m3_from_float(orc.e4m3_to_double(b)) != b:
                return False
            lo, hi = orc.e4m3_to_double(b), orc.e4m3_to_double(b + 1)
            mid = (lo + hi) / 2
            if float(np.float32(mid)) == mid and orc.e4m3_from_float(mid) != (b if b % 2 == 0 else b + 1):
                return False
        for kv, bs in ((None, 16), (wl.FP8_E4M3, 16), (None, 8)):
            W = wl.build_workload("m", 31, [1, 6, 1, 20], [30, 6, 17, 52], 4, 2, 16, kv_dtype=kv,
                                  block_size=bs)
            kc, vc = oracle_pools(orc, W)
            kt, vt = np.full_like(kc, kc.flat[-1]), np.full_like(vc, vc.flat[-1])
            kt[:], vt[:] = (0x7F if kv else 0x7FC0), (0x7F if kv else 0x7FC0)
            npo.reshape_and_cache(W.prefill_k, W.prefill_v, W.src_dtype, W.prefill_slots, kt, vt,
                                  W.kv_dtype, W.k_scale, W.v_scale)
            npo.reshape_and_cache(W.new_k, W.new_v, W.src_dtype, W.new_slots, kt, vt,
                                  W.kv_dtype, W.k_scale, W.v_scale)
            if not (np.array_equal(kt, kc) and np.array_equal(vt, vc)):
                return False
            out = oracle_attention(orc, W, kc, vc)
            if not np.allclose(out, _sdpa(W, kt, vt), rtol=0, atol=1e-12):
                return False
        from tests.test_oracle_options import _reference
        W = wl.build_workload("mo", 32, [1, 6, 20], [40, 6, 52], 4, 2, 16)
        kc, vc = oracle_pools(orc, W)
        sl = np.array([0.5, 0.25, 0.125, 0.0625], np.float32)
        got = oracle_attention(orc, W, kc, vc, window=11, alibi_slopes=sl)
        if not np.allclose(got, _reference(W, kc, vc, window=11, slopes=sl), rtol=0, atol=1e-12):
            return False
        rng = np.random.default_rng(33)
        pk = rng.integers(0, 1 << 16, (9, 2, 16, 8)).astype(np.uint16)
        pv = rng.integers(0, 1 << 16, (9, 2, 16, 8)).astype(np.uint16)
        hk, hv = np.zeros((5, 2, 16, 8), np.uint16), np.zeros((5, 2, 16, 8), np.uint16)
        wk, wv = pk.copy(), pv.copy()
        wk[[6, 0]], wv[[6, 0]] = pk[[2, 5]], pv[[2, 5]]
        orc.copy_blocks(pk, pv, pk, pv, [[2, 6], [5, 0]])
        orc.copy_blocks(hk, hv, pk, pv, [[3, 4], [7, 1]])
        if not (np.array_equal(pk, wk) and np.array_equal(pv, wv)):
            return False
        if not (np.array_equal(hk[[4, 1]], wk[[3, 7]]) and np.array_equal(hv[[4, 1]], wv[[3, 7]])
                and not hk[[0, 2, 3]].any() and not hv[[0, 2, 3]].any()):
            return False
        return True
    except (ValueError, IndexError):
        return False


def test_real_oracle_passes_compact_pins():
    assert _pins_pass(pa_oracle)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    p = tmp_path / "pa_oracle_mutant.c"
    p.write_text(mutated)
    orc = pa_oracle.compile_variant(str(p), str(tmp_path / "libmutant.so"))
    assert not _pins_pass(orc), f"planted mistake {name} was not caught"
