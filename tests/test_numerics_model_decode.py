"""A NumPy model of the decode kernel's arithmetic (CPU only), in the kernel's
order: a partition's 16-token blocks dealt round-robin to 4 warps, each warp
with its own online-softmax state whose running maximum is raised only when a
block's maximum passes it by more than 2^gap (the raise decided once for the
whole query-head group), P entering PV as a hi + lo pair of 16-bit values
(f16 or bf16 pools) or as one f16 value (E4M3 pools), then the warps merged
and the partitions merged by their log-sum-exp.

It pins the precision claims behind those choices against the exact fp64
softmax (PagedAttention, section 3.6 "PagedAttention Kernel": the kernel
computes plain softmax(q K^T / sqrt(d)) V over the request's blocks):
  * with the pair, the row error stays far inside the 16-bit pools' 2e-3 bound;
  * with one f16 P the error is bounded by 2^-11 max|v| (f16's unit
    roundoff, for any p up to 2^gap), far inside the E4M3 pools' 5e-2 bound;
    a two-key row comes within a factor of 4 of it, so one f16 P is kept to
    the E4M3 pools;
  * P never exceeds 2^gap, which the kernel's constant keeps inside f16; a
    gap of 16 would overflow it.
"""
import math
import re
import warnings
from pathlib import Path

import numpy as np
import pytest

LOG2E = 1.4426950408889634
KERNEL = Path(__file__).resolve().parents[1] / "paged_kv_cache_lens_b200" / "csrc" / "paged_attention.cu"


def _bf16(x):
    """float32 -> nearest-even bfloat16, returned as float32."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def _f16(x):
    """float32 -> nearest-even float16 (inf past 65504), returned as float32."""
    with warnings.catch_warnings():
        warnings.simplefilter("ignore", RuntimeWarning)
        return np.asarray(x, np.float32).astype(np.float16).astype(np.float32)


def _p_operand(p, mode):
    """The P values the PV product sees."""
    if mode == "f16":
        return _f16(p)
    cut = _f16 if mode == "f16pair" else _bf16
    hi = cut(p)
    with np.errstate(invalid="ignore"):
        return hi + cut((p - hi).astype(np.float32))


def model_decode(q, K, V, scale, mode="f16pair", partition_size=0, gap=8.0, warps=4, block=16,
                 k_mul=1.0, v_mul=1.0, slopes=None, stats=None, rescale_o=True):
    """Output [G, D] of a query-head group q [G, D] over keys K [L, D] and
    values V [L, D] (fp32 arrays), as the decode kernel computes it.
    partition_size 0: one partition.  slopes [G]: ALiBi slopes, added as
    slope * key position (natural-log units, as the kernel's argument).
    rescale_o False plants a mistake (O left unscaled on a raise) for the
    test that shows the model notices it."""
    G, L = q.shape[0], K.shape[0]
    c = np.float32(scale * LOG2E * k_mul)
    al = np.zeros(G, np.float32) if slopes is None else (np.asarray(slopes) * LOG2E).astype(np.float32)
    PS = partition_size or max(L, 1)
    nparts = max(1, -(-L // PS))
    part_m, part_l, part_o = [], [], []
    raises = blocks = 0
    p_max = 0.0
    for part in range(nparts):
        t0, t1 = part * PS, min(L, (part + 1) * PS)
        nblk = -(-(t1 - t0) // block)
        wm, wl, wo = [], [], []
        for w in range(warps):
            m = np.full(G, -np.inf, np.float32)
            lsum = np.zeros(G, np.float32)
            o = np.zeros((G, V.shape[1]), np.float32)
            for i in range(w, nblk, warps):
                a, b = t0 + i * block, min(t1, t0 + (i + 1) * block)
                s = (K[a:b].astype(np.float64) @ q.astype(np.float64).T).astype(np.float32)
                pos = np.arange(a, b, dtype=np.float32)[:, None]
                sv = (s * c + al[None, :] * pos).astype(np.float32)          # [tokens, G]
                bm = sv.max(axis=0)
                blocks += 1
                if np.any(bm > m + np.float32(gap)):
                    raises += 1
                    m_new = np.maximum(m, bm)
                    alpha = np.exp2(m - np.where(np.isneginf(m_new), 0, m_new)).astype(np.float32)
                    m, lsum = m_new, lsum * alpha
                    o = o * alpha[:, None] if rescale_o else o
                m_use = np.where(np.isneginf(m), 0, m).astype(np.float32)
                p = np.exp2((sv - m_use[None, :]).astype(np.float32)).astype(np.float32)
                p_max = max(p_max, float(p.max()))
                lsum = (lsum + p.sum(axis=0, dtype=np.float32)).astype(np.float32)
                pv = _p_operand(p, mode)
                o = (o + (pv.astype(np.float64).T @ V[a:b].astype(np.float64))).astype(np.float32)
            wm.append(m), wl.append(lsum), wo.append(o)
        M = np.max(wm, axis=0)
        Mu = np.where(np.isneginf(M), 0, M).astype(np.float32)
        f = [np.exp2(mw - Mu).astype(np.float32) for mw in wm]
        part_m.append(M)
        part_l.append(sum(fi * lw for fi, lw in zip(f, wl)))
        part_o.append(sum(fi[:, None] * ow for fi, ow in zip(f, wo)))
    M = np.max(part_m, axis=0)
    Mu = np.where(np.isneginf(M), 0, M).astype(np.float32)
    f = [np.exp2(mp - Mu).astype(np.float32) for mp in part_m]
    lsum = sum(fi * lp for fi, lp in zip(f, part_l))
    o = sum(fi[:, None] * op for fi, op in zip(f, part_o))
    if stats is not None:
        stats.update(raises=raises, blocks=blocks, p_max=p_max)
    return np.where(lsum[:, None] > 0, o * np.float32(v_mul) / np.where(lsum > 0, lsum, 1)[:, None], 0)


def exact(q, K, V, scale, k_mul=1.0, v_mul=1.0, slopes=None):
    s = (q.astype(np.float64) @ K.astype(np.float64).T) * scale * k_mul
    if slopes is not None:
        s = s + np.asarray(slopes, np.float64)[:, None] * np.arange(K.shape[0])[None, :]
    w = np.exp(s - s.max(axis=1, keepdims=True))
    return (w @ V.astype(np.float64)) * v_mul / w.sum(axis=1, keepdims=True)


def _rows(rng, G, L, D, cast):
    return (cast(rng.standard_normal((G, D)).astype(np.float32)),
            cast(rng.standard_normal((L, D)).astype(np.float32)),
            cast(rng.standard_normal((L, D)).astype(np.float32)))


@pytest.mark.parametrize("mode,cast", [("f16pair", _f16), ("bf16pair", _bf16)])
def test_pair_stays_far_inside_the_16bit_bound(mode, cast):
    rng = np.random.default_rng(21)
    D = 128
    worst = 0.0
    for G, L, ps in [(1, 1, 0), (4, 15, 0), (8, 16, 0), (1, 17, 0), (4, 100, 64), (8, 513, 512),
                     (2, 700, 64), (8, 2000, 512), (4, 1029, 1024)]:
        q, K, V = _rows(rng, G, L, D, cast)
        got = model_decode(q, K, V, D ** -0.5, mode=mode, partition_size=ps)
        worst = max(worst, float(np.abs(got - exact(q, K, V, D ** -0.5)).max()))
    assert worst < 2e-5


def test_one_f16_p_is_bounded_by_half_an_ulp_of_p():
    """With one f16 P, p_hat = p (1 + d), |d| <= 2^-11 for normal f16 values,
    while l sums the fp32 p: the row error is at most 2^-11 max|v| (plus
    flushed subnormals of weight < 2^-14 each).  E4M3 scales fold into the
    logit multiplier and the output; widened E4M3 values are exact in f16."""
    rng = np.random.default_rng(22)
    D = 128
    for G, L, ps in [(1, 40, 0), (4, 300, 64), (8, 1500, 512), (16, 700, 256)]:
        q = _f16(rng.standard_normal((G, D)).astype(np.float32))
        K = _f16(rng.uniform(-8, 8, (L, D)).astype(np.float32))
        V = _f16(rng.uniform(-8, 8, (L, D)).astype(np.float32))
        ks, vs = 0.05, 0.03
        got = model_decode(q, K, V, D ** -0.5, mode="f16", partition_size=ps, k_mul=ks, v_mul=vs)
        err = np.abs(got - exact(q, K, V, D ** -0.5, k_mul=ks, v_mul=vs)).max()
        assert err <= 2.0 ** -11 * 8 * vs * 1.01 + 1e-7
        assert err < 5e-2


def test_one_f16_p_reaches_its_bound():
    """Two keys, values -v and +v, the second scoring just below the first so
    its p sits just past the midpoint of two f16 neighbours below 1 (spacing
    2^-11): one f16 P is off by about 2^-12 v / l = 2^-13 v, while the pair is
    exact to fp32.  At v = 32 that is 3.7e-3: one f16 P would not hold the
    16-bit pools' 2e-3 bound for values of that size."""
    v = 32.0
    x = -math.log(1.0 - 2.0 ** -12 - 2.0 ** -16)          # p_2 = e^-x, just past the midpoint
    q = np.array([[1.0]], np.float32)
    K = np.array([[0.0], [-x]], np.float32)
    V = np.array([[-v], [v]], np.float32)
    ref = exact(q, K, V, 1.0)
    one = float(np.abs(model_decode(q, K, V, 1.0, mode="f16") - ref).max())
    pair = float(np.abs(model_decode(q, K, V, 1.0, mode="f16pair") - ref).max())
    assert pair < 1e-6
    assert 2e-3 < one <= 2.0 ** -11 * v


def _kernel_gap():
    m = re.search(r"constexpr\s+float\s+kLazyRaise\s*=\s*([0-9.]+)f?\s*;", KERNEL.read_text())
    assert m, "the decode kernel's raise threshold was not found"
    return float(m.group(1))


def test_kernel_gap_keeps_p_inside_f16():
    """Blocks that do not raise the running max have every p <= 2^gap, and P
    is stored as f16 (max 65504): the kernel's gap must stay below 16.  A row
    whose scores climb by just under the gap each block keeps p near 2^gap."""
    gap = _kernel_gap()
    assert 2.0 ** gap <= 65504 / 2
    D, L = 1, 16 * 4 * 6
    q = np.array([[1.0]], np.float32)
    # warp w sees blocks w, w+4, ...: its first block scores 0 and sets the running
    # max, every later one scores gap - 0.25 log2 units higher, so no raise after
    # the first and p reaches 2^(gap - 0.25)
    K = np.zeros((L, D), np.float32)
    K[64:] = (gap - 0.25) / LOG2E
    V = np.linspace(-1, 1, L, dtype=np.float32)[:, None]
    stats = {}
    got = model_decode(q, K, V, 1.0, mode="f16pair", gap=gap, stats=stats)
    assert stats["raises"] == 4                 # one per warp: its first block
    assert 2.0 ** (gap - 1) < stats["p_max"] <= 2.0 ** gap
    assert np.abs(got - exact(q, K, V, 1.0)).max() < 2e-5
    # a gap of 16.5 lets p pass 65504: f16 P overflows and the row is lost
    K[64:] = 16.25 / LOG2E
    bad = model_decode(q, K, V, 1.0, mode="f16pair", gap=16.5)
    assert not np.isfinite(bad).all()
    assert np.isfinite(model_decode(q, K, V, 1.0, mode="f16pair", gap=gap)).all()


def test_raise_is_shared_by_the_group_and_rare_on_typical_rows():
    """One head of the group jumps far above its running max late in the row:
    the group's raise carries every head's max along (never lowering one), and
    all heads stay exact.  On N(0, 1) rows at head_dim 128 most blocks skip
    the rescale."""
    rng = np.random.default_rng(23)
    D, G, L = 128, 8, 4096
    q, K, V = _rows(rng, G, L, D, _bf16)
    stats = {}
    got = model_decode(q, K, V, D ** -0.5, mode="bf16pair", partition_size=1024, stats=stats)
    assert np.abs(got - exact(q, K, V, D ** -0.5)).max() < 2e-5
    assert stats["raises"] <= 0.05 * stats["blocks"] + 16
    K[4000] = _bf16(q[3] * 6)                    # head 3 only: a late, far larger score
    got = model_decode(q, K, V, D ** -0.5, mode="bf16pair", partition_size=1024)
    assert np.isfinite(got).all()
    assert np.abs(got - exact(q, K, V, D ** -0.5)).max() < 2e-5


def test_alibi_climb_and_window_free_partitions():
    """ALiBi slopes make scores climb with key position, so the running max is
    raised every few blocks; partitions of 64 and one partition agree with
    the exact softmax."""
    rng = np.random.default_rng(24)
    D, G, L = 64, 4, 900
    q, K, V = _rows(rng, G, L, D, _f16)
    slopes = np.array([0.5, 0.125, 2.0 ** -5, 0.0])
    for ps in (0, 64, 256):
        stats = {}
        got = model_decode(q, K, V, D ** -0.5, mode="f16pair", partition_size=ps, slopes=slopes,
                           stats=stats)
        assert np.abs(got - exact(q, K, V, D ** -0.5, slopes=slopes)).max() < 2e-5
        assert stats["raises"] > 4


def test_model_catches_a_wrong_rescale():
    """The model is sensitive to the step it pins: skipping the rescale of O
    on a raise (l still rescaled) breaks the row by far more than the bound."""
    rng = np.random.default_rng(25)
    D, L = 64, 300
    q, K, V = _rows(rng, 1, L, D, _f16)
    K[250] = _f16(q[0] * 5)
    ref = exact(q, K, V, D ** -0.5)
    assert np.abs(model_decode(q, K, V, D ** -0.5) - ref).max() < 2e-5

    bad = model_decode(q, K, V, D ** -0.5, rescale_o=False)
    assert np.abs(bad - ref).max() > 1e-2
