"""A NumPy model of the chunk kernel's arithmetic (CPU only): 64-key tiles
(as the kernel runs them; 128 too), a running maximum raised only when a tile exceeds it by 2^8, P = 2^(x - m)
entering PV as a bf16 hi + lo pair, fp32 sums.  It pins the precision claim
behind the hi + lo split against the exact fp64 result: with the pair the error is
far inside the 2e-3 bound; with P as one bf16 value a row with a few large
values leaves it."""
import numpy as np
import pytest


LOG2E = 1.4426950408889634


def _bf16(x):
    """float32 -> nearest-even bfloat16, returned as float32."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def _bf16_trunc(x):
    """float32 -> bfloat16 by dropping the low 16 bits (toward zero)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    return (u & np.uint32(0xFFFF0000)).view(np.float32)


def model_row(q, K, V, scale, split=True, tile=128, gap=8.0, trunc=False):
    """One query row over keys K [L, D], values V [L, D] (fp32 arrays holding
    16-bit values), as the chunk kernel computes it.  trunc: hi and lo are
    truncations (the bf16 chunk kernel's packing), else nearest even."""
    c = np.float32(scale * LOG2E)
    m = -np.inf
    o = np.zeros(V.shape[1], np.float32)
    l = np.float32(0)
    for j0 in range(0, K.shape[0], tile):
        s = (K[j0:j0 + tile].astype(np.float64) @ q.astype(np.float64)).astype(np.float32)
        m_tile = np.float32(s.max() * c)
        if m == -np.inf or m_tile > m + gap:
            alpha = np.float32(0) if m == -np.inf else np.float32(np.exp2(np.float32(m - m_tile)))
            o *= alpha
            l *= alpha
            m = m_tile
        p = np.exp2((s * c - np.float32(m)).astype(np.float32)).astype(np.float32)
        l = np.float32(l + p.sum(dtype=np.float32))
        cut = _bf16_trunc if trunc else _bf16
        hi = cut(p)
        pv = hi if not split else hi + cut((p - hi).astype(np.float32))
        o = (o + (pv.astype(np.float64) @ V[j0:j0 + tile].astype(np.float64))).astype(np.float32)
    return o / l


def exact_row(q, K, V, scale):
    s = (K.astype(np.float64) @ q.astype(np.float64)) * scale
    w = np.exp(s - s.max())
    return (w @ V.astype(np.float64)) / w.sum()


def _bf16_normal(rng, shape, sigma=1.0):
    return _bf16((rng.standard_normal(shape) * sigma).astype(np.float32))


@pytest.mark.parametrize("trunc", [False, True])
@pytest.mark.parametrize("tile", [64, 128])
def test_hi_lo_split_stays_far_inside_the_bound(tile, trunc):
    rng = np.random.default_rng(11)
    D = 128
    scale = D ** -0.5
    worst = 0.0
    for L in (1, 2, 3, 17, 64, 65, 128, 129, 700, 2000):
        K, V = _bf16_normal(rng, (L, D)), _bf16_normal(rng, (L, D))
        q = _bf16_normal(rng, D)
        err = np.abs(model_row(q, K, V, scale, tile=tile, trunc=trunc) -
                     exact_row(q, K, V, scale)).max()
        worst = max(worst, err)
    assert worst < 2e-5


@pytest.mark.parametrize("tile", [64, 128])
def test_lazy_rescale_handles_a_late_large_maximum(tile):
    """A key in the last tile scores far above every earlier one: the running
    maximum must be raised and O and l rescaled, not overflow."""
    rng = np.random.default_rng(12)
    D, L = 64, 600
    K, V = _bf16_normal(rng, (L, D)), _bf16_normal(rng, (L, D))
    q = _bf16_normal(rng, D)
    K[590] = _bf16(q * 8)                                       # score ~ 8 |q|^2 / sqrt(D)
    got = model_row(q, K, V, D ** -0.5, tile=tile)
    assert np.isfinite(got).all()
    assert np.abs(got - exact_row(q, K, V, D ** -0.5)).max() < 2e-5


def test_single_bf16_p_can_leave_the_bound():
    """Two keys with equal scores and values far apart: P = 1 for both under
    the maximum, so this row is exact either way; tilt the scores so one P is
    a value bf16 rounds coarsely, and one 16-bit P is off by ~2^-9 of the
    value spread while the hi + lo pair is not."""
    q = np.array([1.0], np.float32)
    # scores 0 and x (scale 1): P = 2^(x log2e) with x chosen so P is far from a bf16 value
    x = np.float32(np.log(1.0 + 2.0 ** -8 + 2.0 ** -9.5))
    K = np.array([[0.0], [x]], np.float32)
    V = np.array([[-4.0], [4.0]], np.float32)
    exact = exact_row(q, K, V, 1.0)
    one = np.abs(model_row(q, K, V, 1.0, split=False) - exact).max()
    pair = np.abs(model_row(q, K, V, 1.0, split=True) - exact).max()
    assert pair < 1e-5
    assert one > 2e-3


def test_truncated_pair_on_adversarial_rows():
    """The bf16 chunk kernel packs P as two truncations (hi = p's upper 16
    bits, lo = (p - hi)'s): p - (hi + lo) < 2^-14 p, so for values of
    magnitude 4 the row error stays below 2^-14 * 4 = 2.4e-4 whatever the
    scores.  Random scores over +-4 values and the two-key row above."""
    rng = np.random.default_rng(13)
    one = np.array([1.0], np.float32)
    worst = 0.0
    for _ in range(200):
        L = int(rng.integers(2, 300))
        K = rng.uniform(-9, 0, size=(L, 1)).astype(np.float32)
        V = np.where(rng.random((L, 1)) < 0.5, -4.0, 4.0).astype(np.float32)
        err = np.abs(model_row(one, K, V, 1.0, tile=64, trunc=True) - exact_row(one, K, V, 1.0))
        worst = max(worst, float(err.max()))
    assert worst < 2.4e-4
    x = np.float32(np.log(1.0 + 2.0 ** -8 + 2.0 ** -9.5))
    K = np.array([[0.0], [x]], np.float32)
    V = np.array([[-4.0], [4.0]], np.float32)
    assert np.abs(model_row(one, K, V, 1.0, trunc=True) - exact_row(one, K, V, 1.0)).max() < 2e-5
