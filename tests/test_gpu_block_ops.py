"""GPU parity of the whole-block operations through the C ABI: copy-on-write
block copies and device <-> pinned-host block swaps, bit for bit against the
oracle, plus an end-to-end fork: four samples share a prompt, each appends a
token (copy-on-write where the last block is shared) and decodes."""
import numpy as np
import pytest
import torch

from paged_kv_cache_lens_b200 import pa
from paged_kv_cache_lens_b200 import workloads as wl
from paged_kv_cache_lens_b200.block_manager import BlockManager
from tests._gpu import bits_to_dev

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.uint8).cpu().numpy() if t.dtype == torch.uint8 else \
        t.view(torch.int16).cpu().numpy().view(np.uint16)


def _pool(rng, nb, hkv, d, kv):
    if kv == wl.FP8_E4M3:
        return rng.integers(0, 0x7F, size=(nb, hkv, 16, d), dtype=np.uint8)
    return wl.randn_bits(rng, (nb, hkv, 16, d), kv)


def _to_dev(a, kv):
    if kv == wl.FP8_E4M3:
        return torch.from_numpy(a).cuda()
    return bits_to_dev(a, kv)


@pytest.mark.parametrize("kv,hkv,d", [(wl.BF16, 8, 128), (wl.F16, 2, 64), (wl.FP8_E4M3, 8, 128)])
def test_copy_blocks_bit_exact(oracle, kv, hkv, d):
    rng = np.random.default_rng(5)
    nb = 300
    kc, vc = _pool(rng, nb, hkv, d, kv), _pool(rng, nb, hkv, d, kv)
    src = rng.choice(nb // 2, 120, replace=False)
    dst = nb // 2 + rng.choice(nb // 2, 120, replace=False)
    pairs = np.stack([src, dst], 1).astype(np.int64)
    dk, dv = _to_dev(kc, kv), _to_dev(vc, kv)
    pa.pa_copy_blocks(dk, dv, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    oracle.copy_blocks(kc, vc, kc, vc, pairs)
    assert np.array_equal(_bits(dk), kc) and np.array_equal(_bits(dv), vc)


def test_copy_blocks_out_of_range_pair_is_skipped_and_reported():
    rng = np.random.default_rng(6)
    kc = _pool(rng, 8, 2, 64, wl.BF16)
    dk, dv = bits_to_dev(kc, wl.BF16), bits_to_dev(kc, wl.BF16)
    pa.pa_copy_blocks(dk, dv, torch.tensor([[1, 2], [3, 99]], dtype=torch.int64, device="cuda"))
    assert pa.pa_device_error() == 4
    out = _bits(dk)
    assert np.array_equal(out[2], kc[1]) and np.array_equal(out[3:], kc[3:])


def test_swap_out_and_back_in(oracle):
    rng = np.random.default_rng(7)
    nb, nh = 200, 64
    kc, vc = _pool(rng, nb, 8, 128, wl.BF16), _pool(rng, nb, 8, 128, wl.BF16)
    dk, dv = bits_to_dev(kc, wl.BF16), bits_to_dev(vc, wl.BF16)
    hk = torch.zeros((nh, 8, 16, 128), dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    out_pairs = np.array([[10, 0], [11, 1], [12, 2], [50, 7], [199, 63]], np.int64)
    pa.pa_swap_blocks(hk, hv, dk, dv, out_pairs)                 # device -> host
    torch.cuda.synchronize()
    ok, ov = np.zeros((nh, 8, 16, 128), np.uint16), np.zeros((nh, 8, 16, 128), np.uint16)
    oracle.copy_blocks(ok, ov, kc, vc, out_pairs)
    assert np.array_equal(_bits(hk), ok) and np.array_equal(_bits(hv), ov)
    in_pairs = np.array([[0, 100], [1, 101], [2, 102], [7, 3], [63, 150]], np.int64)
    pa.pa_swap_blocks(dk, dv, hk, hv, in_pairs)                  # host -> device
    torch.cuda.synchronize()
    oracle.copy_blocks(kc, vc, ok, ov, in_pairs)
    assert np.array_equal(_bits(dk), kc) and np.array_equal(_bits(dv), vc)
    with pytest.raises(pa.PaError):
        pa.pa_swap_blocks(dk, dv, hk, hv, [[64, 0]])             # past the host pool


def test_fork_with_copy_on_write_then_decode(oracle):
    """Prompt of 43 tokens (3 blocks, last partial) forked into 4 samples;
    each appends one token through the block manager (copy-on-write of block
    2 where it is still shared) and all four decode over their own tables."""
    rng = np.random.default_rng(8)
    hq, hkv, d, nb = 8, 2, 128, 32
    bm = BlockManager(nb)
    prompt_len = 43
    prompt = bm.allocate_table(prompt_len)
    pk = wl.randn_bits(rng, (prompt_len, hkv, d), wl.BF16)
    pv = wl.randn_bits(rng, (prompt_len, hkv, d), wl.BF16)
    slots = np.array([prompt[t // 16] * 16 + t % 16 for t in range(prompt_len)], np.int64)
    kc = torch.full((nb, hkv, 16, d), 0x7FC0, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    vc = torch.full_like(kc.view(torch.int16), 0x7FC0).view(torch.bfloat16)
    pa.pa_reshape_and_cache(bits_to_dev(pk, wl.BF16), bits_to_dev(pv, wl.BF16),
                            torch.from_numpy(slots).cuda(), kc, vc)
    tables = bm.fork(prompt, 4)
    new_slots, copies = [], []
    for t in tables:
        s, c = bm.append_slot(t, prompt_len)
        new_slots.append(s)
        if c:
            copies.append(c)
    assert len(copies) == 3
    pa.pa_copy_blocks(kc, vc, torch.tensor(copies, dtype=torch.int64, device="cuda"))
    nk = wl.randn_bits(rng, (4, hkv, d), wl.BF16)
    nv = wl.randn_bits(rng, (4, hkv, d), wl.BF16)
    pa.pa_reshape_and_cache(bits_to_dev(nk, wl.BF16), bits_to_dev(nv, wl.BF16),
                            torch.tensor(new_slots, dtype=torch.int64, device="cuda"), kc, vc)
    q = wl.randn_bits(rng, (4, hq, d), wl.BF16)
    bt = np.full((4, 4), -1, np.int32)
    for i, t in enumerate(tables):
        bt[i, :len(t)] = t
    lens = np.full(4, prompt_len + 1, np.int32)
    out = torch.empty((4, hq, d), dtype=torch.float32, device="cuda")
    pa.pa_decode(out, bits_to_dev(q, wl.BF16), kc, vc, torch.from_numpy(bt).cuda(),
                 torch.from_numpy(lens).cuda(), prompt_len + 1, float(np.float32(d ** -0.5)))
    torch.cuda.synchronize()
    # oracle: the same writes and copies, in the same order, on host pools
    ok = np.full((nb, hkv, 16, d), 0x7FC0, np.uint16)
    ov = ok.copy()
    oracle.reshape_and_cache(pk, pv, wl.BF16, slots, ok, ov, 16, wl.BF16)
    oracle.copy_blocks(ok, ov, ok, ov, copies)
    oracle.reshape_and_cache(nk, nv, wl.BF16, np.array(new_slots), ok, ov, 16, wl.BF16)
    assert np.array_equal(_bits(kc), ok) and np.array_equal(_bits(vc), ov)
    want = oracle.paged_decode(q, wl.BF16, lens, ok, ov, wl.BF16, bt, float(np.float32(d ** -0.5)))
    got = out.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - want)) < 2e-3
    # the four samples differ only through their own new token
    assert not np.allclose(got[0], got[1])
