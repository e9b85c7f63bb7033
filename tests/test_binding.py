"""The Python binding's marshalling checks (CPU only): every entry point
rejects, before anything reaches the library, tensors it would misread
through a raw pointer (host memory, strided views, wrong element types)."""
import numpy as np
import pytest
import torch

from paged_kv_cache_lens_b200 import pa


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_host_tensors_are_rejected():
    q, out = _bf16(2, 4, 64), _bf16(2, 4, 64)
    kc, vc = _bf16(8, 2, 16, 64), _bf16(8, 2, 16, 64)
    bt = torch.zeros((2, 4), dtype=torch.int32)
    lens = torch.ones(2, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        pa.pa_decode(out, q, kc, vc, bt, lens, 16, 0.125)
    with pytest.raises(ValueError, match="CUDA"):
        pa.pa_varlen(out, q, torch.tensor([0, 1, 2], dtype=torch.int32), lens, 1, 16, kc, vc, bt,
                     0.125)
    with pytest.raises(ValueError, match="CUDA"):
        pa.pa_reshape_and_cache(_bf16(2, 2, 64), _bf16(2, 2, 64),
                                torch.zeros(2, dtype=torch.int64), kc, vc)
    with pytest.raises(ValueError, match="CUDA"):
        pa.pa_copy_blocks(kc, vc, torch.zeros((1, 2), dtype=torch.int64))
    with pytest.raises(ValueError, match="CUDA"):
        pa.pa_hbm_read_probe(torch.zeros(64, dtype=torch.int32),
                             torch.zeros(1, dtype=torch.int32))
    with pytest.raises(ValueError, match="pinned"):
        pa.pa_swap_blocks(kc, vc, kc.clone(), vc.clone(), np.zeros((1, 2), np.int64))


def test_non_tensor_is_rejected():
    with pytest.raises(TypeError):
        pa.pa_hbm_read_probe(np.zeros(64, np.int32), np.zeros(1, np.int32))


def test_layout_and_dtype_checks():
    """Element types and layouts are checked before the device, so these
    host tensors fail on the point each case plants."""
    need = pa._need
    with pytest.raises(ValueError, match="int32"):
        need(torch.zeros((2, 4), dtype=torch.int64), "block_tables", torch.int32)
    with pytest.raises(ValueError, match="contiguous"):
        need(torch.zeros((4, 6)).t(), "q")
    # rows may be strided when each row is contiguous (views into a fused QKV row)
    qkv = torch.zeros((5, 3 * 2 * 8))
    k = qkv[:, 16:32].view(5, 2, 8)
    with pytest.raises(ValueError, match="CUDA"):         # layout accepted, host rejected
        need(k, "key", rows_strided=True)
    with pytest.raises(ValueError, match="each row"):     # a column slice inside each row
        need(torch.zeros((5, 2, 16))[:, :, :8], "key", rows_strided=True)
    with pytest.raises(ValueError, match="contiguous"):   # a strided view where none is allowed
        need(k, "k_cache")
    need(None, "absent")                                  # optional arguments pass
