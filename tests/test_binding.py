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


class _DevTensor:
    """Stands in for a CUDA tensor on a host without a GPU: the attributes the
    binding reads (device, shape, dtype, strides, pointer)."""

    def __init__(self, shape, dtype, device):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self._ptr = 0x10000 * (1 + len(shape))

    def data_ptr(self):
        return self._ptr

    def stride(self, dim=None):
        s = torch.empty(self.shape, device="meta").stride()
        return s if dim is None else s[dim]

    def numel(self):
        return self.shape.numel()

    def element_size(self):
        return torch.empty((), dtype=self.dtype, device="meta").element_size()


class _FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append(name)
            return 0
        return call


def _fake_cuda(monkeypatch):
    """The binding with its tensor checks, library and device switch replaced
    by recorders; returns (library, list of devices made current, list of
    devices whose current stream was taken)."""
    lib, entered, streams = _FakeLib(), [], []
    monkeypatch.setattr(pa, "_need", lambda *a, **k: None)
    monkeypatch.setattr(pa, "load_library", lambda *a, **k: lib)

    class _Dev:
        def __init__(self, d):
            self.d = d

        def __enter__(self):
            entered.append(self.d)

        def __exit__(self, *exc):
            return False

    monkeypatch.setattr(torch.cuda, "device", _Dev)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda d=None: streams.append(d) or 0)
    return lib, entered, streams


def test_each_call_runs_on_its_tensors_device(monkeypatch):
    """Every entry point makes the device of its tensors current for the call
    and takes that device's stream, not the current device's."""
    lib, entered, streams = _fake_cuda(monkeypatch)
    d1 = torch.device("cuda", 1)
    T = lambda *s, dt=torch.bfloat16: _DevTensor(s, dt, d1)  # noqa: E731
    kc, vc = T(8, 2, 16, 64), T(8, 2, 16, 64)
    i32 = torch.int32
    pa.pa_reshape_and_cache(T(2, 2, 64), T(2, 2, 64), T(2, dt=torch.int64), kc, vc)
    pa.pa_decode(T(2, 4, 64), T(2, 4, 64), kc, vc, T(2, 4, dt=i32), T(2, dt=i32), 16, 0.125)
    pa.pa_decode(T(2, 4, 64), T(2, 4, 64), kc, vc, T(2, 4, dt=i32), T(2, dt=i32), 16, 0.125,
                 window=8)
    pa.pa_varlen(T(3, 4, 64), T(3, 4, 64), T(3, dt=i32), T(2, dt=i32), 2, 16, kc, vc,
                 T(2, 4, dt=i32), 0.125)
    pa.pa_varlen(T(3, 4, 64), T(3, 4, 64), T(3, dt=i32), T(2, dt=i32), 2, 16, kc, vc,
                 T(2, 4, dt=i32), 0.125, alibi_slopes=T(4, dt=torch.float32))
    pa.pa_copy_blocks(kc, vc, T(1, 2, dt=torch.int64))
    pa.pa_hbm_read_probe(T(64, dt=i32), T(1, dt=i32))
    host = _DevTensor((8, 2, 16, 64), torch.bfloat16, "cpu")        # a pinned host pool
    pa.pa_swap_blocks(host, host, kc, vc, np.zeros((1, 2), np.int64))
    launched = [c for c in lib.calls if "workspace" not in c]
    assert launched == ["pa_reshape_and_cache", "pa_decode", "pa_decode_ex", "pa_varlen",
                        "pa_varlen_ex", "pa_copy_blocks", "pa_hbm_read_probe", "pa_swap_blocks"]
    assert entered == [d1] * len(launched)
    assert streams == [d1] * len(launched)


def test_tensors_on_two_devices_are_refused(monkeypatch):
    lib, entered, _ = _fake_cuda(monkeypatch)
    a = lambda *s, dt=torch.bfloat16: _DevTensor(s, dt, "cuda:0")  # noqa: E731
    b = lambda *s, dt=torch.bfloat16: _DevTensor(s, dt, "cuda:1")  # noqa: E731
    i32 = torch.int32
    with pytest.raises(ValueError, match="one CUDA device"):
        pa.pa_decode(a(2, 4, 64), a(2, 4, 64), b(8, 2, 16, 64), b(8, 2, 16, 64), a(2, 4, dt=i32),
                     a(2, dt=i32), 16, 0.125)
    with pytest.raises(ValueError, match="one CUDA device"):
        pa.pa_copy_blocks(a(8, 2, 16, 64), a(8, 2, 16, 64), b(1, 2, dt=torch.int64))
    with pytest.raises(ValueError, match="one CUDA device"):
        pa.pa_swap_blocks(a(8, 2, 16, 64), a(8, 2, 16, 64), b(8, 2, 16, 64), b(8, 2, 16, 64),
                          np.zeros((1, 2), np.int64))
    assert lib.calls == [] and entered == []


def test_device_of_skips_host_and_absent_tensors():
    host = _DevTensor((4,), torch.float32, "cpu")
    dev = _DevTensor((4,), torch.float32, "cuda:3")
    assert pa._device_of(None, host) is None
    assert pa._device_of(host, None, dev, dev) == torch.device("cuda", 3)
