"""The read-only HBM probe (a measurement helper beside the roofline): it must
read every byte it is given, which its XOR of all 32-bit words shows exactly."""
import numpy as np
import pytest
import torch

from paged_kv_cache_lens_b200 import pa

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nbytes", [16, 4096 + 48, (96 << 20) + 16 * 7])
def test_probe_reads_every_word(nbytes):
    rng = np.random.default_rng(nbytes)
    host = rng.integers(-2**31, 2**31, size=nbytes // 4, dtype=np.int64).astype(np.int32)
    buf = torch.from_numpy(host).cuda()
    sink = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    pa.pa_hbm_read_probe(buf, sink)
    torch.cuda.synchronize()
    want = np.bitwise_xor.reduce(host.view(np.uint32))
    assert int(sink.cpu().numpy().view(np.uint32)[0]) == int(want)


def test_probe_empty_and_misaligned():
    sink = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    pa.pa_hbm_read_probe(torch.empty(0, dtype=torch.int32, device="cuda"), sink)
    torch.cuda.synchronize()
    assert int(sink.item()) == 0
    buf = torch.zeros(64, dtype=torch.int32, device="cuda")
    with pytest.raises(pa.PaError):
        pa.pa_hbm_read_probe(buf[1:5], sink)          # 4-byte offset: not 16-byte aligned
    with pytest.raises(pa.PaError):
        pa.pa_hbm_read_probe(buf[:3], sink)           # 12 bytes: not a multiple of 16
