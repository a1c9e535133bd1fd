"""The read-only stream used to measure this GPU's read rate (pa_hbm_read): it reads
every word of the buffer once, which the XOR it leaves in its sink shows."""
import numpy as np
import pytest
import torch

from paged_kv_cache_370_b200 import abi

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines too; every test here needs the GPU
    pytest.skip("no CUDA device", allow_module_level=True)


@pytest.mark.parametrize("nwords", [4, 4 * 1000 + 8, 32 << 20])
def test_hbm_read_folds_every_word(nwords):
    rng = np.random.default_rng(nwords)
    host = rng.integers(0, 2**32, size=nwords, dtype=np.uint32)
    buf = torch.from_numpy(host.view(np.int32)).cuda()
    sink = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    abi.pa_hbm_read(buf, sink)
    torch.cuda.synchronize()
    want = np.bitwise_xor.reduce(host)
    assert int(sink.cpu().numpy().view(np.uint32)[0]) == int(want)


def test_hbm_read_rejects_bad_sizes():
    buf = torch.zeros(6, dtype=torch.int32, device="cuda")  # 24 bytes: not a multiple of 16
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError):
        abi.pa_hbm_read(buf, sink)
    with pytest.raises(RuntimeError):
        abi.pa_hbm_read(buf[:4], sink, ctas_per_sm=5)
