"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies gives up, surfaces as IC_ERR_TIMEOUT, and the context stays usable."""
import numpy as np
import pytest
import torch

from lightning_indexer_top_relu_b200 import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ic():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    from lightning_indexer_top_relu_b200 import indexcache
    return indexcache


def test_timed_out_wait_is_reported_and_context_survives(ic):
    assert ic.get_last_device_error() == 0
    ic.selftest_wait_timeout(20000)                 # 20 ms limit
    assert ic.get_last_device_error() == 6          # IC_ERR_TIMEOUT
    assert ic.get_last_device_error() == 0          # cleared on read
    # the context still runs work correctly
    sc = torch.tensor(np.arange(64, dtype=np.float32)[None, None, :].repeat(64, 1), device="cuda")
    idx = ic.topk_select(sc.contiguous(), 4)
    want = [max(0, t - 3) + np.arange(min(4, t + 1)) for t in range(64)]
    got = idx.cpu().numpy()[0]
    for t in range(64):
        assert got[t][: len(want[t])].tolist() == want[t].tolist()
