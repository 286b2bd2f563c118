"""The timeout path of the bounded device-side waits, on the GPU, without a
hang: a wait on an mbarrier that nothing completes gives up after a short
bound, the error word reports HS2_ERR_TIMEOUT, and the context stays usable
for the next call."""
import pytest
import torch

from long_context_sparse_flash_b200 import native as nv
from long_context_sparse_flash_b200 import workloads as wl
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from long_context_sparse_flash_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load()


def test_bounded_wait_reports_timeout_and_the_context_stays_usable():
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    nv.hs2_workspace_init(ws)
    rc, info = nv.hs2_get_device_status(ws)
    assert rc == nv.HS2_OK, (rc, info)
    before = nv.hs2_launch_count()
    nv.hs2_selftest_wait(ws, 1 << 20)  # about half a millisecond
    rc, info = nv.hs2_get_device_status(ws)
    assert nv.hs2_launch_count() - before == 1
    assert rc == 6 and list(info) == [6, 17, 1, 0], (rc, list(info))
    # a later call on this context runs normally
    w = wl.WORKLOADS["tiny"]
    inp = wl.make_inputs(w, "cuda")
    gpu = P.run_gpu(w, inp)
    P.compare_rows(w, inp, gpu, 0, [0, 127, 128, 1000, w.n_q - 1])
