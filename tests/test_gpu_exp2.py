"""The FMA-pipe 2^x polynomials against float64 2^x and the hardware ex2, on
the device: relative error within the fitted bounds over the range the
kernels use, exact powers of two, and 0 below -127 (masked entries)."""
import numpy as np
import pytest
import torch

from long_context_sparse_flash_b200 import native as nv

pytestmark = pytest.mark.gpu


def test_exp2_polynomials_error_bounds():
    xs = torch.cat([torch.linspace(-126.0, 20.0, 400001), torch.arange(-126, 21, dtype=torch.float32),
                    torch.tensor([-127.5, -200.0, float("-inf")])]).cuda()
    hw, p3, p5, q5, q5h = (y.cpu().numpy().astype(np.float64) for y in nv.hs2_selftest_exp2(xs))
    x = xs.cpu().numpy().astype(np.float64)
    # the packed two-lane form computes the same function, bit for bit
    assert np.array_equal(q5, p5)
    xh = (xs * 0.5).cpu().numpy().astype(np.float64)
    okh = xh >= -125.0
    assert np.abs(q5h[okh] / np.exp2(xh[okh]) - 1).max() < 3e-7
    assert np.all(q5h[xh < -127.0] == 0)
    ref = np.exp2(x)
    ok = x >= -125.0  # normal results
    rel = lambda y: np.abs(y[ok] / ref[ok] - 1)
    assert rel(hw).max() < 1e-6
    assert rel(p3).max() < 1.3e-4
    assert rel(p5).max() < 3e-7
    ints = np.isin(x, np.arange(-125, 21))
    assert np.all(p3[ints] == ref[ints]) and np.all(p5[ints] == ref[ints])  # exact powers of two
    low = x < -127.0
    assert np.all(p3[low] == 0) and np.all(p5[low] == 0)


def test_gather_probe_reads_and_skips_bad_indices():
    """The gather probe behind the sparse layer's roofline runs, counts as a launch,
    and tolerates out-of-range indices (read as row 0 on the device)."""
    rows = torch.ones(1 << 20, dtype=torch.uint8, device="cuda")  # 4096 rows of 256 bytes
    order = torch.randint(0, 4096, (4096,), dtype=torch.int32, device="cuda")
    order[::97] = -5
    order[::89] = 1 << 30
    sink = torch.zeros(4, dtype=torch.int32, device="cuda")
    before = nv.hs2_launch_count()
    nv.hs2_gather_probe(rows, order, 2, sink)
    torch.cuda.synchronize()
    assert nv.hs2_launch_count() == before + 1
    assert torch.all(sink == 0)  # the keep-alive store is not taken


def test_ex2_probe_counts_and_runs():
    """The special-function-unit probe behind the selection sweep's roofline runs as
    one launch and reports (SM count x 8 CTAs) x 256 threads x 8 chains x iters ex2."""
    sink = torch.zeros(4, dtype=torch.float32, device="cuda")
    before = nv.hs2_launch_count()
    n = nv.hs2_ex2_probe(16, sink)
    torch.cuda.synchronize()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert n == sms * 8 * 256 * 8 * 16
    assert nv.hs2_launch_count() == before + 1
    assert torch.all(sink == 0)
