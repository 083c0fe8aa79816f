"""The measured peaks the roofline fractions are reported against: the
pure-read HBM probe (the decode kernels' second denominator) on this device,
and its argument checks."""
import pytest
import torch

import decode_matvec_sq_b200 as sq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built(cuda_device):
    from decode_matvec_sq_b200 import build
    build.build_all()
    sq.device_check()
    yield


def test_read_probe_is_plausible():
    """Read-only sweeps of 1 GiB (8x the L2): between a tenth of and 1.2x
    the nominal 8 TB/s of HBM3e.  A 1 MiB buffer (launch-bound) reads at a
    rate well below it: the rate follows the bytes swept, not a constant."""
    buf = torch.zeros(1 << 30, dtype=torch.uint8, device="cuda")
    r = sq.testing_read_peak(buf, iters=10)
    assert 0.8e12 < r < 9.6e12
    small = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")  # 1 MiB: L2-resident, launch-bound
    assert sq.testing_read_peak(small, iters=10) < 2 * r


def test_read_probe_rejects_bad_arguments():
    buf = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(sq.SQError) as e:
        sq.testing_read_peak(buf[1:17])  # not 16-byte aligned
    assert e.value.name == "SQ_ERR_ALIGN"
    with pytest.raises(sq.SQError) as e:
        sq.testing_read_peak(buf[:40])  # not a multiple of 16 bytes
    assert e.value.name == "SQ_ERR_SHAPE"
    for iters in (0, 1001):
        with pytest.raises(sq.SQError) as e:
            sq.testing_read_peak(buf, iters=iters)
        assert e.value.name == "SQ_ERR_SHAPE"
    with pytest.raises(sq.SQError) as e:
        sq.testing_read_peak(torch.zeros(64, dtype=torch.uint8))  # host memory
    assert e.value.name == "SQ_ERR_INVALID_ARG"
