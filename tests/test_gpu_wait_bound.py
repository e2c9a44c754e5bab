"""Failure detection without a GPU fault: a device wait that nothing ever
releases gives up after its bound, records BI_DEV_WAIT_TIMEOUT in the status
word, and leaves the context usable for the next launch."""
import pytest
import torch

from invariant_deterministic_03_b200 import synth
from oracle import fp64
from tests.checker import check
from tests.gpu_common import dev, f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_and_recovers(cuda_device):
    from invariant_deterministic_03_b200 import bi
    bi.bi_device_status(clear=True)
    bi.bi_check_wait_bound(2_000_000)            # ~1 ms at the B200's clock
    torch.cuda.synchronize()
    st = bi.bi_device_status(clear=True)
    assert st & 0x1, f"status {st:#x}"           # BI_DEV_WAIT_TIMEOUT
    assert bi.bi_device_status(clear=True) == 0  # cleared
    # the context still runs kernels, with correct results
    x = synth.normal_bf16((8, 4096), 1.0, 5)
    g = synth.uniform_bf16((4096,), 0.5, 1.5, 6)
    y = bi.rmsnorm(dev(x), dev(g), 1e-6)
    check(f64(y), fp64.rmsnorm(f64(x), f64(g), 1e-6), what="rmsnorm after a timed-out wait")
    assert bi.bi_device_status(clear=True) == 0
