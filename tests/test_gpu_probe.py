"""GPU: the shared-memory gather probe returns a rate inside what the hardware
can deliver (at most one 128-byte wavefront per SM clock), for the plain
random-row pattern and for the forward kernel's own corner pattern."""
import pytest

import deformable_convolution_sparse_b200 as dcn

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("pattern", [0, 1])
def test_probe_rate_is_plausible(pattern, cuda_device):
    rate = dcn.probe_smem_gather(pattern)
    assert 16.0 < rate <= 128.5, rate
