"""GPU: the probes return rates inside what the hardware can deliver: the
shared-memory gather (at most one 128-byte wavefront per SM clock) for the
plain random-row pattern and the forward kernel's own corner pattern, and the
fp32 vector reductions into L2 that bound the backward's scatter."""
import pytest

import deformable_convolution_sparse_b200 as dcn

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("pattern", [0, 1])
def test_probe_rate_is_plausible(pattern, cuda_device):
    rate = dcn.probe_smem_gather(pattern)
    assert 16.0 < rate <= 128.5, rate


def test_reduction_probe_rates_are_plausible_and_grow_with_the_segment(cuda_device):
    """fp32 vector reductions into L2: payload per SM clock stays below the
    SM's 64-byte-per-clock L1 -> L2 path, and fuller segments (more of a
    128-byte line per request) move at least as many bytes per clock."""
    rates = [dcn.probe_red_global(b) for b in (32, 64, 128)]
    assert all(1.0 < r < 64.0 for r in rates), rates
    assert rates[0] <= rates[1] * 1.05 and rates[1] <= rates[2] * 1.05, rates


def test_shared_atomic_probe_rates_are_plausible(cuda_device):
    """Atomic adds to shared memory, one bank per lane: at most 32 per SM clock
    (one warp instruction per clock), fp32 and integer alike."""
    for fp32 in (True, False):
        r = dcn.probe_red_shared(fp32)
        assert 0.1 < r <= 32.5, (fp32, r)
