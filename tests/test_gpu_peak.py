"""The measured FMA rate behind the ALU rooflines (tdm_fma_rate)."""
import pytest

from tests.gpu_util import needs_gpu, torch

pytestmark = [pytest.mark.gpu, needs_gpu]


def test_fma_rate_is_near_one_fma_per_lane_per_clock():
    import tiled_distance_maps_b200 as tdm
    rate = tdm.fma_rate()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # 128 float32 lanes per SM; SM clocks between 1.0 and 2.1 GHz
    assert sms * 128 * 1.0e9 * 0.5 < rate < sms * 128 * 2.1e9, rate
    # repeatable to a few per cent
    assert abs(tdm.fma_rate() - rate) < 0.05 * rate
