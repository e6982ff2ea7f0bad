"""The integer-throughput probe that gives the attention kernels their roof."""
import pytest
import torch

import integer_only_quantized_int8_b200 as ivit
from integer_only_quantized_int8_b200 import build as ivit_build

pytestmark = pytest.mark.gpu


def test_int_rate_probe_counts_and_rate():
    ivit_build.build()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    sink = torch.zeros(4 * sms, dtype=torch.int32, device="cuda")
    ops = ivit.ivit_selftest_int_rate(16, sink)
    torch.cuda.synchronize()
    assert ops == 4 * sms * 256 * 16 * 8 * 10
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    ops = ivit.ivit_selftest_int_rate(4096, sink)
    b.record()
    torch.cuda.synchronize()
    tops = ops / (a.elapsed_time(b) / 1e3) / 1e12
    # far below one operation per lane per clock of 128 lanes per SM would be
    # a broken probe; far above it, a probe whose work was optimised away
    nominal = sms * 128 * 2.1e9 / 1e12
    print(f"[probe] integer Shiftmax mix: {tops:.2f} TOP/s (nominal issue {nominal:.1f})")
    assert 0.1 * nominal < tops < 1.2 * nominal
    with pytest.raises(ivit.IvitError):
        ivit.ivit_selftest_int_rate(16, sink[:10])
