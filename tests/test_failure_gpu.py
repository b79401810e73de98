"""Failure detection on the GPU without a fault: every wait in the
library's kernels is bounded, and on expiry records a timeout in the device
error word and lets the kernel return.  Here a wait on a barrier that
nothing completes runs out (a short limit); the host reads HQ_ERR_TIMEOUT
once, the word is cleared, and the context keeps working."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from fp8_dynamic_quantization_amax_b200 import _hq as H
from _gpu import dev_bf16, host

pytestmark = pytest.mark.gpu
HQ_ERR_TIMEOUT = 7


def test_bounded_wait_reports_a_timeout_and_the_context_survives():
    torch.cuda.synchronize()
    H.hq_check_device_error()  # start from a clear error word
    assert H.lib.hq_debug_bounded_wait(50_000_000, None) == 0  # 50 ms
    torch.cuda.synchronize()
    with pytest.raises(H.HQError) as e:
        H.hq_check_device_error()
    assert e.value.status == HQ_ERR_TIMEOUT
    H.hq_check_device_error()  # read once, then clear
    # the context still runs kernels, with bit-exact results
    rng = np.random.default_rng(4)
    xb = W.f32_to_bf16_bits(rng.standard_normal((64, 512)).astype(np.float32))
    q, s = H.hq_quantize_fp8(dev_bf16(xb), H.E4M3, H.PER_TOKEN)
    torch.cuda.synchronize()
    qo, so, _ = O.quantize(xb, O.E4M3, O.PER_TOKEN)
    assert np.array_equal(host(q), qo) and np.array_equal(host(s), so)
    H.hq_check_device_error()
