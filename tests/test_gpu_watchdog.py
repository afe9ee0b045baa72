"""GPU test of the failure path: a kernel's bounded wait that runs out (on a barrier nothing arrives
on) must surface as JF_ERR_TIMEOUT through jf_device_status, clear, and leave the context usable."""
import time

import numpy as np
import pytest
import torch

import int8_fully_quantized_b200 as jf
import oracle as O
from inputs import synthetic as S

from gpu_common import dev_f32, host

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert jf.jf_device_status() == 0
    t0 = time.monotonic()
    jf.jf_selftest_wait_timeout(200_000_000)          # 0.2 s
    assert jf.jf_device_status() == -7                 # JF_ERR_TIMEOUT
    assert time.monotonic() - t0 < 10.0
    assert jf.jf_device_status() == 0                  # read and cleared
    # the context is still usable: a kernel afterwards runs and is exact
    x = S.activation(np.random.default_rng(70), 64, 96, 2, 30.0)
    q, s = jf.quantize_block(dev_f32(x))
    qr, sr = O.quantize_block(x)
    assert np.array_equal(host(q), qr) and np.array_equal(host(s), sr)
    assert jf.jf_device_status() == 0


def test_selftest_argument_range():
    lib = jf.load_library()
    assert lib.jf_selftest_wait_timeout(10, None) == -10
