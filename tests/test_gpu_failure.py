"""Failure detection on the GPU (needs a B200): a bounded wait that never
completes reports COSMOT_ERR_TIMEOUT through the device status word, the
kernel returns, and the context keeps working.  Nothing faults or traps."""

import time

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from flow_matching_dit_cosmot_b200 import api as A  # noqa: E402
from flow_matching_dit_cosmot_b200 import _lib as L  # noqa: E402
from gpu_helpers import bits, to_dev  # noqa: E402


def test_a_wait_that_never_completes_reports_timeout_and_the_context_stays_usable():
    sh = A.stream_handle()
    L.cosmot_get_device_status(sh)  # start from a clear status word
    try:
        t0 = time.perf_counter()
        L.cosmot_selftest_wait_timeout(sh)
        torch.cuda.synchronize()
        waited = time.perf_counter() - t0
        st, where = L.cosmot_get_device_status(sh)
        assert (st, where) == (L.COSMOT_ERR_TIMEOUT, L.COSMOT_SITE_SELFTEST)
        assert 0.9 < waited < 30.0  # the one-second bound, not a hang
        assert L.cosmot_get_device_status(sh) == (0, 0)  # reading cleared it

        # The context still runs kernels: an Euler step on fresh buffers.
        x = to_dev(synth.normal_bf16((64, 128), 4500, 1))
        v = to_dev(synth.normal_bf16((64, 128), 4501, 1))
        x0 = bits(x).copy()
        L.cosmot_flow_euler_step(x.data_ptr(), 128, v.data_ptr(), 128, 0, 64, 128, 0.9, 0.5, sh)
        torch.cuda.synchronize()
        assert L.cosmot_get_device_status(sh)[0] == 0
        want = synth.bf16_to_f64(x0) - 0.4 * synth.bf16_to_f64(bits(v))
        got = synth.bf16_to_f64(bits(x))
        np.testing.assert_allclose(got, want, rtol=1e-2, atol=1e-2)
    finally:
        L.cosmot_get_device_status(sh)  # never leave a latched failure for later tests
