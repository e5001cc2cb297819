"""Bounded waits: a wait that nothing completes runs out after the limit,
the host reads SVDQ_ERR_TIMEOUT, the error word is cleared by that read,
and the context stays usable (a layer run afterwards matches the oracle).

The failure is made with a barrier that no thread arrives at; no test here
faults, traps or hangs the GPU.
"""

import time

import pytest
import torch

from nvfp4_w4a4_quantized_smooth_b200 import synth

import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from nvfp4_w4a4_quantized_smooth_b200 import build
    build.build()
    torch.cuda.init()
    yield
    H.svdq().set_wait_timeout_ns(0)


def test_completed_wait_reports_nothing():
    s = H.svdq()
    s.check_device_error()
    s.wait_probe(True)
    s.check_device_error()


def test_wait_that_nothing_completes_times_out_and_clears():
    s = H.svdq()
    s.check_device_error()
    s.set_wait_timeout_ns(20_000_000)          # 20 ms
    try:
        t0 = time.perf_counter()
        s.wait_probe(False)
        with pytest.raises(s.SvdqError) as e:
            s.check_device_error()
        dt = time.perf_counter() - t0
        assert e.value.status == s.SVDQ_ERR_TIMEOUT
        assert 0.015 <= dt < 5.0, dt
        # the read cleared the word
        s.check_device_error()
    finally:
        s.set_wait_timeout_ns(0)


def test_context_usable_after_timeout():
    s = H.svdq()
    s.set_wait_timeout_ns(5_000_000)
    try:
        s.wait_probe(False)
        with pytest.raises(s.SvdqError):
            s.check_device_error()
    finally:
        s.set_wait_timeout_ns(0)
    L = synth.make_layer(300, 512, 384, seed=77)
    r = H.gpu_layer(L)
    y_ref, q_ref, a_ref, _ = H.oracle_y(L)
    H.assert_quant_exact(r["qact"], r["ascales"], q_ref, a_ref, "quant after timeout")
    H.assert_y_close(r["y"], y_ref, "y after timeout")
