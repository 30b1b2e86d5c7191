"""Failure detection on the GPU without a fault: a bounded device-side wait
that nothing completes must give up, report W4A16_ERR_TIMEOUT through the
status word, and leave the CUDA context usable."""
import numpy as np
import pytest

import oracle
from gemm_w4a16_b200 import synth, w4a16
from tests.gpu_util import assert_close, pack_problem, to_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def test_bounded_wait_times_out_and_context_survives():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gemm_w4a16_b200 import build

    build.build()
    assert w4a16.device_status() == w4a16.OK
    w4a16.selftest_wait_timeout(2_000_000)          # about 1 ms of SM clock
    assert w4a16.device_status() == w4a16.ERR_TIMEOUT
    assert w4a16.device_status() == w4a16.OK        # read-and-clear
    p = synth.make_problem(256, 256, 3, seed=21)
    w, x = pack_problem(p)
    for path in (w4a16.PATH_GEMV, w4a16.PATH_TC):
        y = w4a16.gemm_ex(w, x, path=path)
        torch.cuda.synchronize()
        assert_close(to_f64(y), oracle.gemm(p.q, p.zeros, p.scales, p.x), f"after timeout path={path}")
    assert w4a16.device_status() == w4a16.OK
