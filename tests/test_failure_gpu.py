"""The device-side failure path, exercised without a GPU fault.

aqlm_selftest_bounded_wait launches a kernel whose wait (the bounded mbarrier wait
every matmul kernel uses) can never complete: it must give up after its limit,
record its site code in the library's status word and return, leaving the context
usable.  aqlm_check_device_status must report AQLM_ERR_TIMEOUT with that site once,
then be clean again, and a matmul afterwards must still be right.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from weight_only_additive_b200 import layer as L
from weight_only_additive_b200 import native, synth
from weight_only_additive_b200.native import Path, Status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    native.lib()
    torch.cuda.set_device(0)
    return torch.device("cuda", 0)


def test_bounded_wait_gives_up_and_reports(dev):
    st, _ = L.check_device_status()
    assert st == Status.OK  # start clean
    t0 = time.perf_counter()
    native.aqlm_selftest_bounded_wait(2000)  # 2 ms limit
    st, detail = L.check_device_status()
    elapsed = time.perf_counter() - t0
    assert st == Status.TIMEOUT and detail == native.SITE_SELFTEST, (st, hex(detail))
    assert elapsed < 5.0, elapsed
    # read-and-clear: the next check is clean
    st, detail = L.check_device_status()
    assert st == Status.OK, (st, hex(detail))


def test_context_usable_after_a_recorded_timeout(dev):
    native.aqlm_selftest_bounded_wait(1000)
    st, detail = L.check_device_status()
    assert st == Status.TIMEOUT and detail == native.SITE_SELFTEST
    for path, batch in ((Path.GEMV_LUT, 1), (Path.TENSOR_CORE, 16)):
        ld = synth.make_layer(2, 8, 8, 1024, 300, seed=60)
        x = synth.make_x(batch, 1024, seed=60)
        w = L.AqlmWeights.from_numpy(ld, dev)
        y = L.matmul(torch.from_numpy(x).to(dev), w, path=path).cpu().numpy().astype(np.float64)
        st, detail = L.check_device_status()
        assert st == Status.OK, (st, hex(detail))
        y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, None, 2, 8, 8)
        assert np.abs(y - y_ref).max() / np.abs(y_ref).max() <= 5e-3
