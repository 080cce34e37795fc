"""Failure detection without a GPU fault.

Every wait on a bulk copy in the kernels is bounded (2 s or 2^24 tries,
whichever comes first); when it gives up
the kernel sets DFW_ST_TIMEOUT in the device status word and returns, so the
host learns of it and the context stays usable.  dfw_selftest_wait_timeout
runs that wait on an mbarrier whose transaction nothing completes; corrupt
plans and streams (the other status bits) are covered with the decode tests.
"""
import time

import numpy as np
import pytest
import torch

import lossless_entropy_coded_canonical_b200 as dfw
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dfw.lib()
    dfw.check()


def test_bounded_wait_gives_up_and_reports_timeout():
    t0 = time.monotonic()
    assert dfw.lib().dfw_selftest_wait_timeout(None) == dfw.OK
    st, bits = dfw.status_bits()
    elapsed = time.monotonic() - t0
    assert st == dfw.ECORRUPT and bits == dfw.ST_TIMEOUT
    # the wait really waited, and stopped: its limit is 2 s or 2^24 tries, whichever comes first
    assert 0.1 < elapsed < 30.0, elapsed
    # the word was cleared, and the context still decodes correctly
    assert dfw.status_bits() == (dfw.OK, 0)
    u = np.concatenate([workloads.as_u16_numpy(t) for t in
                        workloads.generate_block(workloads.scaled(workloads.c3(), 200_000), "cpu")])
    enc = dfw.encode(u)
    out = dfw.decode_lanes(dfw.DeviceLanes.upload(enc, dfw.plan_lanes(enc), "cuda"))
    assert dfw.status_bits() == (dfw.OK, 0)
    assert np.array_equal(workloads.as_u16_numpy(out), u)


def test_corrupt_plan_sets_a_status_bit_not_timeout():
    u = np.concatenate([workloads.as_u16_numpy(t) for t in
                        workloads.generate_block(workloads.scaled(workloads.c3(), 300_000), "cpu")])
    enc = dfw.encode(u)
    pl = dfw.plan_lanes(enc)
    dl = dfw.DeviceLanes.upload(enc, pl, "cuda")
    dl.chunk_bits[5] += 1  # one chunk claims a bit more than it uses
    dfw.decode_lanes(dl)
    st, bits = dfw.status_bits()
    assert st == dfw.ECORRUPT and bits and not bits & dfw.ST_TIMEOUT
