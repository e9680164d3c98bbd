"""Failure detection without a GPU fault: a bounded wait that nothing satisfies runs out,
the status word reports it, and the context stays usable for the next call."""
import time

import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    assert api.get_status() == 0
    t0 = time.time()
    assert api.selftest_wait_timeout(20000) == 0        # 20 ms bound
    assert api.get_status() == 6                        # FA_ERR_TIMEOUT, read and cleared
    assert time.time() - t0 < 5.0
    assert api.get_status() == 0                        # cleared
    # the context still works: a normal forward runs and reports no error
    inp = make_inputs(1, 1, 200, 64, seed=3)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, _ = api.fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    assert torch.isfinite(o.float()).all()


def test_status_site_names_the_wait_that_ran_out():
    assert api.get_status_site() == (0, 0)
    assert api.selftest_wait_timeout(20000) == 0
    assert api.get_status_site() == (6, 99)             # FA_ERR_TIMEOUT at the self-test's wait
    assert api.get_status_site() == (0, 0)              # read and cleared, site included


def test_selftest_rejects_bad_bound():
    assert api.selftest_wait_timeout(0) == 1
    assert api.selftest_wait_timeout(2_000_000) == 1
