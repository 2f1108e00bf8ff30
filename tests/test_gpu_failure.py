"""Failure detection without a GPU fault (needs a B200): the bounded pipeline
wait that every TMA / tensor-core kernel uses gives up on its own -- after its
time limit, or when another warp raises the abort flag -- and reports through
the device error word; the context stays usable afterwards."""
import numpy as np
import pytest
import torch

from parity import TOL, run_parity
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_347_b200 import pagedattn
    pagedattn.device_errors(clear=True)
    yield pagedattn
    pagedattn.device_errors(clear=True)


def test_wait_on_a_phase_nothing_completes_times_out(pa):
    took = pa.selftest_wait(0.02)
    assert 0.02 <= took < 1.0, took
    assert pa.device_errors(clear=True) == ["timeout"]


def test_abort_flag_ends_the_wait_early(pa):
    took = pa.selftest_wait(2.0, abort_after_s=0.005)
    assert 0.005 <= took < 0.5, took
    assert pa.device_errors(clear=True) == ["timeout"]


def test_context_usable_after_a_timeout(pa):
    pa.selftest_wait(0.01)
    assert pa.device_errors(clear=True) == ["timeout"]
    errs, _, _ = run_parity(workloads.tiny(), table_width=4)
    assert max(errs) <= TOL["f32"], errs
    assert pa.device_errors(clear=True) == []
