"""Failure detection on the GPU without a fault: a device-side wait that
nothing completes runs out at its time limit, sets LIME_FLAG_TIMEOUT in the
workspace's status word (read and cleared by lime_get_status), and the
context stays usable for the next call."""
import time

import pytest
import torch

from recsys_decoupled_link_b200 import lime

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports_it():
    dims = lime.make_dims(128, 4, 32, 256, 64, "bf16")
    ws = lime.Workspace(dims, 0, 0)
    assert lime.lime_get_status(ws) == 0
    t0 = time.perf_counter()
    lime.lime_debug_wait_timeout(ws)
    flags = lime.lime_get_status(ws)   # synchronises: the kernel has given up
    waited = time.perf_counter() - t0
    assert flags & lime.LIME_FLAG_TIMEOUT
    assert 1.0 < waited < 60.0
    assert lime.lime_get_status(ws) == 0   # the read cleared it
    # the context is still usable
    x = torch.arange(4096, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 4095 * 4096 / 2
