"""Failure detection without a GPU fault: the bounded-wait path.

Every pipeline kernel waits on mbarriers with a time bound; when a copy never
lands, the waiting role records a device error and the kernel returns.  Here
moe_selftest_wait runs that path on its own (a barrier nothing releases), and
the test checks that the error reaches the host through moe_device_error(),
that reading clears it, and that the device keeps working: a routing call on
the same context still matches the oracle.
"""
import numpy as np
import pytest

import gen
import oracle
from tests.cases import DeviceCase, make_case

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU container
    pytest.skip("needs a CUDA device", allow_module_level=True)

import mxfp4_routed_expert_sqrt_b200 as m  # noqa: E402

DEV = torch.device("cuda:0")


def test_wait_that_runs_out_reports_and_the_device_stays_usable():
    assert m.moe_device_error() == 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    m.moe_selftest_wait(20_000)  # 20 ms
    ev1.record()
    torch.cuda.synchronize()
    waited_ms = ev0.elapsed_time(ev1)
    assert 19.0 <= waited_ms < 1000.0, waited_ms  # gave up after its bound, not before
    assert m.moe_device_error() == m.DEVICE_ERR_WAIT_SELFTEST
    assert m.moe_device_error() == 0  # reading cleared it

    c = make_case(gen.TINY, 16, seed=3)
    dc = DeviceCase(c, DEV)
    d, T, K = c.dims, c.T, c.dims.top_k
    idx = torch.full((T * K,), -1, dtype=torch.int32, device=DEV)
    w = torch.zeros((T * K,), dtype=torch.float32, device=DEV)
    nb = m.moe_route_workspace_size(d, T)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=DEV)
    m.moe_route(d, dc.x, T, dc.router, dc.bias, dc.tok, dc.table, 0, idx, w, ws, nb)
    torch.cuda.synchronize()
    ridx, _, _, _ = oracle.route(c.x, c.router, c.bias, K, d.route_scale)
    assert np.array_equal(idx.view(T, K).cpu().numpy(), ridx)
    assert m.moe_device_error() == 0
