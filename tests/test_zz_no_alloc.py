"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Some callers -- a serving runtime that reserves the whole device for its own
pool at start-up, or code that must not call cudaMalloc on its hot path --
cannot provide moe_route's workspace.  moe_route_noalloc keeps its logits in a
scratch array inside the library instead.  This test calls it through the C
ABI on three batches in a row (each call reuses the array the previous one
left behind), up to the largest batch the array holds at V4-Flash shape
(T = 256, where moe_route itself would take its tensor-core router), and
checks every call against the fp64 oracle: expert ids bit-exact (inputs are
redrawn until the 6th/7th score gap exceeds 1e-4; the smallest gap is
reported) and weights within 1e-5.  Batches one token above the limit are
refused before anything is enqueued.  The file is named to be collected last.
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

W_TOL = 1e-5
DEV = torch.device("cuda:0")


def _route(dc, noalloc):
    c = dc.case
    d, T, K = c.dims, c.T, c.dims.top_k
    idx = torch.full((T * K,), -1, dtype=torch.int32, device=DEV)
    w = torch.full((T * K,), -1.0, dtype=torch.float32, device=DEV)
    hashed = c.table is not None
    vocab = c.table.shape[0] if hashed else 0
    if noalloc:
        m.moe_route_noalloc(d, dc.x, T, dc.router, dc.bias, dc.tok, dc.table, vocab, idx, w)
    else:
        nb = m.moe_route_workspace_size(d, T)
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=DEV)
        m.moe_route(d, dc.x, T, dc.router, dc.bias, dc.tok, dc.table, vocab, idx, w, ws, nb)
    torch.cuda.synchronize()
    return idx.view(T, K).cpu().numpy(), w.view(T, K).cpu().numpy()


def test_noalloc_route_matches_the_oracle_on_consecutive_calls():
    import __graft_entry__
    __graft_entry__.build()
    t_max = m.ROUTE_NOALLOC_MAX_LOGITS // gen.V4.n_experts  # 256 at V4-Flash shape
    # three batches back to back through the one scratch array: the largest it
    # holds, one between the two routers of moe_route, one small with a bias
    cases = [make_case(gen.V4, t_max, seed=3, with_shared=False),
             make_case(gen.V4, 100, seed=5, with_shared=False),
             make_case(gen.V4, 37, seed=4, bias=gen.zipf_bias(4, 256, 0.08), with_shared=False)]
    for c in cases:
        dc = DeviceCase(c, DEV)
        got_idx, got_w = _route(dc, noalloc=True)
        ref_idx, ref_w, _, gap = oracle.route(c.x, c.router, c.bias, c.dims.top_k, c.dims.route_scale)
        assert gap.min() > 1e-4, f"T={c.T}: smallest 6th/7th gap {gap.min():.2e}"
        assert np.array_equal(got_idx, ref_idx), f"T={c.T}: ids differ (smallest gap {gap.min():.2e})"
        assert np.abs(got_w - ref_w).max() <= W_TOL
    assert m.moe_device_error() == 0


def test_noalloc_route_rejects_oversized_batches():
    d = gen.V4
    T = m.ROUTE_NOALLOC_MAX_LOGITS // d.n_experts + 1
    fake = 1 << 40  # never dereferenced: the size check comes first
    with pytest.raises(m.MoeError) as e:
        m.moe_route_noalloc(d, fake, T, fake, None, None, None, 0, fake, fake)
    assert e.value.status == 3
