"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Some callers -- a serving runtime that reserves the whole device for its own
pool at start-up, or code that must not call cudaMalloc on its hot path --
cannot provide moe_route's workspace.  moe_route_noalloc keeps its logits in a
scratch array inside the library instead.  This test calls it through the C
ABI twice in a row (the second call reuses the array left over from the first)
and checks both against moe_route on the same inputs: expert ids identical,
weights within the routing tolerance.  The file is named to be collected last.
"""
import numpy as np
import pytest

import gen
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


def test_noalloc_route_matches_workspace_route_twice():
    import __graft_entry__
    __graft_entry__.build()
    # two different batches, back to back through the shared scratch array
    cases = [make_case(gen.V4, 64, seed=3, with_shared=False),
             make_case(gen.V4, 37, seed=4, bias=gen.zipf_bias(4, 256, 0.08), with_shared=False)]
    for c in cases:
        dc = DeviceCase(c, DEV)
        ref_idx, ref_w = _route(dc, noalloc=False)
        got_idx, got_w = _route(dc, noalloc=True)
        assert np.array_equal(got_idx, ref_idx)
        assert np.abs(got_w - ref_w).max() <= W_TOL
    assert m.moe_device_error() == 0


def test_noalloc_route_rejects_oversized_batches():
    d = gen.V4
    T = m.ROUTE_NOALLOC_MAX_LOGITS // d.n_experts + 1
    fake = 1 << 40  # never dereferenced: the size check comes first
    with pytest.raises(m.MoeError) as e:
        m.moe_route_noalloc(d, fake, T, fake, None, None, None, 0, fake, fake)
    assert e.value.status == 3
