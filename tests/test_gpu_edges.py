"""GPU parity at the edges of the number formats, on both expert paths.

Weights, E8M0 bytes far beyond the workloads' [118, 124]:
  * w_row_bases: every weight row draws its own base in [0, 224] and its
    groups lie within 6 octaves of it, so across rows every byte from 0 to
    230 occurs (230 keeps every fp32 intermediate of a V4-shape layer
    finite); every output is divided by 2^(m - 127), m the largest E8M0 byte
    of its row of the down projection, before the tolerance applies, so the
    small rows are held to the same bar as the large ones;
  * w_rows_small: every group in [100, 106], weights of about 2^-24 (every
    row's largest group far below 2^13, where a wrong exponent shift shows);
  * w_mixed_96_124: groups within a row 28 octaves apart.
  Spans much wider than that inside one row ([96, 140]) are ill-conditioned
  for any fp32 accumulator -- near the SwiGLU kink the rounding of g (a sum
  of terms ~1e6) moves h by O(1), and a down weight 2^44 above its row's
  others carries that to the output -- so they are not a parity case.
Activations: outlier channels a thousand times the rest, all-zero 32-value
groups, groups near 2^-20, and a few values beyond the f16 range
(|x| > 65504).  Each case runs moe_expert_gemm at a decode size (the
block-scaled path, stacked terms) and at T 1100 (26 pairs per expert, the
dequantising path), compares sampled pairs against the fp64 oracle at the
layer tolerance, and checks the device status the call leaves.  A whole layer with every
activation edge at once is checked at decode size (routing bit-exact through
the gap-redrawn inputs).
"""
import numpy as np
import pytest

import gen
import oracle
from tests.cases import DeviceCase, make_case, oracle_pairs, rel_errors

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU container
    pytest.skip("needs a CUDA device", allow_module_level=True)

import mxfp4_routed_expert_sqrt_b200 as m  # noqa: E402

MAX_TOL, MEAN_TOL = 1e-2, 2e-3
DEV = torch.device("cuda:0")
V4 = gen.V4


@pytest.fixture(scope="module", autouse=True)
def _build():
    import __graft_entry__
    __graft_entry__.build()
    assert m.moe_device_error() == 0
    yield
    assert m.moe_device_error() == 0


def _edit(fn):
    """Wraps an fp32 edit of one activation row as an edit of its bf16 bits."""
    def edit(t, row_bits):
        v = gen.bf16_bits_to_f32(row_bits).astype(np.float32)
        return gen.f32_to_bf16_bits(fn(t, v))
    return edit


OUTLIER_CH = np.array([5, 77, 1000, 2047, 2048, 3001, 4000, 4095])


def outliers(t, v):
    v[OUTLIER_CH] *= 1000.0
    return v


def zero_groups(t, v):
    v.reshape(-1, 32)[t % 4::4] = 0.0
    return v


def tiny_groups(t, v):
    v.reshape(-1, 32)[(t + 1) % 3::3] *= 2.0 ** -20
    return v


def beyond_f16(t, v):
    v[[t % 4096, (7 * t + 3) % 4096]] = (1.0e5, -2.5e5)
    return v


def all_edges(t, v):
    return beyond_f16(t, tiny_groups(t, zero_groups(t, outliers(t, v))))


def _expert_gemm(dc, T):
    c = dc.case
    d = c.dims
    H, I, E, K = d.hidden, d.inter, d.n_experts, d.top_k
    idx = torch.empty(T * K, dtype=torch.int32, device=DEV)
    w = torch.empty(T * K, dtype=torch.float32, device=DEV)
    nb = m.moe_route_workspace_size(d, T)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=DEV)
    m.moe_route(d, dc.x, T, dc.router, None, None, None, 0, idx, w, ws, nb)
    off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * K, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * K, dtype=torch.int32, device=DEV)
    m.moe_permute(idx, T, K, E, off, perm, inv)
    y = torch.empty(T * K * H, dtype=torch.float32, device=DEV)
    nb = m.moe_expert_gemm_workspace_size(d, T)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=DEV)
    m.moe_expert_gemm(d, dc.x, T, m.proj(dc.gate, I, H), m.proj(dc.up, I, H), m.proj(dc.down, H, I), off, perm,
                      y, ws, nb)
    torch.cuda.synchronize()
    return (idx.view(T, K).cpu().numpy(), perm.cpu().numpy(), y.view(T * K, H).cpu().numpy())


def _dequant_path(T):
    """The library's path choice (include/moe.h): more than 24 pairs per expert
    on average runs the dequantising kernel."""
    return -(-T * V4.top_k // V4.n_experts) > 24


# (name, e_range (lo, hi[, row_span]), x_edit, per_row_check)
EDGE_CASES = [
    ("w_row_bases", (0, 230, 6), None, True),   # checked per output row
    ("w_rows_small", (100, 106), None, False),
    ("w_mixed_96_124", (96, 124), None, False),
    ("x_outliers", None, outliers, False),
    ("x_zero_groups", None, zero_groups, False),
    ("x_tiny_groups", None, tiny_groups, False),
    ("x_beyond_f16", None, beyond_f16, False),
    ("x_all_edges", None, all_edges, False),
]


def _down_row_scales(c, idx, perm, positions):
    """2^-(m - 127) per sampled pair and output row, m = the largest E8M0 byte
    of that row of the pair's expert's down projection: the scale of that
    output element.  Dividing by it holds every output to the tolerance
    relative to its own row's magnitude (read from the format's scale plane)."""
    H, I, K = V4.hidden, V4.inter, V4.top_k
    nib = H * I // 2
    out = np.empty((len(positions), H))
    for i, pos in enumerate(positions):
        t, k = divmod(int(perm[pos]), K)
        sc = c.blob("down", int(idx[t, k]))[nib:nib + H * I // 32].reshape(H, I // 32)
        out[i] = np.ldexp(1.0, 127 - sc.max(axis=1).astype(np.int64))
    return out


@pytest.mark.parametrize("T", [8, 1100], ids=["decode_T8", "T1100"])
@pytest.mark.parametrize("name,e_range,x_edit,per_row", EDGE_CASES, ids=[c[0] for c in EDGE_CASES])
def test_expert_gemm_edges(name, e_range, x_edit, per_row, T):
    c = make_case(V4, T, seed=7, with_shared=False, e_range=e_range,
                  x_edit=None if x_edit is None else _edit(x_edit))
    dc = DeviceCase(c, DEV)
    idx, perm, y = _expert_gemm(dc, T)
    status = m.moe_device_error()
    K = V4.top_k
    rng = np.random.default_rng(T)
    positions = np.unique(rng.choice(T * K, size=min(48, T * K), replace=False))
    if _dequant_path(T) and x_edit in (beyond_f16, all_edges):
        # activations beyond f16 cannot enter the f16 MMAs: refused with a status
        assert status == m.DEVICE_ERR_F16_RANGE, hex(status)
        return
    if _dequant_path(T) and name == "w_rows_small":
        # weights of ~2^-24 give h ~1e-10: below f16's normal range, which the
        # dequantising path's f16 h cannot carry -- refused with a status
        assert status == m.DEVICE_ERR_F16_SMALL, hex(status)
        return
    assert status == 0, hex(status)
    got = y[positions]
    assert np.isfinite(got).all()
    want = oracle_pairs(c, idx, perm, positions)
    if per_row:
        f = _down_row_scales(c, idx, perm, positions)
        got, want = got * f, want * f
    mx, mean = rel_errors(got, want)
    assert mx <= MAX_TOL and mean <= MEAN_TOL, f"{name} T={T}: max {mx:.2e} mean {mean:.2e}"


def test_layer_with_every_activation_edge():
    T = 32
    c = make_case(V4, T, seed=9, e_range=(96, 124), x_edit=_edit(all_edges))
    assert c.min_gap > 1e-4
    dc = DeviceCase(c, DEV)
    layer = m.MoeLayer(V4, T, DEV)
    out = torch.empty(T * V4.hidden, dtype=torch.float32, device=DEV)
    layer.forward(dc.weights, dc.x, T, out)
    torch.cuda.synchronize()
    assert m.moe_device_error() == 0
    got = out.view(T, V4.hidden).cpu().numpy()
    sel = np.arange(0, T, 4)
    ridx, _, _, _ = oracle.route(c.x[sel], c.router, None, V4.top_k, V4.route_scale)
    gb, ub, db = c.blobs_for(np.unique(ridx))
    want, _, _ = oracle.moe_layer(V4, c.x, sel, c.router, None, gb, ub, db, shared=c.shared)
    mx, mean = rel_errors(got[sel], want)
    assert mx <= MAX_TOL and mean <= MEAN_TOL, f"max {mx:.2e} mean {mean:.2e}"


def test_dequant_path_flags_a_row_span_beyond_f16():
    """Groups 44 octaves apart inside a weight row (E8M0 bytes drawn per group
    from [96, 140]) cannot all be exact in f16 on the dequantising path: the
    groups more than 36 octaves below their row's largest are flushed and the
    call records 0x302 (include/moe.h).  The block-scaled path applies the
    scales in the MMA and records nothing.  (Such rows are ill-conditioned for
    any fp32 accumulator near the SwiGLU kink, so only the status is checked.)"""
    for T, want in ((1100, m.DEVICE_ERR_SPAN_FLUSH), (8, 0)):
        assert _dequant_path(T) == (want != 0)
        c = make_case(V4, T, seed=11, with_shared=False, e_range=(96, 140))
        dc = DeviceCase(c, DEV)
        _, _, y = _expert_gemm(dc, T)
        assert m.moe_device_error() == want, f"T={T}"
        if want == 0:
            assert np.isfinite(y).all()
