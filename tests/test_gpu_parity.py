"""GPU parity: every C-ABI call against the fp64 oracle on the same seeded inputs.

Tolerances (from the layer's acceptance bar): expert ids and the permutation
bit-exact (inputs are redrawn until the biased K-th/(K+1)-th score gap
exceeds 1e-4); routing weights |dw| <= 1e-5; float outputs
max|err| <= 1e-2 * RMS(ref) and sum|err| / sum|ref| <= 2e-3.
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

MAX_TOL, MEAN_TOL, W_TOL = 1e-2, 2e-3, 1e-5
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _build():
    import __graft_entry__
    __graft_entry__.build()
    yield
    assert m.moe_device_error() == 0


def _i32(n):
    return torch.empty(max(n, 1), dtype=torch.int32, device=DEV)


def _f32(n):
    return torch.empty(max(n, 1), dtype=torch.float32, device=DEV)


def _ws(n):
    return torch.empty(max(n, 256), dtype=torch.uint8, device=DEV), n


def run_route(dc):
    c = dc.case
    d, T, K = c.dims, c.T, c.dims.top_k
    idx, w = _i32(T * K), _f32(T * K)
    ws, nb = _ws(m.moe_route_workspace_size(d, T))
    hashed = c.table is not None
    m.moe_route(d, dc.x, T, dc.router, None if hashed else dc.bias, dc.tok, dc.table,
                c.table.shape[0] if hashed else 0, idx, w, ws, nb)
    torch.cuda.synchronize()
    return idx[:T * K].view(T, K).cpu().numpy(), w[:T * K].view(T, K).cpu().numpy()


def run_permute(idx_dev, T, K, E):
    off, perm, inv = _i32(E + 1), _i32(T * K), _i32(T * K)
    m.moe_permute(idx_dev, T, K, E, off, perm, inv)
    torch.cuda.synchronize()
    return off.cpu().numpy()[:E + 1], perm.cpu().numpy()[:T * K], inv.cpu().numpy()[:T * K]


# ---- inputs -----------------------------------------------------------------

def test_device_generator_matches_host():
    d = gen.V4
    c = make_case(gen.TINY, 4)
    dc = DeviceCase(c, DEV)
    eb = gen.blob_layout(gen.TINY.inter, gen.TINY.hidden)[2]
    g = dc.gate.cpu().numpy()
    for e in (0, 5, 15):
        assert np.array_equal(g[e * eb:(e + 1) * eb], c.blob("gate", e))
    dn = dc.down.cpu().numpy()
    assert np.array_equal(dn[3 * eb:4 * eb], c.blob("down", 3))
    # a V4-shape projection, two experts
    I, H = d.inter, d.hidden
    eb4 = gen.blob_layout(I, H)[2]
    buf = torch.empty(2 * eb4, dtype=torch.uint8, device=DEV)
    gen.mxfp4_fill_device(buf.data_ptr(), torch.cuda.current_stream().cuda_stream, 0, 0, "up", 2, I, H)
    b = buf.cpu().numpy()
    assert np.array_equal(b[eb4:], gen.mxfp4_expert_host(0, 0, "up", 1, I, H))
    # per-row exponent bases (the edge-case weights)
    gen.mxfp4_fill_device(buf.data_ptr(), torch.cuda.current_stream().cuda_stream, 3, 1, "down", 2, H, I, 0, 230, 6)
    b = buf.cpu().numpy()
    assert np.array_equal(b[eb4:], gen.mxfp4_expert_host(3, 1, "down", 1, H, I, 0, 230, 6))


# ---- routing ------------------------------------------------------------------

ROUTE_CASES = [
    ("tiny_T8", gen.TINY, 8, None, False),
    ("tiny_T37", gen.TINY, 37, None, False),
    ("v4_T1", gen.V4, 1, None, False),
    ("v4_T64", gen.V4, 64, None, False),
    ("v4_T64_bias", gen.V4, 64, "zipf", False),
    ("v4_T300", gen.V4, 300, None, False),          # T > 64: tensor-core logits
    ("v4_T1000_bias", gen.V4, 1000, "zipf", False),
    ("v4_hash_T64", gen.V4, 64, None, True),
    ("v4_hash_T500", gen.V4, 500, None, True),
]


@pytest.mark.parametrize("name,dims,T,bias,hashed", ROUTE_CASES, ids=[c[0] for c in ROUTE_CASES])
def test_route_parity(name, dims, T, bias, hashed):
    b = gen.zipf_bias(0, dims.n_experts, 0.08) if bias == "zipf" else None
    c = make_case(dims, T, bias=b, hashed=hashed, vocab=4096, with_shared=False)
    dc = DeviceCase(c, DEV)
    idx, w = run_route(dc)
    if hashed:
        ridx, rw = oracle.route_hash(c.x, c.router, dims.top_k, dims.route_scale, c.tok, c.table)
    else:
        ridx, rw, _, gap = oracle.route(c.x, c.router, c.bias, dims.top_k, dims.route_scale)
        assert gap.min() > 1e-4
    assert np.array_equal(idx, ridx), f"{name}: expert ids differ (redraws={c.redraws})"
    assert np.abs(w - rw).max() <= W_TOL
    assert np.allclose(w.sum(1), dims.route_scale, atol=1e-5)


# ---- grouping --------------------------------------------------------------------

# the largest calls moe_permute accepts: T*K up to 2^22 pairs, E up to 1024, K up to 32
@pytest.mark.parametrize("T,K,E,mode", [(0, 6, 256, "rand"), (1, 6, 256, "rand"), (64, 6, 256, "rand"),
                                        (4096, 6, 256, "rand"), (37, 2, 16, "rand"),
                                        (1000, 6, 256, "one_hot"), (2048, 6, 256, "skew"),
                                        (699050, 6, 256, "stride"), (131072, 32, 1024, "stride")])
def test_permute_parity(T, K, E, mode):
    rng = np.random.default_rng(T + E)
    if mode == "rand":
        idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]) if T else np.zeros((0, K))
    elif mode == "stride":  # K distinct ids per token: (r + k * s) mod E, s odd, E a power of two
        r = rng.integers(0, E, size=(T, 1))
        st = 2 * rng.integers(0, E // 2, size=(T, 1)) + 1
        idx = (r + np.arange(K)[None, :] * st) % E
    elif mode == "one_hot":  # every token picks the same K experts
        idx = np.tile(np.arange(K), (T, 1))
    else:  # Zipf-like popularity
        p = 1.0 / np.arange(1, E + 1) ** 1.1
        idx = np.stack([rng.choice(E, K, replace=False, p=p / p.sum()) for _ in range(T)])
    idx = idx.astype(np.int32)
    d_idx = torch.from_numpy(idx.reshape(-1).copy()).to(DEV) if T else _i32(1)
    off, perm, inv = run_permute(d_idx, T, K, E)
    roff, rperm, rinv = oracle.permute(idx, E)
    assert np.array_equal(off, roff)
    assert np.array_equal(perm, rperm)
    assert np.array_equal(inv, rinv)


def test_permute_reports_an_expert_id_out_of_range():
    # the kernel's own bounds check: the bad ids count as expert 0 and device
    # error 0x201 is recorded; every write stays inside the output buffers
    T, K, E = 64, 6, 256
    rng = np.random.default_rng(7)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    idx[3, 2] = E
    idx[40, 5] = -1
    assert m.moe_device_error() == 0
    off, perm, inv = run_permute(torch.from_numpy(idx.reshape(-1).copy()).to(DEV), T, K, E)
    assert m.moe_device_error() == m.DEVICE_ERR_BAD_EXPERT
    assert np.array_equal(np.sort(perm), np.arange(T * K))
    assert np.array_equal(inv[perm], np.arange(T * K))
    assert off[E] == T * K


# ---- experts, shared, combine -------------------------------------------------------

def _expert_gemm(dc, T):
    c = dc.case
    d = c.dims
    H, I, E, K = d.hidden, d.inter, d.n_experts, d.top_k
    idx, _ = run_route(dc)
    d_idx = torch.from_numpy(idx.reshape(-1).copy()).to(DEV)
    off, perm, inv = _i32(E + 1), _i32(T * K), _i32(T * K)
    m.moe_permute(d_idx, T, K, E, off, perm, inv)
    y = _f32(T * K * H)
    ws, nb = _ws(m.moe_expert_gemm_workspace_size(d, T))
    m.moe_expert_gemm(d, dc.x, T, m.proj(dc.gate, I, H), m.proj(dc.up, I, H), m.proj(dc.down, H, I),
                      off, perm, y, ws, nb)
    torch.cuda.synchronize()
    return idx, perm.cpu().numpy()[:T * K], y[:T * K * H].view(T * K, H).cpu().numpy()


# The call picks its path and token chunk from the mean pairs per expert: at
# most 24 runs the block-scaled kernel in 32-pair chunks (every case here up
# to v4_T1024 and the tiny T8/T37/T100 ones), more runs the dequantising
# kernel in 128-pair chunks (tiny T200/T1000, v4_T1025, the prefill size).
# The zipf case piles most pairs onto a few experts, so their groups span many
# 32-pair chunks, and it samples both sides of every chunk boundary of the
# most loaded expert.
EXPERT_CASES = [("tiny_T8", gen.TINY, 8, 64, None), ("tiny_T37", gen.TINY, 37, 74, None),
                ("v4_T1", gen.V4, 1, 6, None), ("v4_T8", gen.V4, 8, 48, None), ("v4_T37", gen.V4, 37, 24, None),
                ("v4_T64", gen.V4, 64, 24, None), ("tiny_T100", gen.TINY, 100, 200, None),
                ("tiny_T200_tc", gen.TINY, 200, 200, None), ("tiny_T1000_tc", gen.TINY, 1000, 120, None),
                ("v4_T96", gen.V4, 96, 24, None), ("v4_T300", gen.V4, 300, 24, None),
                ("v4_zipf_T256_chunks", gen.V4, 256, 16, "zipf"),
                # the two sides of the path switch: 24 pairs per expert on average
                # (the largest block-scaled call, many experts past one 32-pair
                # chunk), then 25 (the smallest dequantising one)
                ("v4_T1024_block_scaled_max", gen.V4, 1024, 32, None),
                ("v4_T1025_dequant_min", gen.V4, 1025, 24, None),
                # the prefill size: 256 pairs spread over the call plus every pair of
                # the four most loaded experts (each of their chunk positions)
                ("v4_T4096_prefill", gen.V4, 4096, 256, "chunks")]


@pytest.mark.parametrize("name,dims,T,nsample,bias", EXPERT_CASES, ids=[c[0] for c in EXPERT_CASES])
def test_expert_gemm_parity(name, dims, T, nsample, bias):
    c = make_case(dims, T, with_shared=False, bias=_zipf_bias() if bias == "zipf" else None)
    assert c.min_gap > 1e-4
    dc = DeviceCase(c, DEV)
    idx, perm, y = _expert_gemm(dc, T)
    K = dims.top_k
    rng = np.random.default_rng(1)
    positions = rng.choice(T * K, size=min(nsample, T * K), replace=False)
    if bias == "zipf":
        counts = np.bincount(idx.reshape(-1), minlength=dims.n_experts)
        hot = int(np.argmax(counts))
        assert counts[hot] > 2 * 32, f"{name}: the most loaded expert has only {counts[hot]} pairs"
        start = int(counts[:hot].sum())
        edges = [j for b in range(32, int(counts[hot]), 32) for j in (b - 1, b)] + [0, int(counts[hot]) - 1]
        positions = np.concatenate([positions, start + np.array(edges)])
    if bias == "chunks":
        # every position of a chunk: all pairs of the experts that hold the
        # sampled positions' neighbours at chunk starts, middles and ends
        counts = np.bincount(idx.reshape(-1), minlength=dims.n_experts)
        starts = np.concatenate([[0], np.cumsum(counts)])
        extra = []
        for e in np.argsort(-counts)[:4]:
            extra.extend(range(int(starts[e]), int(starts[e + 1])))
        positions = np.concatenate([positions, np.array(extra, np.int64)])
    positions = np.unique(positions)
    got = y[positions]
    want = oracle_pairs(c, idx, perm, positions)
    mx, mean = rel_errors(got, want)
    assert mx <= MAX_TOL and mean <= MEAN_TOL, f"{name}: max {mx:.2e} mean {mean:.2e}"


@pytest.mark.parametrize("dims,T", [(gen.TINY, 8), (gen.TINY, 100), (gen.V4, 1), (gen.V4, 8), (gen.V4, 64),
                                    (gen.V4, 65), (gen.V4, 300), (gen.V4, 4096)])
def test_shared_expert_parity(dims, T):
    c = make_case(dims, T)
    dc = DeviceCase(c, DEV)
    H, I = dims.hidden, dims.inter
    out = _f32(T * H)
    ws, nb = _ws(m.shared_expert_workspace_size(dims, T))
    m.shared_expert(dims, dc.x, T, dc.sg, dc.su, dc.sd, out, ws, nb)
    torch.cuda.synchronize()
    got = out[:T * H].view(T, H).cpu().numpy()
    sel = np.arange(T) if T <= 8 else np.linspace(0, T - 1, 8).astype(int)
    xs = (c.x[sel].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    want = oracle.shared_ffn(*c.shared, H, I, dims.swiglu_limit, xs)
    mx, mean = rel_errors(got[sel], want)
    assert mx <= MAX_TOL and mean <= MEAN_TOL, f"max {mx:.2e} mean {mean:.2e}"


@pytest.mark.parametrize("T,K,H,with_shared,with_bf16", [(1, 6, 4096, True, True), (37, 6, 4096, True, False),
                                                          (8, 2, 256, False, True)])
def test_combine_parity(T, K, H, with_shared, with_bf16):
    key = gen.derive(11, T, K, H)
    y = gen.normal(key, T * K * H).astype(np.float32).reshape(T * K, H)
    w = gen.uniform01(gen.derive(12, T), np.arange(T * K, dtype=np.uint64)).astype(np.float32).reshape(T, K)
    sh = gen.normal(gen.derive(13, T), T * H).astype(np.float32).reshape(T, H) if with_shared else None
    rng = np.random.default_rng(T)
    idx = np.stack([rng.permutation(16)[:K] for _ in range(T)]).astype(np.int32)
    _, _, inv = oracle.permute(idx, 16)
    dims = gen.Dims(hidden=H, inter=128, n_experts=16, top_k=K)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    out = _f32(T * H)
    ob = torch.empty(T * H, dtype=torch.bfloat16, device=DEV) if with_bf16 else None
    m.moe_combine(dims, T, t(y), t(inv), t(w), t(sh) if with_shared else None, out, ob)
    torch.cuda.synchronize()
    want = oracle.combine(y.astype(np.float64), inv, w.astype(np.float64),
                          None if sh is None else sh.astype(np.float64))
    got = out.view(T, H).cpu().numpy()
    assert np.allclose(got, want, rtol=1e-5, atol=1e-5 * np.abs(want).max())
    if with_bf16:
        assert torch.equal(ob, out.to(torch.bfloat16))


# ---- the whole layer -------------------------------------------------------------------

def _zipf_bias():
    import json
    import os
    k = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "zipf_kappa.json")))["kappa"]
    return gen.zipf_bias(0, gen.V4.n_experts, k)


LAYER_CASES = [("tiny_T8", gen.TINY, 8, None, False, 8), ("tiny_T1", gen.TINY, 1, None, False, 1),
               ("v4_zipf_T32_layer0", gen.V4, 32, "zipf", False, 8),
               ("v4_decode_T1", gen.V4, 1, None, False, 1), ("v4_decode_T8", gen.V4, 8, None, False, 8),
               ("v4_decode_T32", gen.V4, 32, None, False, 8), ("v4_decode_T64", gen.V4, 64, None, False, 8),
               ("v4_hash_T2048", gen.V4, 2048, None, True, 6), ("v4_prefill_T4096", gen.V4, 4096, None, False, 48),
               # degenerate routing: every table row names the same 6 experts, so all
               # 1,800 pairs land on them (ten 32-pair chunks each) and 250 experts are empty
               ("v4_hash_all_same_T300", gen.V4, 300, None, "same", 6)]


@pytest.mark.parametrize("name,dims,T,bias,hashed,nsample", LAYER_CASES, ids=[c[0] for c in LAYER_CASES])
def test_layer_parity(name, dims, T, bias, hashed, nsample):
    c = make_case(dims, T, hashed=bool(hashed), bias=_zipf_bias() if bias == "zipf" else None)
    if hashed == "same":
        c.table = np.ascontiguousarray(np.broadcast_to(c.table[0], c.table.shape))
    dc = DeviceCase(c, DEV)
    layer = m.MoeLayer(dims, T, DEV)
    out = _f32(T * dims.hidden)
    layer.forward(dc.weights, dc.x, T, out, token_ids=dc.tok)
    torch.cuda.synchronize()
    got = out.view(T, dims.hidden).cpu().numpy()
    sel = np.unique(np.linspace(0, T - 1, nsample).astype(np.int32))
    # only the experts the sampled tokens use are regenerated on the host
    if hashed:
        ridx, _ = oracle.route_hash(c.x[sel], c.router, dims.top_k, dims.route_scale, c.tok[sel], c.table)
    else:
        ridx, _, _, _ = oracle.route(c.x[sel], c.router, c.bias, dims.top_k, dims.route_scale)
    gb, ub, db = c.blobs_for(np.unique(ridx))
    want, _, _ = oracle.moe_layer(dims, c.x, sel, c.router, c.bias, gb, ub, db, shared=c.shared,
                                  tok=c.tok, table=c.table)
    mx, mean = rel_errors(got[sel], want)
    assert mx <= MAX_TOL and mean <= MEAN_TOL, f"{name}: max {mx:.2e} mean {mean:.2e}"
    assert m.moe_device_error() == 0
