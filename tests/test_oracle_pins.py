"""Pins of the fp64 oracle against the pages, closed forms and brute force.

No GPU needed.  Each test is chosen so that a plausible slip in the oracle (a
dropped term, a wrong sign, a swapped index, a transposed operand, a wrong
nibble or scale position) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import gen
from tests import indep

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --- element formats ---------------------------------------------------------

def test_e2m1_table_matches_bitfield_definition(oracle_lib):
    for code in range(16):
        v = oracle_lib.e2m1(code)
        ref = indep.e2m1_bitfield(code)
        assert v == ref
        assert math.copysign(1.0, v) == math.copysign(1.0, ref)  # -0 for code 8


def test_e8m0_anchors_and_doubling(oracle_lib):
    assert oracle_lib.e8m0(127) == 1.0
    assert oracle_lib.e8m0(128) == 2.0
    assert oracle_lib.e8m0(126) == 0.5
    assert oracle_lib.e8m0(0) == float.fromhex("0x1p-127")
    for e in range(0, 254):
        assert oracle_lib.e8m0(e + 1) == 2.0 * oracle_lib.e8m0(e)
    assert math.isnan(oracle_lib.e8m0(255))


def test_blob_bytes_reproduce_page_total(oracle_lib):
    """ElytronAI build card, Sizes: 138 routed projections x 256 experts."""
    g = json.load(open(os.path.join(GOLDEN, "pulsar_sizes.json")))
    cfg = json.load(open(os.path.join(GOLDEN, "v4_flash_moe_config.json")))
    H, I, E = cfg["hidden_size"], cfg["intermediate_size"], cfg["routed_experts"]
    gate = oracle_lib.expert_bytes(I, H)
    down = oracle_lib.expert_bytes(H, I)
    assert gate == down == 4_456_448
    assert g["routed_projections"] * E * gate == g["expert_payload_bytes"]
    assert gate % 32 == 0  # Layout: every tensor offset 32-byte aligned


def test_dequant_exhaustive_codes_and_scales(oracle_lib):
    rows, cols = 253, 32
    codes = np.tile(np.concatenate([np.arange(16), np.arange(16)[::-1]]), (rows, 1))
    scales = np.arange(rows).reshape(rows, 1)
    blob = indep.pack_blob(codes, scales)
    got = oracle_lib.dequant(blob, rows, cols)
    want = indep.E2M1_BITFIELD[codes] * np.power(2.0, scales - 127.0)
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))


def test_pack_unpack_roundtrip_random(oracle_lib):
    rng = np.random.default_rng(7)
    rows, cols = 24, 160
    codes = rng.integers(0, 16, size=(rows, cols))
    scales = rng.integers(100, 140, size=(rows, cols // 32))
    blob = indep.pack_blob(codes, scales)
    assert blob.size == oracle_lib.expert_bytes(rows, cols)
    got = oracle_lib.dequant(blob, rows, cols)
    assert np.array_equal(got, indep.dequant_dense(blob, rows, cols))
    # the nibble order matters: swapping the two nibbles of every byte changes it
    swapped = blob.copy()
    nib = rows * cols // 2
    swapped[:nib] = ((blob[:nib] & 0xF) << 4) | (blob[:nib] >> 4)
    assert not np.array_equal(oracle_lib.dequant(swapped, rows, cols), got)


def test_generated_blob_layout(oracle_lib):
    d = gen.TINY
    b = gen.mxfp4_expert_host(0, 0, "gate", 3, d.inter, d.hidden)
    assert b.size == oracle_lib.expert_bytes(d.inter, d.hidden)
    sc = b[d.inter * d.hidden // 2:]
    assert sc.min() >= gen.E8M0_LO and sc.max() <= gen.E8M0_HI
    # codes cover all 16 values
    nib = b[:d.inter * d.hidden // 2]
    assert len(np.unique(np.concatenate([nib & 15, nib >> 4]))) == 16


# --- scoring and routing -----------------------------------------------------

def test_sqrt_softplus_matches_library(oracle_lib):
    for z in np.linspace(-30, 30, 241):
        assert oracle_lib.sqrt_softplus(z) == pytest.approx(math.sqrt(np.logaddexp(0.0, z)), rel=1e-14)
    assert oracle_lib.sqrt_softplus(100.0) == pytest.approx(10.0, rel=1e-15)
    assert oracle_lib.sqrt_softplus(-800.0) == 0.0
    assert oracle_lib.sqrt_softplus(0.0) == pytest.approx(math.sqrt(math.log(2.0)), rel=1e-15)


def _tiny_inputs(T=24, seed=0, with_bias=False):
    d = gen.TINY
    x = gen.x_rows(seed, 0, T, d.hidden)
    wr = gen.router_weight(seed, 0, d.n_experts, d.hidden)
    bias = gen.zipf_bias(seed, d.n_experts, 0.05) if with_bias else None
    return d, x, wr, bias


@pytest.mark.parametrize("with_bias", [False, True])
def test_route_matches_bruteforce_sort(oracle_lib, with_bias):
    d, x, wr, bias = _tiny_inputs(T=40, with_bias=with_bias)
    idx, w, s, gap = oracle_lib.route(x, wr, bias, d.top_k, d.route_scale)
    s_ref = indep.scores(x, wr)
    assert np.allclose(s, s_ref, rtol=1e-13, atol=0)
    b = np.zeros(d.n_experts) if bias is None else bias.astype(np.float64)
    for t in range(x.shape[0]):
        want = indep.topk_sorted(s_ref[t] + b, d.top_k)
        assert list(idx[t]) == list(want)
        assert len(set(idx[t])) == d.top_k
        wt = d.route_scale * s_ref[t, want] / s_ref[t, want].sum()
        assert np.allclose(w[t], wt, rtol=1e-13, atol=0)
        assert abs(w[t].sum() - 1.5) < 1e-12
        others = np.setdiff1d(np.arange(d.n_experts), want)
        assert gap[t] == pytest.approx((s_ref[t] + b)[want[-1]] - (s_ref[t] + b)[others].max(), abs=1e-12)
        assert gap[t] >= 0


def test_bias_selects_but_does_not_weight(oracle_lib):
    """Aux-loss-free balancing: the bias moves the selection, not the weights."""
    d, x, wr, _ = _tiny_inputs(T=8)
    bias = np.zeros(d.n_experts, np.float32)
    bias[5] = 100.0  # expert 5 is always picked first
    idx, w, s, _ = oracle_lib.route(x, wr, bias, d.top_k, d.route_scale)
    assert (idx[:, 0] == 5).all()
    for t in range(8):
        assert w[t, 0] == pytest.approx(1.5 * s[t, 5] / s[t, idx[t]].sum(), rel=1e-14)


def test_route_equal_logits_gives_uniform_weights(oracle_lib):
    d = gen.TINY
    x = gen.x_rows(0, 0, 4, d.hidden)
    wr = np.tile(gen.router_weight(0, 0, 1, d.hidden), (d.n_experts, 1))
    idx, w, _, gap = oracle_lib.route(x, wr, None, d.top_k, d.route_scale)
    assert (idx == np.arange(d.top_k)).all()  # ties go to the lower id
    assert np.allclose(w, d.route_scale / d.top_k, rtol=1e-15)
    assert (gap == 0).all()


def test_route_k_equals_e_is_dense_mixture(oracle_lib):
    d, x, wr, _ = _tiny_inputs(T=6)
    idx, w, s, _ = oracle_lib.route(x, wr, None, d.n_experts, d.route_scale)
    for t in range(6):
        assert sorted(idx[t]) == list(range(d.n_experts))
        dense = np.zeros(d.n_experts)
        dense[idx[t]] = w[t]
        assert np.allclose(dense, 1.5 * s[t] / s[t].sum(), rtol=1e-14)


def test_hash_route_is_table_lookup(oracle_lib):
    d = gen.TINY
    x = gen.x_rows(0, 0, 32, d.hidden)
    wr = gen.router_weight(0, 0, d.n_experts, d.hidden)
    table = gen.hash_table(0, 1000, d.n_experts, d.top_k)
    tok = gen.token_ids(0, 0, 32, 1000)
    idx, w = oracle_lib.route_hash(x, wr, d.top_k, d.route_scale, tok, table)
    assert np.array_equal(idx, table[tok])
    s = indep.scores(x, wr)
    for t in range(32):
        assert np.allclose(w[t], 1.5 * s[t, idx[t]] / s[t, idx[t]].sum(), rtol=1e-13)


def test_hash_table_rows_distinct_and_uniform():
    table = gen.hash_table(0, 4096, 256, 6)
    assert all(len(set(r)) == 6 for r in table)
    counts = np.bincount(table.reshape(-1), minlength=256)
    assert counts.min() > 0.6 * counts.mean() and counts.max() < 1.4 * counts.mean()


# --- grouping ----------------------------------------------------------------

@pytest.mark.parametrize("T,K,E", [(1, 6, 256), (37, 2, 16), (500, 6, 256), (0, 6, 256)])
def test_permute_is_stable_counting_sort(oracle_lib, T, K, E):
    rng = np.random.default_rng(T)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32) if T else np.zeros((0, K), np.int32)
    off, perm, inv = oracle_lib.permute(idx, E)
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=E)
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(counts)]))
    assert np.array_equal(perm, np.argsort(flat, kind="stable"))
    assert np.array_equal(inv[perm], np.arange(T * K))
    for e in range(E):
        seg = perm[off[e]:off[e + 1]]
        assert (flat[seg] == e).all() and (np.diff(seg) > 0).all()


# --- expert FFN and the whole layer ------------------------------------------

def test_swiglu_limit_infinity_is_textbook(oracle_lib):
    for g, u in [(-3.0, 2.0), (0.5, -1.5), (7.0, 9.0), (40.0, -50.0)]:
        want = g / (1.0 + math.exp(-g)) * u
        assert oracle_lib.swiglu(g, u, 1e300) == pytest.approx(want, rel=1e-15)


def test_swiglu_clamps_one_sided_gate_two_sided_up(oracle_lib):
    L = 10.0
    # gate clamped above only, then silu; up clamped to [-L, L]
    assert oracle_lib.swiglu(15.0, 2.0, L) == pytest.approx(10.0 / (1 + math.exp(-10.0)) * 2.0, rel=1e-15)
    assert oracle_lib.swiglu(-15.0, 2.0, L) == pytest.approx(-15.0 / (1 + math.exp(15.0)) * 2.0, rel=1e-15)
    assert oracle_lib.swiglu(1.0, 25.0, L) == pytest.approx(1.0 / (1 + math.exp(-1.0)) * 10.0, rel=1e-15)
    assert oracle_lib.swiglu(1.0, -25.0, L) == pytest.approx(1.0 / (1 + math.exp(-1.0)) * -10.0, rel=1e-15)


def test_expert_ffn_all_ones_closed_form(oracle_lib):
    """Every code 2 (=1.0) with e=127: each weight row is all ones, so
    g = u = sum(x), h_i = swiglu(sum x, sum x) for all i and y_j = I * h."""
    H, I, L = 256, 128, 10.0
    g_blob = indep.pack_blob(np.full((I, H), 2), np.full((I, H // 32), 127))
    d_blob = indep.pack_blob(np.full((H, I), 2), np.full((H, I // 32), 127))
    rng = np.random.default_rng(1)
    xs = rng.normal(size=(5, H)) * 0.05
    xs[3] *= 40  # pushes the sum past the clamp
    ys = oracle_lib.expert_ffn(g_blob, g_blob, d_blob, H, I, L, xs)
    for j in range(5):
        sx = xs[j].sum()
        h = oracle_lib.swiglu(sx, sx, L)
        assert np.allclose(ys[j], I * h, rtol=1e-12, atol=1e-12)
    assert abs(xs[3].sum()) > L


def test_expert_ffn_matches_dense_numpy(oracle_lib):
    d = gen.TINY
    blobs = [gen.mxfp4_expert_host(0, 0, p, 2, *((d.inter, d.hidden) if p != "down" else (d.hidden, d.inter)))
             for p in ("gate", "up", "down")]
    # x4 so that the gate/up pre-activations (std ~10) reach the clamp
    xs = 4.0 * indep.bf16_to_f64(gen.x_rows(0, 0, 3, d.hidden))
    ys = oracle_lib.expert_ffn(*blobs, d.hidden, d.inter, d.swiglu_limit, xs)
    Wg = indep.dequant_dense(blobs[0], d.inter, d.hidden)
    Wu = indep.dequant_dense(blobs[1], d.inter, d.hidden)
    Wd = indep.dequant_dense(blobs[2], d.hidden, d.inter)
    want = indep.swiglu(xs @ Wg.T, xs @ Wu.T, d.swiglu_limit) @ Wd.T
    assert np.allclose(ys, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    # the clamp is exercised at this scale
    assert (np.abs(xs @ Wg.T) > d.swiglu_limit).any()


def test_shared_ffn_matches_dense_numpy(oracle_lib):
    H, I = 128, 64
    wg, wu, wd = (gen.normal_bf16(gen.derive(9, k), n, s).reshape(shape) for k, n, s, shape in
                  [(1, I * H, 1.0, (I, H)), (2, I * H, 1.0, (I, H)), (3, H * I, 0.1, (H, I))])
    xs = np.random.default_rng(3).normal(size=(4, H))
    ys = oracle_lib.shared_ffn(wg, wu, wd, H, I, 10.0, xs)
    g = xs @ indep.bf16_to_f64(wg).T
    u = xs @ indep.bf16_to_f64(wu).T
    want = indep.swiglu(g, u, 10.0) @ indep.bf16_to_f64(wd).T
    assert np.allclose(ys, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_combine_fixed_slot_order(oracle_lib):
    rng = np.random.default_rng(5)
    T, K, H = 7, 3, 16
    idx = np.stack([rng.permutation(8)[:K] for _ in range(T)]).astype(np.int32)
    off, perm, inv = oracle_lib.permute(idx, 8)
    y = rng.normal(size=(T * K, H))
    w = rng.random((T, K))
    sh = rng.normal(size=(T, H))
    out = oracle_lib.combine(y, inv, w, sh)
    want = sh + np.einsum("tk,tkh->th", w, y[inv].reshape(T, K, H))
    assert np.allclose(out, want, rtol=1e-14, atol=1e-14)


def _tiny_layer_blobs(seed=0, layer=0):
    d = gen.TINY
    gates = [gen.mxfp4_expert_host(seed, layer, "gate", e, d.inter, d.hidden) for e in range(d.n_experts)]
    ups = [gen.mxfp4_expert_host(seed, layer, "up", e, d.inter, d.hidden) for e in range(d.n_experts)]
    downs = [gen.mxfp4_expert_host(seed, layer, "down", e, d.hidden, d.inter) for e in range(d.n_experts)]
    return gates, ups, downs


@pytest.mark.parametrize("mode", ["learned", "learned_bias", "hashed"])
def test_tiny_layer_equals_dense_bruteforce(oracle_lib, mode):
    """Tiny config: every expert evaluated densely and masked by the routing.
    With a selection bias strong enough to change which experts win, the
    layer must route through it (a layer that dropped the bias on its way to
    the router would pick different experts and fail)."""
    d = gen.TINY
    T = 8
    x = gen.x_rows(0, 0, T, d.hidden)
    wr = gen.router_weight(0, 0, d.n_experts, d.hidden)
    gates, ups, downs = _tiny_layer_blobs()
    shared = gen.shared_weights(0, 0, d.hidden, d.inter)
    tok = table = bias = None
    if mode == "hashed":
        table = gen.hash_table(0, 64, d.n_experts, d.top_k)
        tok = gen.token_ids(0, 0, T, 64)
    if mode == "learned_bias":
        bias = gen.zipf_bias(0, d.n_experts, 0.6)
    out, idx, w = oracle_lib.moe_layer(d, x, np.arange(T), wr, bias, gates, ups, downs,
                                       shared=shared, tok=tok, table=table, nthreads=4)
    want, mask = indep.dense_layer(d, x, wr, bias, gates, ups, downs, shared=shared, tok=tok, table=table)
    assert np.allclose(out, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    for t in range(T):
        assert np.allclose(mask[t, idx[t]], w[t], rtol=1e-13)
    if mode == "learned_bias":
        # the bias changes the selection of some tokens, and the unbiased
        # layer differs from the biased one there
        nob, idx0, _ = oracle_lib.moe_layer(d, x, np.arange(T), wr, None, gates, ups, downs,
                                            shared=shared, nthreads=4)
        changed = [t for t in range(T) if set(idx0[t]) != set(idx[t])]
        assert changed, "the bias must change at least one token's experts"
        assert not np.allclose(nob[changed], out[changed])
    # a subset of tokens gives exactly those rows
    sub, _, _ = oracle_lib.moe_layer(d, x, np.array([5, 2]), wr, bias, gates, ups, downs,
                                     shared=shared, tok=tok, table=table, nthreads=2)
    assert np.array_equal(sub, out[[5, 2]])


def test_layer_missing_expert_blob_is_an_error(oracle_lib):
    d = gen.TINY
    x = gen.x_rows(0, 0, 2, d.hidden)
    wr = gen.router_weight(0, 0, d.n_experts, d.hidden)
    with pytest.raises(ValueError):
        oracle_lib.moe_layer(d, x, np.arange(2), wr, None, {}, {}, {}, nthreads=1)


def test_generator_row_bases():
    """The per-row exponent mode: every row's bytes lie within row_span of a
    base in [lo, hi - row_span], and the bases cover the range."""
    rows, cols = 64, 256
    blob = gen.mxfp4_expert_host(5, 0, "down", 3, rows, cols, 0, 230, 6)
    sc = blob[rows * cols // 2:].reshape(rows, cols // 32).astype(int)
    assert (sc.max(1) - sc.min(1) <= 6).all()
    assert sc.min() >= 0 and sc.max() <= 230
    assert sc.min(1).max() - sc.min(1).min() > 100  # bases spread over the range
    # the default mode is unchanged by the new parameter
    assert np.array_equal(gen.mxfp4_expert_host(5, 0, "down", 3, rows, cols),
                          gen.mxfp4_expert_host(5, 0, "down", 3, rows, cols, gen.E8M0_LO, gen.E8M0_HI, -1))
