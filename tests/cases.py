"""Seeded test cases shared by the GPU parity tests.

Inputs come from gen/ only.  Activation rows whose biased K-th/(K+1)-th score
gap is <= GAP_MIN under the fp64 oracle are redrawn from the next sub-stream
(attempt + 1) so expert selection is decided far from any rounding; the case
records how many rows were redrawn and the smallest remaining gap.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

import gen
import oracle

GAP_MIN = 1e-4


@dataclass
class Case:
    dims: gen.Dims
    T: int
    seed: int
    layer: int
    x: np.ndarray            # bf16 bits [T, H]
    router: np.ndarray       # fp32 [E, H]
    bias: np.ndarray | None  # fp32 [E]
    tok: np.ndarray | None   # int32 [T] (hash layers)
    table: np.ndarray | None
    shared: tuple            # bf16 bits (gate [I,H], up [I,H], down [H,I])
    redraws: int = 0
    min_gap: float = float("inf")
    e_range: tuple = (gen.E8M0_LO, gen.E8M0_HI)  # E8M0 exponents of the routed weights, per group
    _blobs: dict = field(default_factory=dict)

    def blob(self, proj: str, e: int) -> np.ndarray:
        key = (proj, e)
        if key not in self._blobs:
            d = self.dims
            rc = (d.inter, d.hidden) if proj != "down" else (d.hidden, d.inter)
            self._blobs[key] = gen.mxfp4_expert_host(self.seed, self.layer, proj, e, *rc, *self.e_range)
        return self._blobs[key]

    def blobs_for(self, experts):
        return tuple({int(e): self.blob(p, int(e)) for e in experts} for p in ("gate", "up", "down"))


def make_case(dims: gen.Dims, T: int, seed: int = 0, layer: int = 0, bias=None, hashed: bool = False,
              vocab: int = gen.HASH_VOCAB, with_shared: bool = True, e_range=None, x_edit=None) -> Case:
    """A seeded case.  e_range: (lo, hi) E8M0 exponents of the routed weights
    (default [118, 124]), or (lo, hi, row_span): a base per weight row in
    [lo, hi - row_span] plus [0, row_span] per group.  x_edit(t, row_bits) -> row_bits: applied to every
    drawn activation row (and to every redraw) before routing, to shape edge
    cases such as outlier channels or all-zero groups."""
    H, I, E, K = dims.hidden, dims.inter, dims.n_experts, dims.top_k
    router = gen.router_weight(seed, layer, E, H)
    attempts = np.zeros(T, np.int64)
    x = gen.x_rows(seed, layer, T, H, attempts)
    if x_edit is not None:
        for t in range(T):
            x[t] = x_edit(t, x[t])
    tok = table = None
    redraws, min_gap = 0, float("inf")
    if hashed:
        table = gen.hash_table(seed, vocab, E, K)
        tok = gen.token_ids(seed, layer, T, vocab)
    elif T > 0:
        for _ in range(50):
            _, _, _, gap = oracle.route(x, router, bias, K, dims.route_scale)
            bad = np.nonzero(gap <= GAP_MIN)[0]
            if len(bad) == 0:
                min_gap = float(gap.min())
                break
            redraws += len(bad)
            for t in bad:
                attempts[t] += 1
                x[t] = gen.normal_bf16(gen.derive(seed, layer, gen.T_X, int(t), int(attempts[t])), H)
                if x_edit is not None:
                    x[t] = x_edit(int(t), x[t])
        else:
            raise RuntimeError("could not redraw rows above the gap threshold")
    shared = gen.shared_weights(seed, layer, H, I) if with_shared else None
    c = Case(dims, T, seed, layer, x, router, bias, tok, table, shared, redraws, min_gap)
    if e_range is not None:
        c.e_range = tuple(e_range)
    return c


def rel_errors(got: np.ndarray, want: np.ndarray):
    """(max |err| / RMS(want), sum |err| / sum |want|)."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    rms = np.sqrt(np.mean(want ** 2))
    return float(err.max() / rms), float(err.sum() / np.abs(want).sum())


class DeviceCase:
    """Device tensors of a Case (weights filled on the device by gen)."""

    def __init__(self, case: Case, device="cuda"):
        import torch

        import mxfp4_routed_expert_sqrt_b200 as m
        self.case = case
        d = case.dims
        H, I, E = d.hidden, d.inter, d.n_experts
        dev = torch.device(device)
        self.dev = dev

        def t(a, dt):
            return torch.from_numpy(np.ascontiguousarray(a)).to(dev).view(dt)

        self.x = t(case.x.view(np.int16), torch.bfloat16)
        self.router = t(case.router, torch.float32)
        self.bias = None if case.bias is None else t(case.bias, torch.float32)
        self.tok = None if case.tok is None else t(case.tok, torch.int32)
        self.table = None if case.table is None else t(case.table, torch.int32)
        eb = I * H // 2 + I * H // 32
        stream = torch.cuda.current_stream().cuda_stream
        self.gate = torch.empty(E * eb, dtype=torch.uint8, device=dev)
        self.up = torch.empty(E * eb, dtype=torch.uint8, device=dev)
        self.down = torch.empty(E * eb, dtype=torch.uint8, device=dev)
        er = case.e_range
        gen.mxfp4_fill_device(self.gate.data_ptr(), stream, case.seed, case.layer, "gate", E, I, H, *er)
        gen.mxfp4_fill_device(self.up.data_ptr(), stream, case.seed, case.layer, "up", E, I, H, *er)
        gen.mxfp4_fill_device(self.down.data_ptr(), stream, case.seed, case.layer, "down", E, H, I, *er)
        if case.shared is not None:
            self.sg, self.su, self.sd = (t(a.view(np.int16), torch.bfloat16) for a in case.shared)
        else:
            self.sg = self.su = self.sd = None
        self.weights = m.LayerWeights(gate=self.gate, up=self.up, down=self.down, router_w=self.router,
                                      bias=self.bias, shared_gate=self.sg, shared_up=self.su,
                                      shared_down=self.sd, hash_table=self.table)


def bits_to_f64(x_bits: np.ndarray) -> np.ndarray:
    """bf16 bits -> fp64 values."""
    return (np.asarray(x_bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def oracle_pairs(case: Case, idx: np.ndarray, perm: np.ndarray, positions, nthreads: int = 16) -> np.ndarray:
    """fp64 oracle outputs of the grouped pairs at `positions` (rows of
    y_perm): each expert's sampled tokens go through one oracle call, and the
    experts run in parallel threads (the oracle is C and releases the GIL)."""
    from concurrent.futures import ThreadPoolExecutor

    K = case.dims.top_k
    d = case.dims
    xs_all = bits_to_f64(case.x)
    groups = {}
    for pos in positions:
        t, k = divmod(int(perm[pos]), K)
        groups.setdefault(int(idx[t, k]), []).append((int(pos), t))

    def run(e):
        items = groups[e]
        ys = oracle.expert_ffn(case.blob("gate", e), case.blob("up", e), case.blob("down", e), d.hidden, d.inter,
                               d.swiglu_limit, xs_all[[t for _, t in items]])
        return [(pos, ys[i]) for i, (pos, _) in enumerate(items)]

    want = {}
    with ThreadPoolExecutor(max_workers=nthreads) as ex:
        for res in ex.map(run, list(groups)):
            for pos, y in res:
                want[pos] = y
    return np.stack([want[int(p)] for p in positions])
