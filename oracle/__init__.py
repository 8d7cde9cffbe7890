"""ctypes wrapper of the fp64 CPU oracle (oracle/moe_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
cpu_baseline / reference legs of bench.py.  The product package never imports
it, and it never imports the product package.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_fp = ctypes.POINTER(ctypes.c_float)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (strict IEEE fp64: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", _LIB, _SRC, "-lm"])
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_e2m1.restype = ctypes.c_double
        L.oracle_e2m1.argtypes = [ctypes.c_int]
        L.oracle_e8m0.restype = ctypes.c_double
        L.oracle_e8m0.argtypes = [ctypes.c_int]
        L.oracle_expert_bytes.restype = ctypes.c_int64
        L.oracle_expert_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
        L.oracle_sqrt_softplus.restype = ctypes.c_double
        L.oracle_sqrt_softplus.argtypes = [ctypes.c_double]
        L.oracle_swiglu.restype = ctypes.c_double
        L.oracle_swiglu.argtypes = [ctypes.c_double, ctypes.c_double, ctypes.c_double]
        L.oracle_dequant.restype = None
        L.oracle_dequant.argtypes = [_u8p, ctypes.c_int, ctypes.c_int, _dp]
        L.oracle_affine_expert_bytes.restype = ctypes.c_int64
        L.oracle_affine_expert_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int]
        L.oracle_affine_dequant.restype = ctypes.c_int
        L.oracle_affine_dequant.argtypes = [_u8p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp]
        L.oracle_affine_expert_ffn.restype = ctypes.c_int
        L.oracle_affine_expert_ffn.argtypes = [_u8p, ctypes.c_int, ctypes.c_int, _u8p, ctypes.c_int, ctypes.c_int,
                                               _u8p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_double, _dp, ctypes.c_int, _dp]
        L.oracle_route.restype = None
        L.oracle_route.argtypes = [_u16p, ctypes.c_int, ctypes.c_int, _fp, _fp, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_double, _ip, _dp, _dp, _dp]
        L.oracle_route_hash.restype = None
        L.oracle_route_hash.argtypes = [_u16p, ctypes.c_int, ctypes.c_int, _fp, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_double, _ip, _ip, ctypes.c_int,
                                        _ip, _dp]
        L.oracle_permute.restype = None
        L.oracle_permute.argtypes = [_ip, ctypes.c_int, ctypes.c_int, ctypes.c_int, _ip, _ip, _ip]
        L.oracle_expert_ffn.restype = None
        L.oracle_expert_ffn.argtypes = [_u8p, _u8p, _u8p, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_double, _dp, ctypes.c_int, _dp]
        L.oracle_shared_ffn.restype = None
        L.oracle_shared_ffn.argtypes = [_u16p, _u16p, _u16p, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_double, _dp, ctypes.c_int, _dp]
        L.oracle_combine.restype = None
        L.oracle_combine.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _ip, _dp, _dp, _dp]
        L.oracle_moe_layer.restype = ctypes.c_int
        L.oracle_moe_layer.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_double, ctypes.c_double, _u16p, ctypes.c_int,
                                       _ip, ctypes.c_int, _fp, _fp, _ip, _ip, ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_void_p),
                                       ctypes.POINTER(ctypes.c_void_p),
                                       ctypes.POINTER(ctypes.c_void_p),
                                       _u16p, _u16p, _u16p, ctypes.c_int, _dp, _ip, _dp]
        _lib = L
    return _lib


def _p(a, t):
    return None if a is None else a.ctypes.data_as(t)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def e2m1(code: int) -> float:
    return lib().oracle_e2m1(code)


def e8m0(e: int) -> float:
    return lib().oracle_e8m0(e)


def expert_bytes(rows: int, cols: int) -> int:
    return lib().oracle_expert_bytes(rows, cols)


def sqrt_softplus(z: float) -> float:
    return lib().oracle_sqrt_softplus(z)


def swiglu(g: float, u: float, limit: float) -> float:
    return lib().oracle_swiglu(g, u, limit)


def dequant(blob: np.ndarray, rows: int, cols: int) -> np.ndarray:
    blob = _c(blob, np.uint8)
    out = np.empty((rows, cols), dtype=np.float64)
    lib().oracle_dequant(_p(blob, _u8p), rows, cols, _p(out, _dp))
    return out


def affine_expert_bytes(rows: int, cols: int, bits: int, group: int) -> int:
    """Bytes of one affine-format expert blob (-1: a shape the format cannot hold)."""
    return lib().oracle_affine_expert_bytes(rows, cols, bits, group)


def affine_dequant(blob: np.ndarray, rows: int, cols: int, bits: int, group: int) -> np.ndarray:
    """W = scale * q + bias of an affine blob, fp64 [rows][cols]."""
    blob = _c(blob, np.uint8)
    out = np.empty((rows, cols), dtype=np.float64)
    if lib().oracle_affine_dequant(_p(blob, _u8p), rows, cols, bits, group, _p(out, _dp)) != 0:
        raise ValueError("affine_dequant: bad shape")
    return out


def affine_expert_ffn(g, u, d, H, I, limit, xs):
    """One affine expert on xs[n][H]; g, u, d = (blob, bits, group)."""
    xs = _c(xs, np.float64)
    n = xs.shape[0]
    ys = np.empty((n, H), np.float64)
    (gb, gbits, ggr), (ub, ubits, ugr), (db, dbits, dgr) = ((_c(b, np.uint8), bi, gr) for b, bi, gr in (g, u, d))
    if lib().oracle_affine_expert_ffn(_p(gb, _u8p), gbits, ggr, _p(ub, _u8p), ubits, ugr, _p(db, _u8p), dbits, dgr,
                                      H, I, limit, _p(xs, _dp), n, _p(ys, _dp)) != 0:
        raise ValueError("affine_expert_ffn: bad shape")
    return ys


def route(x_bits, router_w, bias, K, alpha):
    """Learned routing: returns (idx [T,K] int32, w [T,K], scores [T,E], gap [T])."""
    x_bits = _c(x_bits, np.uint16)
    router_w = _c(router_w, np.float32)
    bias = _c(bias, np.float32)
    T, H = x_bits.shape
    E = router_w.shape[0]
    idx = np.empty((T, K), np.int32)
    w = np.empty((T, K), np.float64)
    s = np.empty((T, E), np.float64)
    gap = np.empty(T, np.float64)
    lib().oracle_route(_p(x_bits, _u16p), T, H, _p(router_w, _fp), _p(bias, _fp), E, K, alpha,
                       _p(idx, _ip), _p(w, _dp), _p(s, _dp), _p(gap, _dp))
    return idx, w, s, gap


def route_hash(x_bits, router_w, K, alpha, tok, table):
    x_bits = _c(x_bits, np.uint16)
    router_w = _c(router_w, np.float32)
    tok = _c(tok, np.int32)
    table = _c(table, np.int32)
    T, H = x_bits.shape
    E = router_w.shape[0]
    idx = np.empty((T, K), np.int32)
    w = np.empty((T, K), np.float64)
    lib().oracle_route_hash(_p(x_bits, _u16p), T, H, _p(router_w, _fp), E, K, alpha,
                            _p(tok, _ip), _p(table, _ip), table.shape[0], _p(idx, _ip), _p(w, _dp))
    return idx, w


def permute(idx, E):
    idx = _c(idx, np.int32)
    T, K = idx.shape
    off = np.empty(E + 1, np.int32)
    perm = np.empty(T * K, np.int32)
    inv = np.empty(T * K, np.int32)
    lib().oracle_permute(_p(idx, _ip), T, K, E, _p(off, _ip), _p(perm, _ip), _p(inv, _ip))
    return off, perm, inv


def expert_ffn(g_blob, u_blob, d_blob, H, I, limit, xs):
    xs = _c(xs, np.float64)
    n = xs.shape[0]
    ys = np.empty((n, H), np.float64)
    g_blob, u_blob, d_blob = (_c(b, np.uint8) for b in (g_blob, u_blob, d_blob))
    lib().oracle_expert_ffn(_p(g_blob, _u8p), _p(u_blob, _u8p), _p(d_blob, _u8p), H, I, limit,
                            _p(xs, _dp), n, _p(ys, _dp))
    return ys


def shared_ffn(wg, wu, wd, H, I, limit, xs):
    xs = _c(xs, np.float64)
    n = xs.shape[0]
    ys = np.empty((n, H), np.float64)
    wg, wu, wd = (_c(b, np.uint16) for b in (wg, wu, wd))
    lib().oracle_shared_ffn(_p(wg, _u16p), _p(wu, _u16p), _p(wd, _u16p), H, I, limit,
                            _p(xs, _dp), n, _p(ys, _dp))
    return ys


def combine(y_perm, inv, w, shared):
    y_perm = _c(y_perm, np.float64)
    inv = _c(inv, np.int32)
    w = _c(w, np.float64)
    shared = _c(shared, np.float64)
    T, K = w.shape
    H = y_perm.shape[1]
    out = np.empty((T, H), np.float64)
    lib().oracle_combine(T, K, H, _p(y_perm, _dp), _p(inv, _ip), _p(w, _dp), _p(shared, _dp),
                         _p(out, _dp))
    return out


def moe_layer(dims, x_bits, sel, router_w, bias, gate_blobs, up_blobs, down_blobs,
              shared=None, tok=None, table=None, nthreads=None):
    """Layer output rows for tokens ``sel`` (fp64), plus their routing.

    gate_blobs/up_blobs/down_blobs: dict or list expert -> uint8 blob (only the
    experts used by the selected tokens are needed).  shared: (wg, wu, wd) bf16
    bits or None.  tok/table: hash routing when both are given.
    """
    L = lib()
    H, I, E, K = dims.hidden, dims.inter, dims.n_experts, dims.top_k
    x_bits = _c(x_bits, np.uint16)
    sel = _c(sel, np.int32)
    n = len(sel)
    router_w = _c(router_w, np.float32)
    bias = _c(bias, np.float32)
    tok = _c(tok, np.int32)
    table = _c(table, np.int32)
    keep = []

    def ptrs(blobs):
        arr = (ctypes.c_void_p * E)()
        for e in range(E):
            b = blobs.get(e) if isinstance(blobs, dict) else (blobs[e] if e < len(blobs) else None)
            if b is not None:
                b = _c(b, np.uint8)
                keep.append(b)
                arr[e] = b.ctypes.data
        return arr

    gp, up_, dp = ptrs(gate_blobs), ptrs(up_blobs), ptrs(down_blobs)
    wg = wu = wd = None
    if shared is not None:
        wg, wu, wd = (_c(b, np.uint16) for b in shared)
    out = np.empty((n, H), np.float64)
    idx = np.empty((n, K), np.int32)
    w = np.empty((n, K), np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = L.oracle_moe_layer(H, I, E, K, dims.route_scale, dims.swiglu_limit,
                            _p(x_bits, _u16p), x_bits.shape[0], _p(sel, _ip), n,
                            _p(router_w, _fp), _p(bias, _fp), _p(tok, _ip), _p(table, _ip),
                            0 if table is None else table.shape[0], gp, up_, dp,
                            _p(wg, _u16p), _p(wu, _u16p), _p(wd, _u16p), nthreads,
                            _p(out, _dp), _p(idx, _ip), _p(w, _dp))
    if rc != 0:
        raise ValueError("oracle_moe_layer: a selected token uses an expert whose blob was not given")
    return out, idx, w
