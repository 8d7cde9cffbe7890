"""Independent numpy formulations used to pin the oracle in tests.

These are written from the format and layer definitions with different
mechanics from the oracle (bitfield decode instead of a value table, dense
numpy matmuls over every expert instead of per-row sparse loops, library
softplus instead of the log1p form), so a slip in either shows up as a
mismatch.
"""
import numpy as np


def e2m1_bitfield(code: int) -> float:
    """OCP MX E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0."""
    s = (code >> 3) & 1
    ex = (code >> 1) & 3
    m = code & 1
    mag = (m * 0.5) if ex == 0 else (2.0 ** (ex - 1)) * (1.0 + 0.5 * m)
    return -mag if s else mag


E2M1_BITFIELD = np.array([e2m1_bitfield(c) for c in range(16)], dtype=np.float64)


def dequant_dense(blob: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Dense fp64 [rows, cols] from a blob, vectorised over the whole matrix."""
    nib = rows * cols // 2
    b = blob[:nib].reshape(rows, cols // 2)
    codes = np.empty((rows, cols), dtype=np.int64)
    codes[:, 0::2] = b & 0xF
    codes[:, 1::2] = b >> 4
    scales = blob[nib:nib + rows * cols // 32].reshape(rows, cols // 32).astype(np.int64)
    factor = np.power(2.0, (scales - 127).astype(np.float64))
    return E2M1_BITFIELD[codes] * np.repeat(factor, 32, axis=1)


def pack_blob(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Pack codes [rows, cols] (0..15) and exponents [rows, cols/32] into a blob."""
    rows, cols = codes.shape
    lo = codes[:, 0::2].astype(np.uint8)
    hi = codes[:, 1::2].astype(np.uint8)
    nib = (lo | (hi << 4)).reshape(-1)
    return np.concatenate([nib, scales.astype(np.uint8).reshape(-1)])


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def scores(x_bits, router_w):
    z = bf16_to_f64(x_bits) @ np.asarray(router_w, np.float64).T
    return np.sqrt(np.logaddexp(0.0, z))


def topk_sorted(biased_row: np.ndarray, K: int) -> np.ndarray:
    """Top-K ids in descending value, ties to the lower id (stable sort)."""
    return np.argsort(-biased_row, kind="stable")[:K]


def swiglu(g, u, limit):
    gc = np.minimum(g, limit)
    uc = np.clip(u, -limit, limit)
    return gc / (1.0 + np.exp(-gc)) * uc


def dense_layer(dims, x_bits, router_w, bias, gates, ups, downs, shared=None, tok=None, table=None):
    """Every expert on every token, then masked by the routing (brute force)."""
    H, I, E, K = dims.hidden, dims.inter, dims.n_experts, dims.top_k
    x = bf16_to_f64(x_bits)
    s = scores(x_bits, router_w)
    T = x.shape[0]
    mask = np.zeros((T, E))
    for t in range(T):
        if table is not None:
            ids = table[tok[t]]
        else:
            ids = topk_sorted(s[t] + (0.0 if bias is None else bias.astype(np.float64)), K)
        mask[t, ids] = dims.route_scale * s[t, ids] / s[t, ids].sum()
    out = np.zeros((T, H))
    for e in range(E):
        Wg = dequant_dense(gates[e], I, H)
        Wu = dequant_dense(ups[e], I, H)
        Wd = dequant_dense(downs[e], H, I)
        Y = swiglu(x @ Wg.T, x @ Wu.T, dims.swiglu_limit) @ Wd.T
        out += mask[:, e:e + 1] * Y
    if shared is not None:
        wg, wu, wd = (bf16_to_f64(a) for a in shared)
        out += swiglu(x @ wg.T, x @ wu.T, dims.swiglu_limit) @ wd.T
    return out, mask


def affine_dequant_dense(blob: np.ndarray, rows: int, cols: int, bits: int, group: int) -> np.ndarray:
    """Affine low-bit weights w = scale * q + bias, dense fp64 [rows, cols]:
    the code bit stream unpacked with numpy's little-endian unpackbits and
    weighted by powers of two (not extracted code by code), scales and biases
    read as bf16 planes."""
    cb = rows * cols * bits // 8
    b = np.asarray(blob, np.uint8)
    bitsarr = np.unpackbits(b[:cb].reshape(rows, cols * bits // 8), axis=1, bitorder="little")
    q = (bitsarr.reshape(rows, cols, bits).astype(np.int64) * (1 << np.arange(bits))).sum(axis=2)
    ng = rows * (cols // group)
    s = bf16_to_f64(b[cb:cb + 2 * ng].view(np.uint16)).reshape(rows, cols // group)
    z = bf16_to_f64(b[cb + 2 * ng:cb + 4 * ng].view(np.uint16)).reshape(rows, cols // group)
    return np.repeat(s, group, axis=1) * q + np.repeat(z, group, axis=1)


def affine_pack(q: np.ndarray, scale_bits: np.ndarray, bias_bits: np.ndarray, bits: int) -> np.ndarray:
    """Blob from codes [rows, cols] (0 .. 2^bits - 1) and bf16 scale / bias
    bits [rows, cols/G]: each code's bits spread LSB first with packbits."""
    rows, cols = q.shape
    bitmat = ((q[:, :, None] >> np.arange(bits)) & 1).astype(np.uint8).reshape(rows, cols * bits)
    codes = np.packbits(bitmat, axis=1, bitorder="little").reshape(-1)
    return np.concatenate([codes, np.asarray(scale_bits, np.uint16).reshape(-1).view(np.uint8),
                           np.asarray(bias_bits, np.uint16).reshape(-1).view(np.uint8)])
