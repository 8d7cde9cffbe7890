"""Seeded synthetic input generators shared by the oracle's tests and the CUDA path.

This module holds no arithmetic of the MoE layer itself: it only draws random
bytes, integers and normals.  Both sides receive exactly the same bytes, so
any disagreement between the CUDA path and the oracle is in their arithmetic.

Random source: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014; constants as in Vigna's public-domain
reference `splitmix64.c`) used as a counter-based generator: output number
``i`` of stream ``key`` is ``mix64(key + (i + 1) * GOLDEN)``.  Integer outputs
are bit-identical here (numpy uint64) and on the device (``gen_device.cu``),
which is how 27 GB of expert weights can be filled on the GPU while the
oracle regenerates any single expert on the host.

Input recipe (the shapes and distributions of the V4-Flash workloads):
  * routed expert weights: E2M1 codes uniform over the 16 codes (each byte of
    the nibble plane uniform over 256), E8M0 exponents uniform over [lo, hi]
    (default [118, 124]), or, for edge cases, a uniform base per weight row
    plus a small uniform offset per group;
  * activations X ~ N(0, 1) rounded to bf16, one independent sub-stream per
    (token row, attempt) so a row can be redrawn;
  * router weight ~ N(0, 1/H) in fp32; shared-expert weights ~ N(0, 1/fan_in)
    in bf16;
  * hash table: K distinct uniform expert ids per token id (partial
    Fisher-Yates); token ids uniform over the vocabulary;
  * Zipf-style selection bias b_e = -kappa * ln(rank_e) with rank a seeded
    permutation of 1..E.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK = (1 << 64) - 1

# tensor ids of the sub-streams (part of the key derivation)
T_X, T_ROUTER, T_BIAS_RANK = 1, 2, 3
T_SHARED_GATE, T_SHARED_UP, T_SHARED_DOWN = 4, 5, 6
T_CODES = {"gate": 7, "up": 9, "down": 11}
T_SCALES = {"gate": 8, "up": 10, "down": 12}
T_HASH_TABLE, T_TOKEN_IDS, T_CALIB_X = 13, 14, 15
T_ROW_BASE = {"gate": 16, "up": 17, "down": 18}

E8M0_LO, E8M0_HI = 118, 124


def mix64_int(z: int) -> int:
    """SplitMix64 output function on a Python int (mod 2^64)."""
    z &= _MASK
    z = ((z ^ (z >> 30)) * _M1) & _MASK
    z = ((z ^ (z >> 27)) * _M2) & _MASK
    return z ^ (z >> 31)


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function, vectorised over a uint64 array."""
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= np.uint64(_M1)
        z ^= z >> np.uint64(27)
        z *= np.uint64(_M2)
        z ^= z >> np.uint64(31)
    return z


def derive(*ids: int) -> int:
    """Stream key for a tuple of non-negative ids (seed, layer, tensor, ...)."""
    k = 0x243F6A8885A308D3
    for i in ids:
        k = mix64_int(k ^ mix64_int((int(i) + GOLDEN) & _MASK))
    return k


def u64(key: int, counters: np.ndarray) -> np.ndarray:
    """Outputs number ``counters`` of the stream ``key`` (uint64 array)."""
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (c + np.uint64(1)) * np.uint64(GOLDEN)
    return mix64(z)


def uniform01(key: int, counters: np.ndarray) -> np.ndarray:
    """53-bit uniforms in [0, 1)."""
    return (u64(key, counters) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(key: int, n: int, start: int = 0) -> np.ndarray:
    """n standard normals (Box-Muller, fp64): normal i uses outputs 2i, 2i+1."""
    i = np.arange(start, start + n, dtype=np.uint64)
    r1 = u64(key, 2 * i)
    r2 = u64(key, 2 * i + np.uint64(1))
    u1 = ((r1 >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)  # (0, 1]
    u2 = (r2 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)          # [0, 1)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(key: int, n: int, sigma: float = 1.0) -> np.ndarray:
    """N(0, sigma^2) draws rounded fp64 -> fp32 -> bf16; uint16 bits."""
    return f32_to_bf16_bits((normal(key, n) * sigma).astype(np.float32))


def normal_f32(key: int, n: int, sigma: float = 1.0) -> np.ndarray:
    return (normal(key, n) * sigma).astype(np.float32)


# ----------------------------------------------------------------------------
# MXFP4 expert blobs: [rows][cols/2] nibble plane, then [rows][cols/32] E8M0.
# ----------------------------------------------------------------------------

def blob_layout(rows: int, cols: int):
    nib = rows * cols // 2
    sc = rows * cols // 32
    return nib, sc, nib + sc


def _below(r: np.ndarray, n: int) -> np.ndarray:
    """Integers in [0, n) from the high 32 bits of uint64 draws (multiply-shift)."""
    return ((r >> np.uint64(32)) * np.uint64(n)) >> np.uint64(32)


def mxfp4_expert_host(seed: int, layer: int, proj: str, x: int, rows: int, cols: int,
                      e_lo: int = E8M0_LO, e_hi: int = E8M0_HI, row_span: int = -1) -> np.ndarray:
    """Bytes of expert ``x`` of one projection, identical to the device fill.

    row_span < 0: every E8M0 byte uniform over [e_lo, e_hi].  row_span >= 0:
    each weight row draws a base uniform over [e_lo, e_hi - row_span] (from
    its own stream, counter = global row x * rows + r) and its bytes are the
    base plus a uniform offset in [0, row_span]."""
    nib, sc, total = blob_layout(rows, cols)
    assert nib % 8 == 0
    kc = derive(seed, layer, T_CODES[proj])
    ks = derive(seed, layer, T_SCALES[proj])
    out = np.empty(total, dtype=np.uint8)
    w0 = x * (nib // 8)
    out[:nib] = u64(kc, np.arange(w0, w0 + nib // 8, dtype=np.uint64)).view(np.uint8)
    r = u64(ks, np.arange(x * sc, (x + 1) * sc, dtype=np.uint64))
    if row_span < 0:
        out[nib:] = (np.uint64(e_lo) + _below(r, e_hi - e_lo + 1)).astype(np.uint8)
    else:
        kr = derive(seed, layer, T_ROW_BASE[proj])
        per_row = cols // 32
        grow = np.uint64(x * rows) + np.arange(sc, dtype=np.uint64) // np.uint64(per_row)
        base = np.uint64(e_lo) + _below(u64(kr, grow), e_hi - row_span - e_lo + 1)
        out[nib:] = (base + _below(r, row_span + 1)).astype(np.uint8)
    return out


_lib = None


def _load_device_lib():
    global _lib
    if _lib is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoegen.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(path)
        lib.moegen_fill_mxfp4.restype = ctypes.c_int
        lib.moegen_fill_mxfp4.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint64,
                                          ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_void_p]
        _lib = lib
    return _lib


def mxfp4_fill_device(dst_ptr: int, stream_ptr: int, seed: int, layer: int, proj: str,
                      n_experts: int, rows: int, cols: int,
                      e_lo: int = E8M0_LO, e_hi: int = E8M0_HI, row_span: int = -1) -> None:
    """Fill n_experts back-to-back blobs at device address dst_ptr on a stream
    (the same bytes as mxfp4_expert_host for every expert)."""
    lib = _load_device_lib()
    rc = lib.moegen_fill_mxfp4(ctypes.c_void_p(dst_ptr), n_experts, rows, cols,
                               derive(seed, layer, T_CODES[proj]),
                               derive(seed, layer, T_SCALES[proj]),
                               derive(seed, layer, T_ROW_BASE[proj]), e_lo, e_hi, row_span,
                               ctypes.c_void_p(stream_ptr))
    if rc != 0:
        raise RuntimeError(f"moegen_fill_mxfp4 failed with CUDA error {rc}")


# ----------------------------------------------------------------------------
# Dense tensors
# ----------------------------------------------------------------------------

def x_rows(seed: int, layer: int, T: int, H: int, attempts=None, tensor: int = T_X) -> np.ndarray:
    """Activations [T, H] as bf16 bits; row t uses sub-stream (t, attempts[t])."""
    out = np.empty((T, H), dtype=np.uint16)
    for t in range(T):
        a = 0 if attempts is None else int(attempts[t])
        out[t] = normal_bf16(derive(seed, layer, tensor, t, a), H)
    return out


def router_weight(seed: int, layer: int, E: int, H: int) -> np.ndarray:
    return normal_f32(derive(seed, layer, T_ROUTER), E * H, 1.0 / np.sqrt(H)).reshape(E, H)


def shared_weights(seed: int, layer: int, H: int, I: int):
    """(gate [I,H], up [I,H], down [H,I]) bf16 bits, N(0, 1/fan_in)."""
    g = normal_bf16(derive(seed, layer, T_SHARED_GATE), I * H, 1.0 / np.sqrt(H)).reshape(I, H)
    u = normal_bf16(derive(seed, layer, T_SHARED_UP), I * H, 1.0 / np.sqrt(H)).reshape(I, H)
    d = normal_bf16(derive(seed, layer, T_SHARED_DOWN), H * I, 1.0 / np.sqrt(I)).reshape(H, I)
    return g, u, d


def hash_table(seed: int, vocab: int, E: int, K: int) -> np.ndarray:
    """[vocab, K] int32: K distinct uniform ids per row (partial Fisher-Yates)."""
    key = derive(seed, 0, T_HASH_TABLE)
    perm = np.tile(np.arange(E, dtype=np.int32), (vocab, 1))
    rows = np.arange(vocab)
    for i in range(K):
        u = uniform01(key, rows.astype(np.uint64) * np.uint64(K) + np.uint64(i))
        j = i + np.minimum((u * (E - i)).astype(np.int64), E - i - 1)
        a = perm[rows, i].copy()
        perm[rows, i] = perm[rows, j]
        perm[rows, j] = a
    return np.ascontiguousarray(perm[:, :K])


def token_ids(seed: int, layer: int, n: int, vocab: int) -> np.ndarray:
    u = uniform01(derive(seed, layer, T_TOKEN_IDS), np.arange(n, dtype=np.uint64))
    return np.minimum((u * vocab).astype(np.int64), vocab - 1).astype(np.int32)


def bias_ranks(seed: int, E: int) -> np.ndarray:
    """A seeded permutation of 1..E (Fisher-Yates, SplitMix uniforms)."""
    key = derive(seed, 0, T_BIAS_RANK)
    r = np.arange(1, E + 1, dtype=np.int64)
    u = uniform01(key, np.arange(E, dtype=np.uint64))
    for i in range(E - 1, 0, -1):
        j = min(int(u[i] * (i + 1)), i)
        r[i], r[j] = r[j], r[i]
    return r


def zipf_bias(seed: int, E: int, kappa: float) -> np.ndarray:
    """b_e = -kappa * ln(rank_e) in fp32."""
    return (-kappa * np.log(bias_ranks(seed, E).astype(np.float64))).astype(np.float32)


# ----------------------------------------------------------------------------
# The workloads (shapes only)
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class Dims:
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    route_scale: float = 1.5
    swiglu_limit: float = 10.0


TINY = Dims(hidden=256, inter=128, n_experts=16, top_k=2)
V4 = Dims(hidden=4096, inter=2048, n_experts=256, top_k=6)

HASH_VOCAB = 131072
DECODE_BATCHES = (1, 8, 32, 64)
PREFILL_T = 4096
HASH_T = 2048
STACK_LAYERS = 8
STACK_BATCH = 32
ZIPF_S = 1.1
