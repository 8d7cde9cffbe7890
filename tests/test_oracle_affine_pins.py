"""Pins of the oracle's affine low-bit expert format (the oracle step of the
"DeepSeek-V4-Flash-0731-JANG" Dynamic affine recipe variant; its CUDA path is
not built).  No GPU needed.

The page gives the bits and group sizes per tensor role (2-bit G64 gate/up,
2-bit G32 down, 3-bit G64 gate in six layers, 8-bit G64 shared expert) and
the affine form; the packing (one little-endian bit stream per row) and the
bf16 scale / bias planes are this build's readings.  Each test below fails on
a plausible slip: a wrong bit order or group mapping, scale and bias swapped,
(q - zero) * scale instead of scale * q + bias, a transposed projection.
"""
import numpy as np
import pytest

from tests import indep


def _bf16_bits(v):
    return (np.asarray(v, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _random_blob(rng, rows, cols, bits, group):
    q = rng.integers(0, 1 << bits, size=(rows, cols))
    s = _bf16_bits(rng.uniform(0.01, 0.05, size=(rows, cols // group)))
    z = _bf16_bits(rng.uniform(-0.1, 0.1, size=(rows, cols // group)))
    return q, s, z, indep.affine_pack(q, s, z, bits)


RECIPE = [(2, 64), (2, 32), (3, 64), (8, 64)]


def test_affine_blob_bytes_and_shapes(oracle_lib):
    # 2-bit G64 gate/up [2048][4096], 2-bit G32 down [4096][2048], 3-bit G64
    # gate [2048][4096]: codes plus a bf16 scale and bias per group
    assert oracle_lib.affine_expert_bytes(2048, 4096, 2, 64) == 2_097_152 + 524_288
    assert oracle_lib.affine_expert_bytes(4096, 2048, 2, 32) == 2_097_152 + 1_048_576
    assert oracle_lib.affine_expert_bytes(2048, 4096, 3, 64) == 3_145_728 + 524_288
    assert oracle_lib.affine_expert_bytes(4096, 2048, 8, 64) == 8_388_608 + 524_288
    assert oracle_lib.affine_expert_bytes(64, 100, 2, 64) == -1  # cols not a multiple of the group
    assert oracle_lib.affine_expert_bytes(64, 128, 0, 64) == -1
    with pytest.raises(ValueError):
        oracle_lib.affine_dequant(np.zeros(64, np.uint8), 1, 100, 2, 64)


@pytest.mark.parametrize("bits,group", RECIPE)
def test_affine_dequant_matches_unpackbits(oracle_lib, bits, group):
    rng = np.random.default_rng(bits * 100 + group)
    rows, cols = 24, 256
    q, s, z, blob = _random_blob(rng, rows, cols, bits, group)
    assert blob.size == oracle_lib.affine_expert_bytes(rows, cols, bits, group)
    got = oracle_lib.affine_dequant(blob, rows, cols, bits, group)
    want = indep.affine_dequant_dense(blob, rows, cols, bits, group)
    assert np.array_equal(got, want)  # every value exact in fp64
    # and against the codes and planes the blob was packed from
    sf = indep.bf16_to_f64(s)
    zf = indep.bf16_to_f64(z)
    assert np.array_equal(got, np.repeat(sf, group, 1) * q + np.repeat(zf, group, 1))


@pytest.mark.parametrize("bits,group", RECIPE)
def test_affine_extreme_codes(oracle_lib, bits, group):
    rows, cols = 4, 128
    s = _bf16_bits(np.full((rows, cols // group), 0.25))
    z = _bf16_bits(np.full((rows, cols // group), -1.5))
    zero = oracle_lib.affine_dequant(indep.affine_pack(np.zeros((rows, cols), np.int64), s, z, bits),
                                     rows, cols, bits, group)
    assert np.all(zero == -1.5)  # q = 0: the bias alone
    top = oracle_lib.affine_dequant(indep.affine_pack(np.full((rows, cols), (1 << bits) - 1), s, z, bits),
                                    rows, cols, bits, group)
    assert np.all(top == 0.25 * ((1 << bits) - 1) - 1.5)  # scale * q + bias


@pytest.mark.parametrize("bits", [2, 3])
def test_affine_bit_order_is_pinned(oracle_lib, bits):
    rng = np.random.default_rng(7 + bits)
    rows, cols, group = 8, 128, 64
    q, s, z, blob = _random_blob(rng, rows, cols, bits, group)
    rev = sum(((q >> i) & 1) << (bits - 1 - i) for i in range(bits))  # each code's bits reversed
    got = oracle_lib.affine_dequant(blob, rows, cols, bits, group)
    other = oracle_lib.affine_dequant(indep.affine_pack(rev, s, z, bits), rows, cols, bits, group)
    assert not np.array_equal(got, other)


def test_affine_expert_ffn_equals_dense_numpy(oracle_lib):
    # the recipe's mix on a small expert: gate 3-bit G64, up 2-bit G64, down 2-bit G32
    rng = np.random.default_rng(11)
    H, I, limit = 128, 64, 10.0
    _, _, _, gb = _random_blob(rng, I, H, 3, 64)
    _, _, _, ub = _random_blob(rng, I, H, 2, 64)
    _, _, _, db = _random_blob(rng, H, I, 2, 32)
    xs = rng.standard_normal((5, H)) * 4
    got = oracle_lib.affine_expert_ffn((gb, 3, 64), (ub, 2, 64), (db, 2, 32), H, I, limit, xs)
    Wg = indep.affine_dequant_dense(gb, I, H, 3, 64)
    Wu = indep.affine_dequant_dense(ub, I, H, 2, 64)
    Wd = indep.affine_dequant_dense(db, H, I, 2, 32)
    want = indep.swiglu(xs @ Wg.T, xs @ Wu.T, limit) @ Wd.T
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    with pytest.raises(ValueError):  # a projection given the other one's shape
        oracle_lib.affine_expert_ffn((gb, 3, 64), (ub, 2, 64), (db, 2, 48), H, I, limit, xs)
