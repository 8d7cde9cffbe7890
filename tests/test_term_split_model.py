"""Error model of the activation encoding on the block-scaled expert path.

The decode path feeds the tensor cores E4M3 activation terms with E8M0
group-32 scales (term p encodes the residual of terms 0..p-1 with scale
2^(floor(log2 max|r|) - 7), round to nearest even).  The encoding is internal
to the kernel: its outputs are compared with the exact oracle under the layer
tolerance.  These tests pin the properties that the tolerance budget relies on,
on a numpy restatement of the encoding whose E4M3 rounding is checked against
torch's float8_e4m3fn conversion:
  - two terms carry a bf16 value exactly unless it is far below its group max;
  - three terms leave at most 2^-12 of the group max (h between the GEMMs);
  - two terms leave at most 2^-8 of the group max.
Each term leaves at most half an E4M3 step of 4 significant bits of its input,
i.e. at most 2^-4 of that input's group max, which gives both bounds.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")


def e4m3_rne(v):
    """Round to the nearest E4M3 value (bias 7, 3 mantissa bits, subnormal step
    2^-9), ties to even; |v| must stay below 464 (no saturation needed here)."""
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)  # subnormals share the exponent of the smallest normal
    ulp = 2.0 ** (e - 3)
    return np.round(v / ulp) * ulp  # np.round rounds halves to even


def split_terms(x, parts):
    """x [n, k] (k a multiple of 32) -> list of `parts` decoded terms."""
    n, k = x.shape
    r = x.reshape(n, k // 32, 32).astype(np.float64)
    terms = []
    for _ in range(parts):
        amax = np.abs(r).max(axis=2, keepdims=True)
        # E8M0 byte s = max(biased exponent of amax - 7, 0): scale 2^(s - 127)
        eb = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) + 127, 0)
        s = np.maximum(eb - 7, 0)
        scale = 2.0 ** (s - 127)
        q = e4m3_rne(r / scale)
        assert np.abs(q).max() <= 256  # |r| / scale < 256 rounds to at most 256 < 448
        t = q * scale
        terms.append(t.reshape(n, k))
        r = r - t
    return terms


def bf16_values(rng, n, k, sigma=1.0):
    a = rng.normal(0, sigma, (n, k)).astype(np.float32)
    b = a.view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16  # round to bf16, ties to even
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def test_e4m3_rounding_matches_torch():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-255, 255, 20000), rng.normal(0, 1e-2, 20000),
                        np.ldexp(rng.integers(-300, 300, 4000).astype(np.float64), -11)])
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(e4m3_rne(v.astype(np.float32).astype(np.float64)), ref)


def test_two_terms_carry_bf16_exactly():
    rng = np.random.default_rng(1)
    x = bf16_values(rng, 64, 4096)
    t = split_terms(x, 2)
    err = np.abs(t[0] + t[1] - x)
    gmax = np.repeat(np.abs(x.reshape(64, -1, 32)).max(axis=2), 32, axis=1)
    big = np.abs(x) >= 2.0 ** -12 * gmax
    assert big.mean() > 0.999
    assert err[big].max() == 0.0
    assert np.all(err <= 2.0 ** -20 * gmax)


@pytest.mark.parametrize("parts,bound", [(3, 2.0 ** -12), (2, 2.0 ** -8)])
def test_terms_of_fp32_values(parts, bound):
    rng = np.random.default_rng(2)
    # h-like values: a clamped-SwiGLU output spans about +-100 with many small values
    g = np.minimum(rng.normal(0, 4, (32, 2048)), 10.0)
    u = np.clip(rng.normal(0, 4, (32, 2048)), -10, 10)
    h = (g / (1 + np.exp(-g)) * u).astype(np.float32).astype(np.float64)
    t = split_terms(h, parts)
    err = np.abs(sum(t) - h)
    gmax = np.repeat(np.abs(h.reshape(32, -1, 32)).max(axis=2), 32, axis=1)
    assert np.all(err <= bound * gmax)
