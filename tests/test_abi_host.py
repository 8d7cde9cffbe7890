"""Host-side checks of the C ABI (no GPU): exported symbols and argument errors.

Argument validation happens on the host before any launch, so these calls
return their status without touching a device.
"""
import ctypes
import os
import re

import pytest

import gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def m():
    import __graft_entry__
    __graft_entry__.build()
    import mxfp4_routed_expert_sqrt_b200 as pkg
    return pkg


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_\w+|shared_expert\w*)\s*\(", src)))


def test_header_declares_the_boundary_calls():
    names = _declared_functions()
    for f in ("moe_route", "moe_permute", "moe_expert_gemm", "moe_combine", "shared_expert"):
        assert f in names


def test_library_exports_every_declared_symbol(m):
    lib = ctypes.CDLL(m.LIB_PATH)
    names = _declared_functions()
    for n in names:
        assert hasattr(lib, n), f"libmoe.so does not export {n}"
    assert set(names) == set(m.EXPORTS)


def test_generator_library_exports(m):
    lib = ctypes.CDLL(os.path.join(ROOT, "gen", "libmoegen.so"))
    assert hasattr(lib, "moegen_fill_mxfp4")


def test_abi_version_and_status_strings(m):
    assert m.moe_abi_version() == 1
    for s in range(7):
        assert m.lib().moe_status_string(s)


def test_workspace_sizes(m):
    d = gen.V4
    assert m.moe_route_workspace_size(d, 4096) >= 4096 * 256 * 4
    assert m.moe_expert_gemm_workspace_size(d, 0) == 0
    assert m.moe_permute_workspace_size(4096, 6, 256) == 0


def _r256(n):
    return (n + 255) // 256 * 256


@pytest.mark.parametrize("dims,T", [(gen.V4, 1), (gen.V4, 64), (gen.V4, 1024), (gen.V4, 1025), (gen.V4, 4096),
                                    (gen.TINY, 8), (gen.TINY, 64), (gen.TINY, 65), (gen.TINY, 1000)])
def test_expert_gemm_workspace_covers_both_paths(m, dims, T):
    """The block-scaled path's layout (E4M3 terms and E8M0 scales of x, 2 terms,
    and of h, 3 terms) for every T: it is larger than the dequantising path's
    (x and h in f16), so the size grows with T across the switch from one path
    to the other (moe.h)."""
    H, I, E, K = dims.hidden, dims.inter, dims.n_experts, dims.top_k
    P = T * K
    want = _r256(2 * P * H) + _r256(2 * P * (H // 32)) + _r256(3 * P * I) + _r256(3 * P * (I // 32))
    assert want >= _r256(P * H * 2) + _r256(P * I * 2)
    assert m.moe_expert_gemm_workspace_size(dims, T) == want


def test_expert_gemm_workspace_grows_with_T(m):
    for dims in (gen.V4, gen.TINY):
        sizes = [m.moe_expert_gemm_workspace_size(dims, T) for T in range(0, 700)]
        assert all(a <= b for a, b in zip(sizes, sizes[1:]))


def test_argument_errors_return_before_launch(m):
    d = gen.V4
    fake = 1 << 40  # never dereferenced: validation fails first
    with pytest.raises(m.MoeError) as e:
        m.moe_route(d, None, 4, fake, None, None, None, 0, fake, fake, fake, 1 << 20, 0)
    assert e.value.status == 1
    with pytest.raises(m.MoeError) as e:  # misaligned x
        m.moe_route(d, fake + 2, 4, fake, None, None, None, 0, fake, fake, fake, 1 << 20, 0)
    assert e.value.status == 2
    with pytest.raises(m.MoeError) as e:  # workspace too small
        m.moe_route(d, fake, 4, fake, None, None, None, 0, fake, fake, fake, 16, 0)
    assert e.value.status == 4
    with pytest.raises(m.MoeError) as e:  # hash routing needs both pointers
        m.moe_route(d, fake, 4, fake, None, fake, None, 10, fake, fake, fake, 1 << 20, 0)
    assert e.value.status == 1
    bad = gen.Dims(hidden=4096 + 32, inter=2048, n_experts=256, top_k=6)
    with pytest.raises(m.MoeError) as e:
        m.moe_route(bad, fake, 4, fake, None, None, None, 0, fake, fake, fake, 1 << 30, 0)
    assert e.value.status == 3
    with pytest.raises(m.MoeError) as e:  # top_k > n_experts
        m.moe_route(gen.Dims(256, 128, 4, 6), fake, 4, fake, None, None, None, 0, fake, fake, fake, 1 << 20, 0)
    assert e.value.status == 3
    # T == 0 is a no-op
    m.moe_route(d, None, 0, None, None, None, None, 0, None, None, None, 0, 0)
    m.moe_combine(d, 0, None, None, None, None, None)
    m.moe_expert_gemm(d, None, 0, m.proj(None, 2048, 4096), m.proj(None, 2048, 4096), m.proj(None, 4096, 2048),
                      None, None, None, None, 0, 0)


def test_selftest_wait_rejects_out_of_range_waits(m):
    for bad in (0, -5, 2_000_001):
        with pytest.raises(m.MoeError) as e:
            m.moe_selftest_wait(bad, 0)
        assert e.value.status == 1


def test_projection_validation(m):
    d = gen.V4
    fake = 1 << 40
    g = m.proj(fake, 2048, 4096)
    dn = m.proj(fake, 4096, 2048)
    ws = m.moe_expert_gemm_workspace_size(d, 4)
    with pytest.raises(m.MoeError) as e:  # wrong orientation of down
        m.moe_expert_gemm(d, fake, 4, g, g, g, fake, fake, fake, fake, ws, 0)
    assert e.value.status == 1
    g_bad = m.proj(fake + 16, 2048, 4096)  # 16-byte but not 32-byte aligned
    with pytest.raises(m.MoeError) as e:
        m.moe_expert_gemm(d, fake, 4, g_bad, g, dn, fake, fake, fake, fake, ws, 0)
    assert e.value.status == 2
    g_sz = m.moe_mxfp4_proj(fake, 12345, 2048, 4096)
    with pytest.raises(m.MoeError) as e:
        m.moe_expert_gemm(d, fake, 4, g_sz, g, dn, fake, fake, fake, fake, ws, 0)
    assert e.value.status == 1
    with pytest.raises(m.MoeError) as e:
        m.moe_expert_gemm(d, fake, 4, g, g, dn, fake, fake, fake, fake, ws - 1, 0)
    assert e.value.status == 4


def test_permute_argument_errors(m):
    with pytest.raises(m.MoeError) as e:
        m.moe_permute(None, 4, 6, 2000, None, None, None)
    assert e.value.status == 1
    with pytest.raises(m.MoeError) as e:
        m.moe_permute(1 << 40, 1 << 21, 6, 256, 1 << 40, 1 << 40, 1 << 40)
    assert e.value.status == 3


def test_expert_path_choice(m):
    """moe_expert_gemm's path for T (host only): block-scaled up to 24 pairs
    per expert on average, dequantising above; bench.py's mirror of the switch
    (which labels its roofline line) agrees for every T."""
    import bench
    assert m.moe_expert_gemm_path(gen.V4, 1024) == "block_scaled"
    assert m.moe_expert_gemm_path(gen.V4, 1025) == "dequant"
    assert m.moe_expert_gemm_path(gen.TINY, 192) == "block_scaled"
    assert m.moe_expert_gemm_path(gen.TINY, 193) == "dequant"
    for dims in (gen.V4, gen.TINY):
        for T in list(range(0, 1300)) + [2048, 4096, 65536]:
            assert m.moe_expert_gemm_path(dims, T) == bench.expert_path(dims, T), (dims, T)
    with pytest.raises(m.MoeError):
        m.moe_expert_gemm_path(gen.V4, -1)
