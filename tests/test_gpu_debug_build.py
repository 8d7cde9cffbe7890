"""The bounds-checking debug build (libmoe_debug.so, -DMOE_DEBUG).

compute-sanitizer is not available on the GPU pool, so the library has a
debug build whose kernels check the indices they otherwise trust: the
grouped pair ids (perm, inv) and the group offsets.  A bad index records a
device error code and the access is skipped -- nothing traps and the context
stays usable.  Bad indices are fed ONLY to the debug library; the release
library is never given them.  Each case runs in a child process that selects
the debug library with MOE_LIBRARY=debug.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU container
    pytest.skip("needs a CUDA device", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import json, os, sys
sys.path.insert(0, os.environ["ROOT"])
import numpy as np
import torch
import gen
import mxfp4_routed_expert_sqrt_b200 as m
assert m.LIB_PATH.endswith("libmoe_debug.so"), m.LIB_PATH
dev = torch.device("cuda:0")
d = gen.TINY
H, I, E, K = d.hidden, d.inter, d.n_experts, d.top_k
res = {}
stream = torch.cuda.current_stream().cuda_stream
eb = I * H // 2 + I * H // 32
gate, up, down = (torch.empty(E * eb, dtype=torch.uint8, device=dev) for _ in range(3))
gen.mxfp4_fill_device(gate.data_ptr(), stream, 0, 0, "gate", E, I, H)
gen.mxfp4_fill_device(up.data_ptr(), stream, 0, 0, "up", E, I, H)
gen.mxfp4_fill_device(down.data_ptr(), stream, 0, 0, "down", E, H, I)

def expert_call(T, bad_perm=False, bad_offsets=False):
    rng = np.random.default_rng(T)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32).reshape(-1)
    order = np.argsort(idx, kind="stable").astype(np.int32)
    counts = np.bincount(idx, minlength=E)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    if bad_perm:
        order[3] = T * K + 5
    if bad_offsets:  # a group end before its start
        off[7] = off[8] + 2
    x = torch.from_numpy(gen.x_rows(0, 0, T, H).view(np.int16)).to(dev).view(torch.bfloat16)
    y = torch.zeros(T * K * H, dtype=torch.float32, device=dev)
    nb = m.moe_expert_gemm_workspace_size(d, T)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
    m.moe_expert_gemm(d, x, T, m.proj(gate, I, H), m.proj(up, I, H), m.proj(down, H, I),
                      torch.from_numpy(off).to(dev), torch.from_numpy(order).to(dev), y, ws, nb)
    torch.cuda.synchronize()
    return m.moe_device_error()

for T, path in ((8, "block_scaled"), (200, "dequant")):  # 1 and 25 pairs per expert
    res[f"{path}_valid"] = expert_call(T)
    res[f"{path}_bad_perm"] = expert_call(T, bad_perm=True)
    res[f"{path}_bad_offsets"] = expert_call(T, bad_offsets=True)
    res[f"{path}_valid_after"] = expert_call(T)

# combine with a slot index out of range
T = 4
y = torch.randn(T * K * H, device=dev)
w = torch.rand(T * K, device=dev)
inv = torch.arange(T * K, dtype=torch.int32, device=dev)
out = torch.empty(T * H, device=dev)
m.moe_combine(d, T, y, inv, w, None, out)
torch.cuda.synchronize()
res["combine_valid"] = m.moe_device_error()
inv[5] = T * K + 3
m.moe_combine(d, T, y, inv, w, None, out)
torch.cuda.synchronize()
res["combine_bad_inv"] = m.moe_device_error()
print(json.dumps(res))
'''


def test_debug_build_reports_bad_indices_without_faulting():
    import __graft_entry__
    __graft_entry__.build()  # builds libmoe_debug.so beside libmoe.so
    env = dict(os.environ, MOE_LIBRARY="debug", ROOT=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    for path in ("block_scaled", "dequant"):
        assert res[f"{path}_valid"] == 0
        assert res[f"{path}_bad_perm"] == 0x501
        assert res[f"{path}_bad_offsets"] == 0x502
        assert res[f"{path}_valid_after"] == 0  # the context is still usable
    assert res["combine_valid"] == 0
    assert res["combine_bad_inv"] == 0x501
