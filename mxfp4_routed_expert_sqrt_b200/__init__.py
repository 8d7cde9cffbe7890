"""Python binding of libmoe.so (the C ABI in include/moe.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels
of libmoe.so.  PyTorch provides device memory and streams.  There is no CPU
fallback: importing works without a GPU, but every call needs the compiled
library and a CUDA device, and raises otherwise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_LIBRARY=debug selects libmoe_debug.so: the same kernels built with
# bounds checks on the indices they otherwise trust (moe_device_error()
# reports 0x501 / 0x502 instead of an out-of-bounds access).
LIB_PATH = os.path.join(_HERE, "libmoe_debug.so" if os.environ.get("MOE_LIBRARY") == "debug" else "libmoe.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_ALIGNMENT", 3: "MOE_ERR_UNSUPPORTED",
                4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_CUDA", 6: "MOE_ERR_DEVICE"}

# every symbol include/moe.h declares
EXPORTS = ("moe_abi_version", "moe_status_string", "moe_device_error", "moe_selftest_wait",
           "moe_route_workspace_size",
           "moe_route", "moe_route_noalloc", "moe_permute_workspace_size", "moe_permute",
           "moe_expert_gemm_workspace_size", "moe_expert_gemm_path", "moe_expert_gemm", "shared_expert_workspace_size",
           "shared_expert", "moe_combine")


class MoeError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


class moe_dims(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("route_scale", ctypes.c_float), ("swiglu_limit", ctypes.c_float)]


class moe_mxfp4_proj(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("expert_bytes", ctypes.c_int64), ("rows", ctypes.c_int32),
                ("cols", ctypes.c_int32)]


_lib = None
_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_sz = ctypes.c_size_t


def lib():
    """The loaded libmoe.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        dp = ctypes.POINTER(moe_dims)
        L.moe_abi_version.restype = ctypes.c_int
        L.moe_abi_version.argtypes = []
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_device_error.restype = ctypes.c_int32
        L.moe_device_error.argtypes = []
        L.moe_selftest_wait.restype = ctypes.c_int
        L.moe_selftest_wait.argtypes = [_i32, _vp]
        L.moe_route_workspace_size.restype = _sz
        L.moe_route_workspace_size.argtypes = [dp, _i32]
        L.moe_route.restype = ctypes.c_int
        L.moe_route.argtypes = [dp, _vp, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp]
        L.moe_route_noalloc.restype = ctypes.c_int
        L.moe_route_noalloc.argtypes = [dp, _vp, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp]
        L.moe_permute_workspace_size.restype = _sz
        L.moe_permute_workspace_size.argtypes = [_i32, _i32, _i32]
        L.moe_permute.restype = ctypes.c_int
        L.moe_permute.argtypes = [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_expert_gemm_workspace_size.restype = _sz
        L.moe_expert_gemm_workspace_size.argtypes = [dp, _i32]
        L.moe_expert_gemm_path.restype = _i32
        L.moe_expert_gemm_path.argtypes = [dp, _i32]
        L.moe_expert_gemm.restype = ctypes.c_int
        L.moe_expert_gemm.argtypes = [dp, _vp, _i32, moe_mxfp4_proj, moe_mxfp4_proj, moe_mxfp4_proj,
                                      _vp, _vp, _vp, _vp, _sz, _vp]
        L.shared_expert_workspace_size.restype = _sz
        L.shared_expert_workspace_size.argtypes = [dp, _i32]
        L.shared_expert.restype = ctypes.c_int
        L.shared_expert.argtypes = [dp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_combine.restype = ctypes.c_int
        L.moe_combine.argtypes = [dp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
        _lib = L
    return _lib


def _ptr(t):
    """Device (or host) address of a tensor, an int, or None (NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch
        if not torch.cuda.is_available():
            return 0  # the call then fails in CUDA unless it returns before any launch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn, st):
    if st != MOE_OK:
        raise MoeError(fn, st)


def dims_of(d) -> moe_dims:
    """moe_dims from any object with hidden/inter/n_experts/top_k/route_scale/swiglu_limit."""
    if isinstance(d, moe_dims):
        return d
    return moe_dims(d.hidden, d.inter, d.n_experts, d.top_k, d.route_scale, d.swiglu_limit)


def proj(base, rows: int, cols: int) -> moe_mxfp4_proj:
    """Projection descriptor of back-to-back MXFP4 expert blobs at `base`."""
    return moe_mxfp4_proj(_ptr(base), rows * cols // 2 + rows * cols // 32, rows, cols)


# ---- the C ABI, one wrapper per entry point ---------------------------------

def moe_abi_version() -> int:
    return lib().moe_abi_version()


def moe_device_error() -> int:
    return lib().moe_device_error()


# device error codes (moe_device_error)
DEVICE_ERR_BAD_EXPERT = 0x201
DEVICE_ERR_WAIT_TC = 0x301
DEVICE_ERR_SPAN_FLUSH = 0x302
DEVICE_ERR_F16_RANGE = 0x303
DEVICE_ERR_F16_SMALL = 0x304
DEVICE_ERR_WAIT_SELFTEST = 0x401
DEVICE_ERR_BAD_INDEX = 0x501     # debug build only
DEVICE_ERR_BAD_OFFSETS = 0x502   # debug build only


def moe_selftest_wait(wait_us: int, stream=None):
    """Enqueues the bounded-wait health check: a kernel that waits on a barrier
    nothing releases, gives up after wait_us and records device error 0x401."""
    _check("moe_selftest_wait", lib().moe_selftest_wait(wait_us, _stream(stream)))


def moe_route_workspace_size(dims, T) -> int:
    return lib().moe_route_workspace_size(ctypes.byref(dims_of(dims)), T)


def moe_route(dims, x, T, router_w, bias, token_ids, hash_table, vocab, topk_idx, topk_w, ws, ws_bytes,
              stream=None):
    _check("moe_route", lib().moe_route(ctypes.byref(dims_of(dims)), _ptr(x), T, _ptr(router_w), _ptr(bias),
                                        _ptr(token_ids), _ptr(hash_table), vocab, _ptr(topk_idx),
                                        _ptr(topk_w), _ptr(ws), ws_bytes, _stream(stream)))


ROUTE_NOALLOC_MAX_LOGITS = 65536


def moe_route_noalloc(dims, x, T, router_w, bias, token_ids, hash_table, vocab, topk_idx, topk_w, stream=None):
    """moe_route without a workspace, for callers that cannot allocate device
    memory: the logits go to a scratch array the library keeps on each
    device (T * n_experts <= ROUTE_NOALLOC_MAX_LOGITS).  Calls share that
    array, so calls that may overlap on the GPU must be ordered on one
    stream.  The first call on a device sets up the array's address and
    should come before any stream capture."""
    _check("moe_route_noalloc", lib().moe_route_noalloc(ctypes.byref(dims_of(dims)), _ptr(x), T, _ptr(router_w),
                                                        _ptr(bias), _ptr(token_ids), _ptr(hash_table), vocab,
                                                        _ptr(topk_idx), _ptr(topk_w), _stream(stream)))


def moe_permute_workspace_size(T, K, E) -> int:
    return lib().moe_permute_workspace_size(T, K, E)


def moe_permute(topk_idx, T, K, E, offsets, perm, inv, ws=None, ws_bytes=0, stream=None):
    _check("moe_permute", lib().moe_permute(_ptr(topk_idx), T, K, E, _ptr(offsets), _ptr(perm), _ptr(inv),
                                            _ptr(ws), ws_bytes, _stream(stream)))


def moe_expert_gemm_workspace_size(dims, T) -> int:
    return lib().moe_expert_gemm_workspace_size(ctypes.byref(dims_of(dims)), T)


def moe_expert_gemm_path(dims, T) -> str:
    """'block_scaled' or 'dequant': the path moe_expert_gemm takes for T tokens."""
    r = lib().moe_expert_gemm_path(ctypes.byref(dims_of(dims)), T)
    if r < 0:
        raise MoeError("moe_expert_gemm_path", -r)
    return "block_scaled" if r == 1 else "dequant"


def moe_expert_gemm(dims, x, T, gate, up, down, offsets, perm, y_perm, ws, ws_bytes, stream=None):
    _check("moe_expert_gemm", lib().moe_expert_gemm(ctypes.byref(dims_of(dims)), _ptr(x), T, gate, up, down,
                                                    _ptr(offsets), _ptr(perm), _ptr(y_perm), _ptr(ws),
                                                    ws_bytes, _stream(stream)))


def shared_expert_workspace_size(dims, T) -> int:
    return lib().shared_expert_workspace_size(ctypes.byref(dims_of(dims)), T)


def shared_expert(dims, x, T, wg, wu, wd, out, ws, ws_bytes, stream=None):
    _check("shared_expert", lib().shared_expert(ctypes.byref(dims_of(dims)), _ptr(x), T, _ptr(wg), _ptr(wu),
                                                _ptr(wd), _ptr(out), _ptr(ws), ws_bytes, _stream(stream)))


def moe_combine(dims, T, y_perm, inv, topk_w, shared_out, out_f32, out_bf16=None, stream=None):
    _check("moe_combine", lib().moe_combine(ctypes.byref(dims_of(dims)), T, _ptr(y_perm), _ptr(inv),
                                            _ptr(topk_w), _ptr(shared_out), _ptr(out_f32), _ptr(out_bf16),
                                            _stream(stream)))


# ---- the whole layer (a convenience over the five calls) --------------------

@dataclass
class LayerWeights:
    """Device tensors of one MoE layer (uint8 blobs, fp32 router, bf16 shared)."""
    gate: object      # uint8 [E * expert_bytes]
    up: object
    down: object
    router_w: object  # fp32 [E, H]
    bias: object = None       # fp32 [E] or None
    shared_gate: object = None  # bf16 [I, H]
    shared_up: object = None
    shared_down: object = None  # bf16 [H, I]
    hash_table: object = None   # int32 [vocab, K] for hash-routed layers


def _torch_stream(s):
    """A torch stream object for `s` (None: the current stream; an int: a raw
    cudaStream_t)."""
    import torch
    if s is None:
        return torch.cuda.current_stream()
    if isinstance(s, int):
        return torch.cuda.ExternalStream(s)
    return s


class MoeLayer:
    """Runs route -> permute -> experts -> combine for up to max_T tokens on
    the caller's stream, with the shared expert (which needs only x) on a
    side stream forked at the start of the layer and joined before the
    combine, so it overlaps routing and grouping.  Workspaces and
    intermediates are allocated once (torch) for max_T; a forward allocates
    nothing and can be captured in a CUDA graph."""

    def __init__(self, dims, max_T: int, device=None):
        import torch
        self.dims = dims_of(dims)
        self.max_T = max_T
        d = self.dims
        dev = torch.device("cuda") if device is None else device
        K, E, H = d.top_k, d.n_experts, d.hidden
        self.topk_idx = torch.empty(max_T * K, dtype=torch.int32, device=dev)
        self.topk_w = torch.empty(max_T * K, dtype=torch.float32, device=dev)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.perm = torch.empty(max_T * K, dtype=torch.int32, device=dev)
        self.inv = torch.empty(max_T * K, dtype=torch.int32, device=dev)
        self.y_perm = torch.empty(max_T * K * H, dtype=torch.float32, device=dev)
        self.shared_out = torch.empty(max_T * H, dtype=torch.float32, device=dev)
        self.ws_route_bytes = moe_route_workspace_size(d, max_T)
        self.ws_perm_bytes = moe_permute_workspace_size(max_T, K, E)
        self.ws_exp_bytes = moe_expert_gemm_workspace_size(d, max_T)
        self.ws_sh_bytes = shared_expert_workspace_size(d, max_T)
        self.ws_route = torch.empty(max(self.ws_route_bytes, 256), dtype=torch.uint8, device=dev)
        self.ws_perm = torch.empty(max(self.ws_perm_bytes, 256), dtype=torch.uint8, device=dev)
        self.ws_exp = torch.empty(max(self.ws_exp_bytes, 256), dtype=torch.uint8, device=dev)
        self.ws_sh = torch.empty(max(self.ws_sh_bytes, 256), dtype=torch.uint8, device=dev)
        self.side = torch.cuda.Stream(device=dev)  # the shared expert's stream

    def forward(self, w: LayerWeights, x, T: int, out_f32, token_ids=None, out_bf16=None, stream=None,
                expert_events=None):
        """One layer on T tokens of x (bf16 [T, H] on the device) into out_f32.

        expert_events: optional (start, end) CUDA events recorded around the
        routed-expert call (for timing it inside a captured step)."""
        d = self.dims
        H, I, E, K = d.hidden, d.inter, d.n_experts, d.top_k
        if T > self.max_T:
            raise ValueError(f"T={T} exceeds max_T={self.max_T}")
        import torch
        hashed = w.hash_table is not None
        vocab = w.hash_table.shape[0] if hashed else 0
        main = _torch_stream(stream)
        has_shared = w.shared_gate is not None
        if has_shared:
            # fork: the shared expert runs beside routing and grouping
            fork = torch.cuda.Event()
            fork.record(main)
            self.side.wait_event(fork)
            shared_expert(d, x, T, w.shared_gate, w.shared_up, w.shared_down, self.shared_out, self.ws_sh,
                          self.ws_sh_bytes, self.side)
            join = torch.cuda.Event()
            join.record(self.side)
        moe_route(d, x, T, w.router_w, None if hashed else w.bias, token_ids if hashed else None,
                  w.hash_table if hashed else None, vocab, self.topk_idx, self.topk_w, self.ws_route,
                  self.ws_route_bytes, main)
        moe_permute(self.topk_idx, T, K, E, self.offsets, self.perm, self.inv, self.ws_perm,
                    self.ws_perm_bytes, main)
        if expert_events is not None:
            expert_events[0].record(main)
        moe_expert_gemm(d, x, T, proj(w.gate, I, H), proj(w.up, I, H), proj(w.down, H, I), self.offsets,
                        self.perm, self.y_perm, self.ws_exp, self.ws_exp_bytes, main)
        if expert_events is not None:
            expert_events[1].record(main)
        if has_shared:
            main.wait_event(join)  # join
        moe_combine(d, T, self.y_perm, self.inv, self.topk_w, self.shared_out if has_shared else None,
                    out_f32, out_bf16, main)
        return out_f32

    def graphed(self, w: LayerWeights, T: int, host_x, host_out, token_ids=None, stream=None):
        """A callable that runs, as one CUDA graph on `stream`: the copy of
        host_x (pinned bf16 [T*H]) to the device, the layer, and the copy of
        the fp32 result into host_out (pinned [T*H]).  The caller
        synchronises the stream before reading host_out."""
        import torch
        d = self.dims
        dev = self.topk_idx.device
        x_dev = torch.empty(T * d.hidden, dtype=torch.bfloat16, device=dev)
        out_dev = torch.empty(T * d.hidden, dtype=torch.float32, device=dev)
        s = torch.cuda.Stream(device=dev) if stream is None else stream
        # one eager pass first (sets up the kernels' attributes outside capture)
        with torch.cuda.stream(s):
            x_dev.copy_(host_x, non_blocking=True)
            self.forward(w, x_dev, T, out_dev, token_ids=token_ids)
            host_out.copy_(out_dev, non_blocking=True)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            x_dev.copy_(host_x, non_blocking=True)
            self.forward(w, x_dev, T, out_dev, token_ids=token_ids)
            host_out.copy_(out_dev, non_blocking=True)
        keep = (x_dev, out_dev, host_x, host_out)

        def run():
            with torch.cuda.stream(s):
                g.replay()
            return keep[3]

        run.graph = g
        run.stream = s
        return run
