"""B200 (sm_100a) forward pass of one sparse Mixture-of-Experts layer.

A thin ctypes binding over the C ABI of ``libmoe.so`` (declared in
``include/moe.h``). The functions here only marshal arguments: every step of
the layer runs in the library's CUDA kernels. PyTorch provides device memory
and the current stream. There is no CPU fallback: importing this package
raises if the library has not been built, and every call requires CUDA
tensors.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
# MOE_LIBRARY=debug selects the build with device-side bounds checks
LIB_PATH = os.path.join(_PKG_DIR, "libmoe_debug.so" if os.environ.get("MOE_LIBRARY") == "debug" else "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_BOUNDS = 6

DTYPE_F32 = 0
DTYPE_BF16 = 1
BIAS_NONE = 0
BIAS_LOGIT = 1
BIAS_PROB = 2
GATE_SELECTED = 0
GATE_FULL = 1
DROP_TOKEN = 0
DROP_SLOT = 1
MAX_E = 512
MAX_K = 16

STATS_HEADER_BYTES = 48


class Problem(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("capacity_factor", ctypes.c_float),
                ("dtype", ctypes.c_int32), ("bias_mode", ctypes.c_int32),
                ("d_ff_shared", ctypes.c_int32), ("gate_mode", ctypes.c_int32),
                ("drop_order", ctypes.c_int32), ("pad_rows", ctypes.c_int32), ("train", ctypes.c_int32)]


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("idx", "gate", "pos", "indptr", "row_token", "logits", "xp", "h", "o", "hs", "s", "ab", "total")]


class MoEError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {error_string(code)} (code {code})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m mixture_experts_layer_62_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Problem)
    vp = ctypes.c_void_p
    sz = ctypes.c_size_t
    lib.moe_stats_size.argtypes = [ctypes.c_int32]
    lib.moe_stats_size.restype = sz
    lib.moe_workspace_size.argtypes = [P]
    lib.moe_workspace_size.restype = sz
    lib.moe_workspace_layout.argtypes = [P, ctypes.POINTER(WorkspaceLayout)]
    lib.moe_workspace_layout.restype = ctypes.c_int
    lib.moe_error_string.argtypes = [ctypes.c_int]
    lib.moe_error_string.restype = ctypes.c_char_p
    lib.moe_gemm_variant.argtypes = [P]
    lib.moe_gemm_variant.restype = ctypes.c_int
    lib.moe_router_variant.argtypes = [P, ctypes.c_int]
    lib.moe_router_variant.restype = ctypes.c_int
    lib.moe_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.moe_set_wait_limit.restype = ctypes.c_longlong
    lib.moe_device_sm_count.argtypes = []
    lib.moe_device_sm_count.restype = ctypes.c_int
    lib.moe_permuted_rows.argtypes = [P]
    lib.moe_permuted_rows.restype = ctypes.c_int32
    lib.moe_backward_workspace_size.argtypes = [P]
    lib.moe_backward_workspace_size.restype = sz
    f32 = ctypes.c_float
    lib.moe_backward.argtypes = [P] + [vp] * 9 + [f32, f32] + [vp] * 9 + [vp, sz, vp, sz, vp]
    lib.moe_backward.restype = ctypes.c_int
    lib.moe_bias_update.argtypes = [P, vp, f32, vp, vp]
    lib.moe_bias_update.restype = ctypes.c_int
    lib.moe_forward.argtypes = [P] + [vp] * 11 + [vp, sz, vp]
    lib.moe_forward.restype = ctypes.c_int
    lib.moe_route.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_route.restype = ctypes.c_int
    lib.moe_route_from_logits.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_route_from_logits.restype = ctypes.c_int
    lib.moe_permute.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_permute.restype = ctypes.c_int
    lib.moe_experts.argtypes = [P] + [vp] * 12 + [vp, sz, vp]
    lib.moe_experts.restype = ctypes.c_int
    lib.moe_expert_up.argtypes = [P] + [vp] * 10 + [vp, sz, vp]
    lib.moe_expert_up.restype = ctypes.c_int
    lib.moe_expert_down.argtypes = [P] + [vp] * 8 + [vp, sz, vp]
    lib.moe_expert_down.restype = ctypes.c_int
    lib.moe_combine.argtypes = [P, vp, vp, vp, vp, vp, vp]
    lib.moe_combine.restype = ctypes.c_int
    return lib


_LIB = None


def _lib():
    """The loaded library; raises ImportError when it has not been built."""
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    if name == "lib":
        return _lib()
    raise AttributeError(name)


GEMM_VARIANTS = {0: "single", 1: "pair", 2: "grid_split", 3: "split_k", 4: "simt", 5: "interleaved", 6: "gemv"}


def gemm_variant(p: Problem) -> str:
    """Name of the grouped-GEMM kernel the library uses for p (moe_gemm_variant)."""
    v = int(_lib().moe_gemm_variant(ctypes.byref(p)))
    if v < 0:
        raise MoEError(-v, "moe_gemm_variant")
    return GEMM_VARIANTS[v]


ROUTER_VARIANTS = {0: "small", 1: "fused_mma", 2: "fused_fma", 3: "tensor", 4: "simt"}


def router_variant(p: Problem, forward: bool = True) -> str:
    """Name of the router the library uses for p: moe_forward's (forward=True)
    or moe_route's (moe_router_variant)."""
    v = int(_lib().moe_router_variant(ctypes.byref(p), 1 if forward else 0))
    if v < 0:
        raise MoEError(-v, "moe_router_variant")
    return ROUTER_VARIANTS[v]


def set_wait_limit(ns: int) -> int:
    """Wall-clock limit (nanoseconds) of the device-side bounded waits of the
    tensor-core kernels, process-wide; ns <= 0 restores the 2 s default.
    Returns the previous limit (moe_set_wait_limit)."""
    return int(_lib().moe_set_wait_limit(int(ns)))


def error_string(code: int) -> str:
    return _lib().moe_error_string(int(code)).decode()


def _check(rc, where):
    if rc != MOE_OK:
        raise MoEError(rc, where)


def _dtype_code(dtype) -> int:
    if dtype in (torch.bfloat16, "bf16", DTYPE_BF16):
        return DTYPE_BF16
    if dtype in (torch.float32, "f32", "fp32", DTYPE_F32):
        return DTYPE_F32
    raise ValueError(f"unsupported dtype {dtype}")


def torch_dtype(code: int):
    return torch.bfloat16 if code == DTYPE_BF16 else torch.float32


def problem(T, d, d_ff, E, k, capacity_factor=0.0, dtype="bf16", bias_mode=BIAS_NONE, d_ff_shared=0,
            gate_mode=GATE_SELECTED, drop_order=DROP_TOKEN, pad_rows=0, train=0) -> Problem:
    return Problem(int(T), int(d), int(d_ff), int(E), int(k), float(capacity_factor),
                   _dtype_code(dtype), int(bias_mode), int(d_ff_shared), int(gate_mode), int(drop_order),
                   int(pad_rows), int(train))


def permuted_rows(p: Problem) -> int:
    """Rows the permuted buffers (xp, h, o, row_token) must hold for p."""
    n = int(_lib().moe_permuted_rows(ctypes.byref(p)))
    if n == 0 and p.T * p.k > 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_permuted_rows")
    return n


def stats_size(E: int) -> int:
    return int(_lib().moe_stats_size(int(E)))


def workspace_size(p: Problem) -> int:
    n = int(_lib().moe_workspace_size(ctypes.byref(p)))
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_workspace_size")
    return n


def workspace_layout(p: Problem) -> dict:
    lay = WorkspaceLayout()
    _check(_lib().moe_workspace_layout(ctypes.byref(p), ctypes.byref(lay)), "moe_workspace_layout")
    return {n: getattr(lay, n) for n, _ in WorkspaceLayout._fields_}


def device_sm_count() -> int:
    return int(_lib().moe_device_sm_count())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the MoE library must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the MoE library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def alloc_workspace(p: Problem, device=None) -> torch.Tensor:
    return torch.empty(workspace_size(p), dtype=torch.uint8, device=device or "cuda")


def alloc_stats(E: int, device=None) -> torch.Tensor:
    return torch.zeros(stats_size(E), dtype=torch.uint8, device=device or "cuda")


def forward(p: Problem, x, W_r, W1, W3, W2, out, stats, workspace, bias=None,
            Ws1=None, Ws3=None, Ws2=None, stream=None):
    """out[t] = sum_j gate[t,j] FFN_{idx[t,j]}(x[t]) (+ shared FFN); see moe_forward."""
    rc = _lib().moe_forward(ctypes.byref(p), _ptr(x), _ptr(W_r), _ptr(bias), _ptr(W1), _ptr(W3), _ptr(W2),
                         _ptr(Ws1), _ptr(Ws3), _ptr(Ws2), _ptr(out), _ptr(stats), _ptr(workspace),
                         workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "moe_forward")
    return out


def backward_workspace_size(p: Problem) -> int:
    n = int(_lib().moe_backward_workspace_size(ctypes.byref(p)))
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_backward_workspace_size")
    return n


def alloc_backward_workspace(p: Problem, device=None) -> torch.Tensor:
    return torch.empty(backward_workspace_size(p), dtype=torch.uint8, device=device or "cuda")


def backward(p: Problem, x, W_r, W1, W3, W2, dy, dx, dW_r, dW1, dW3, dW2, stats, workspace, bwd_workspace,
             alpha=0.0, beta=0.0, Ws1=None, Ws3=None, Ws2=None, dWs1=None, dWs3=None, dWs2=None, stream=None):
    """Gradients of <dy, y> + alpha L_aux + beta L_z after a moe_forward with
    p.train = 1 on the same workspace; see moe_backward."""
    rc = _lib().moe_backward(ctypes.byref(p), _ptr(x), _ptr(W_r), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(Ws1),
                             _ptr(Ws3), _ptr(Ws2), _ptr(dy), float(alpha), float(beta), _ptr(dx), _ptr(dW_r),
                             _ptr(dW1), _ptr(dW3), _ptr(dW2), _ptr(dWs1), _ptr(dWs3), _ptr(dWs2), _ptr(stats),
                             _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _ptr(bwd_workspace), bwd_workspace.numel() * bwd_workspace.element_size(),
                             _stream(stream))
    _check(rc, "moe_backward")


def bias_update(p: Problem, stats, bias, gamma, stream=None):
    """bias[e] -= gamma above the mean load, += gamma below (in place)."""
    _check(_lib().moe_bias_update(ctypes.byref(p), _ptr(stats), float(gamma), _ptr(bias), _stream(stream)),
           "moe_bias_update")


def route(p: Problem, x, W_r, idx, gate, stats, workspace, bias=None, logits=None, stream=None):
    rc = _lib().moe_route(ctypes.byref(p), _ptr(x), _ptr(W_r), _ptr(bias), _ptr(idx), _ptr(gate), _ptr(logits),
                       _ptr(stats), _ptr(workspace), workspace.numel() * workspace.element_size(),
                       _stream(stream))
    _check(rc, "moe_route")


def route_from_logits(p: Problem, logits, idx, gate, stats, workspace, bias=None, stream=None):
    rc = _lib().moe_route_from_logits(ctypes.byref(p), _ptr(logits), _ptr(bias), _ptr(idx), _ptr(gate),
                                   _ptr(stats), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check(rc, "moe_route_from_logits")


def permute(p: Problem, x, idx, pos, indptr, row_token, xp, stats, workspace, stream=None):
    rc = _lib().moe_permute(ctypes.byref(p), _ptr(x), _ptr(idx), _ptr(pos), _ptr(indptr), _ptr(row_token),
                         _ptr(xp), _ptr(stats), _ptr(workspace), workspace.numel() * workspace.element_size(),
                         _stream(stream))
    _check(rc, "moe_permute")


def experts(p: Problem, xp, indptr, W1, W3, W2, o, workspace, x=None, Ws1=None, Ws3=None, Ws2=None,
            s=None, stats=None, stream=None):
    rc = _lib().moe_experts(ctypes.byref(p), _ptr(xp), _ptr(indptr), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(x),
                         _ptr(Ws1), _ptr(Ws3), _ptr(Ws2), _ptr(o), _ptr(s), _ptr(stats), _ptr(workspace),
                         workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "moe_experts")


def expert_up(p: Problem, xp, indptr, W1, W3, h, workspace, x=None, Ws1=None, Ws3=None, hs=None,
              stats=None, stream=None):
    rc = _lib().moe_expert_up(ctypes.byref(p), _ptr(xp), _ptr(indptr), _ptr(W1), _ptr(W3), _ptr(x), _ptr(Ws1),
                              _ptr(Ws3), _ptr(h), _ptr(hs), _ptr(stats), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "moe_expert_up")


def expert_down(p: Problem, h, indptr, W2, o, workspace, hs=None, Ws2=None, s=None, stats=None, stream=None):
    rc = _lib().moe_expert_down(ctypes.byref(p), _ptr(h), _ptr(indptr), _ptr(W2), _ptr(hs), _ptr(Ws2), _ptr(o),
                                _ptr(s), _ptr(stats), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream))
    _check(rc, "moe_expert_down")


def combine(p: Problem, o, pos, gate, out, s=None, stream=None):
    rc = _lib().moe_combine(ctypes.byref(p), _ptr(o), _ptr(pos), _ptr(gate), _ptr(s), _ptr(out), _stream(stream))
    _check(rc, "moe_combine")


def permute_noalloc(p: Problem, x, idx, pos, indptr, row_token, xp, stats, stream=None):
    """moe_permute without a workspace: for callers that cannot allocate
    device memory; the library's fixed 1 MiB scratch array is used instead
    (see moe_permute_noalloc in include/moe.h for the limit and the rules)."""
    lib = _lib()
    fn = lib.moe_permute_noalloc
    if fn.restype is not ctypes.c_int:
        fn.argtypes = [ctypes.POINTER(Problem)] + [ctypes.c_void_p] * 8
        fn.restype = ctypes.c_int
    rc = fn(ctypes.byref(p), _ptr(x), _ptr(idx), _ptr(pos), _ptr(indptr), _ptr(row_token), _ptr(xp), _ptr(stats),
            _stream(stream))
    _check(rc, "moe_permute_noalloc")


@dataclass
class Stats:
    status: int
    capacity: int
    rows: int
    dropped: int
    max_count: int
    l_aux: float
    max_over_mean: float
    z_loss: float
    entropy: float
    top_gap: float
    counts: list
    kept: list
    P: list
    f: list


def read_stats(stats: torch.Tensor, E: int) -> Stats:
    """Parse a statistics block (synchronises on the copy to the host)."""
    raw = stats.detach().to("cpu")
    hdr_i = raw[:STATS_HEADER_BYTES].view(torch.int32)
    hdr_f = raw[:STATS_HEADER_BYTES].view(torch.float32)
    body = raw[STATS_HEADER_BYTES:STATS_HEADER_BYTES + 16 * E]
    ints = body[:8 * E].view(torch.int32)
    flts = body[8 * E:].view(torch.float32)
    return Stats(status=int(hdr_i[0]), capacity=int(hdr_i[1]), rows=int(hdr_i[2]), dropped=int(hdr_i[3]),
                 max_count=int(hdr_i[4]), l_aux=float(hdr_f[5]), max_over_mean=float(hdr_f[6]),
                 z_loss=float(hdr_f[7]), entropy=float(hdr_f[8]), top_gap=float(hdr_f[9]),
                 counts=ints[:E].tolist(), kept=ints[E:].tolist(), P=flts[:E].tolist(), f=flts[E:].tolist())


def workspace_view(workspace: torch.Tensor, p: Problem, name: str) -> torch.Tensor:
    """A typed view of one intermediate that moe_forward leaves in the workspace."""
    lay = workspace_layout(p)
    T, k, E, d, dff, dfs = p.T, p.k, p.E, p.d, p.d_ff, p.d_ff_shared
    dt = torch_dtype(p.dtype)
    shapes = {"idx": ((T, k), torch.int32), "gate": ((T, k), torch.float32), "pos": ((T, k), torch.int32),
              "indptr": ((E + 1,), torch.int32), "row_token": ((T * k,), torch.int32),
              "logits": ((T, E), torch.float32), "xp": ((T * k, d), dt), "h": ((T * k, dff), dt),
              "o": ((T * k, d), dt), "hs": ((T, dfs), dt), "s": ((T, d), dt)}
    shape, dtype = shapes[name]
    n = 1
    for s_ in shape:
        n *= s_
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    off = lay[name]
    return workspace[off:off + nbytes].view(dtype).view(*shape)


class MoELayer:
    """Weights of one layer plus the buffers a forward call needs.

    Allocation is done once here (by PyTorch); each call of ``__call__``
    launches the library's kernels on the current stream and allocates
    nothing.
    """

    def __init__(self, p: Problem, W_r, W1, W3, W2, bias=None, Ws1=None, Ws3=None, Ws2=None):
        self.p = p
        self.W_r, self.W1, self.W3, self.W2 = W_r, W1, W3, W2
        self.bias, self.Ws1, self.Ws3, self.Ws2 = bias, Ws1, Ws3, Ws2
        dev = W1.device
        self.workspace = alloc_workspace(p, dev)
        self.stats = alloc_stats(p.E, dev)
        self.out = torch.empty((p.T, p.d), dtype=torch_dtype(p.dtype), device=dev)

    def __call__(self, x, out=None, stream=None):
        out = self.out if out is None else out
        forward(self.p, x, self.W_r, self.W1, self.W3, self.W2, out, self.stats, self.workspace,
                bias=self.bias, Ws1=self.Ws1, Ws3=self.Ws3, Ws2=self.Ws2, stream=stream)
        return out

    def read_stats(self) -> Stats:
        return read_stats(self.stats, self.p.E)
