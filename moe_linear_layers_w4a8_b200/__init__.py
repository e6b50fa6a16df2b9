"""W4A8 quantized Linear / MoE-expert GEMM for NVIDIA B200 (sm_100a).

Thin Python binding of the C ABI in include/w4a8.h (libw4a8.so, built
in-tree).  This module only marshals arguments: torch supplies device memory
and the current CUDA stream; every step of the computation runs in the
library's CUDA kernels.  There is no fallback: if the library cannot be
loaded, every call raises W4A8Error.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import threading
from typing import Optional

import torch

__all__ = [
    "W4A8Error", "WDesc", "PackedWeight", "load_library", "library_path",
    "w4a8_pack_weights", "w4a8_pack_expert_weights", "w4a8_quant_act", "w4a8_gemm",
    "w4a8_gemm_debug_partials", "w4a8_gemm_static_scratch", "w4a8_moe_grouped_gemm", "w4a8_moe_workspace_layout",
    "w4a8_gemm_workspace_size", "w4a8_moe_workspace_size", "w4a8_get_device_status",
    "w4a8_status_string", "w4a8_selftest_bounded_wait", "w4a8_linear", "w4a8_linear_workspace_size", "LAYOUT_VERSION",
    "STATUS", "PackedW8", "w8a8_pack_weights", "w8a8_gemm", "w8a8_gemm_workspace_size", "w8a8_linear",
    "w8a8_linear_workspace_size", "w4a8_moe_route", "w4a8_moe_experts", "w4a8_moe_combine",
    "w4a16_gemm", "w4a16_gemm_workspace_size",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LAYOUT_VERSION = 1
STATUS = {
    0: "W4A8_OK", 1: "W4A8_ERR_INVALID_ARG", 2: "W4A8_ERR_UNSUPPORTED_SHAPE",
    3: "W4A8_ERR_FORMAT_MISMATCH", 4: "W4A8_ERR_NONFINITE", 5: "W4A8_ERR_TIMEOUT",
    6: "W4A8_ERR_CUDA", 7: "W4A8_ERR_WORKSPACE",
}


class W4A8Error(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = int(code)
        super().__init__(f"{where}: {STATUS.get(self.code, 'W4A8_ERR_UNKNOWN')} ({self.code})")


class WDesc(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("symmetric", ctypes.c_int32), ("group", ctypes.c_int32),
                ("K", ctypes.c_int32), ("N", ctypes.c_int32), ("layout_version", ctypes.c_int32)]

    def copy(self) -> "WDesc":
        return WDesc(self.bits, self.symmetric, self.group, self.K, self.N, self.layout_version)


class MoeWsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("perm", "inv", "qx", "sx", "h", "qh", "sh", "yd", "total")]


@dataclasses.dataclass
class PackedWeight:
    """Packed 4-bit weight (one matrix, or E stacked expert matrices)."""
    packed: torch.Tensor           # uint8 [(E,) N*K/2]
    s_w: torch.Tensor              # fp32 [(E,) G, N]
    z: Optional[torch.Tensor]      # uint8 [(E,) G, N] or None (symmetric)
    desc: WDesc
    experts: int = 0               # 0 = single matrix

    @property
    def K(self):
        return self.desc.K

    @property
    def N(self):
        return self.desc.N


_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return os.path.join(_PKG, "libw4a8.so")


def load_library():
    """Loads libw4a8.so (raises W4A8Error(6) when it is missing)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise W4A8Error(6, f"libw4a8.so not built (expected at {path}); run the package build")
        L = ctypes.CDLL(path)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        st = ctypes.c_int
        L.w4a8_abi_version.restype = I
        L.w4a8_status_string.restype = ctypes.c_char_p
        L.w4a8_status_string.argtypes = [st]
        L.w4a8_packed_bytes.restype = S
        L.w4a8_packed_bytes.argtypes = [I, I]
        L.w4a8_gemm_workspace_size.restype = S
        L.w4a8_gemm_workspace_size.argtypes = [I, ctypes.POINTER(WDesc)]
        L.w4a8_moe_workspace_size.restype = S
        L.w4a8_moe_workspace_size.argtypes = [I, I, I, ctypes.POINTER(WDesc), ctypes.POINTER(WDesc)]
        L.w4a8_moe_workspace_layout.restype = st
        L.w4a8_moe_workspace_layout.argtypes = [I, I, I, ctypes.POINTER(WDesc), ctypes.POINTER(WDesc),
                                                ctypes.POINTER(MoeWsLayout)]
        L.w4a8_pack_weights.restype = st
        L.w4a8_pack_weights.argtypes = [P, I, I, I, I, P, P, P, ctypes.POINTER(WDesc), P, P]
        L.w4a8_quant_act.restype = st
        L.w4a8_quant_act.argtypes = [P, I, I, I, I, P, P, P, P, P]
        L.w4a8_gemm.restype = st
        L.w4a8_gemm.argtypes = [P, P, P, P, P, ctypes.POINTER(WDesc), I, P, I, P, S, P, P]
        L.w4a8_gemm_static_scratch.restype = st
        L.w4a8_gemm_static_scratch.argtypes = [P, P, P, P, P, ctypes.POINTER(WDesc), I, P, I, P, P]
        L.w4a8_linear_workspace_size.restype = S
        L.w4a8_linear_workspace_size.argtypes = [I, ctypes.POINTER(WDesc)]
        L.w4a8_linear.restype = st
        L.w4a8_linear.argtypes = [P, I, I, P, P, P, ctypes.POINTER(WDesc), P, I, P, S, P, P]
        L.w4a8_gemm_debug_partials.restype = st
        L.w4a8_gemm_debug_partials.argtypes = [P, P, P, P, P, ctypes.POINTER(WDesc), I, P, I, P, P, S, P, P]
        L.w4a8_moe_grouped_gemm.restype = st
        L.w4a8_moe_grouped_gemm.argtypes = [P, P, I, I, I, P, P, P, ctypes.POINTER(WDesc), P, P, P,
                                            ctypes.POINTER(WDesc), P, P, P, P, P, S, P, P]
        L.w4a8_moe_grouped_gemm_profiled.restype = st
        L.w4a8_moe_grouped_gemm_profiled.argtypes = L.w4a8_moe_grouped_gemm.argtypes + [P]
        L.w4a8_moe_debug_partials.restype = st
        L.w4a8_moe_debug_partials.argtypes = L.w4a8_moe_grouped_gemm.argtypes + [P, P, P]
        L.w4a8_moe_route.restype = st
        L.w4a8_moe_route.argtypes = [P, I, I, I, P, P, P, P]
        L.w4a8_moe_experts_workspace_size.restype = S
        L.w4a8_moe_experts_workspace_size.argtypes = [I, I, ctypes.POINTER(WDesc), ctypes.POINTER(WDesc)]
        L.w4a8_moe_experts.restype = st
        L.w4a8_moe_experts.argtypes = [P, P, I, I, P, P, P, ctypes.POINTER(WDesc), P, P, P, ctypes.POINTER(WDesc),
                                       P, P, S, P, P]
        L.w4a8_moe_combine.restype = st
        L.w4a8_moe_combine.argtypes = [P, P, I, I, I, P, P]
        L.w8a8_pack_weights.restype = st
        L.w8a8_pack_weights.argtypes = [P, I, I, P, P, ctypes.POINTER(WDesc), P, P]
        L.w8a8_gemm_workspace_size.restype = S
        L.w8a8_gemm_workspace_size.argtypes = [I, ctypes.POINTER(WDesc)]
        L.w8a8_gemm.restype = st
        L.w8a8_gemm.argtypes = [P, P, P, P, ctypes.POINTER(WDesc), I, P, I, P, S, P, P]
        L.w8a8_linear_workspace_size.restype = S
        L.w8a8_linear_workspace_size.argtypes = [I, ctypes.POINTER(WDesc)]
        L.w8a8_linear.restype = st
        L.w8a8_linear.argtypes = [P, I, I, P, P, ctypes.POINTER(WDesc), P, I, P, S, P, P]
        L.w4a16_gemm_workspace_size.restype = S
        L.w4a16_gemm_workspace_size.argtypes = [I, ctypes.POINTER(WDesc)]
        L.w4a16_gemm.restype = st
        L.w4a16_gemm.argtypes = [P, I, I, P, P, P, ctypes.POINTER(WDesc), P, I, P, S, P, P]
        L.w4a8_get_device_status.restype = st
        L.w4a8_get_device_status.argtypes = [P, P]
        L.w4a8_selftest_bounded_wait.restype = st
        L.w4a8_selftest_bounded_wait.argtypes = [P, ctypes.c_uint64, P]
        _lib = L
        return L


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _check(code: int, where: str):
    if code != 0:
        raise W4A8Error(code, where)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise W4A8Error(1, "tensors must be on a CUDA device")


def w4a8_status_string(code: int) -> str:
    return load_library().w4a8_status_string(int(code)).decode()


def w4a8_get_device_status(status: torch.Tensor) -> int:
    """Synchronizes the current stream and returns the device status word."""
    return int(load_library().w4a8_get_device_status(_p(status), _stream(status.device)))


def new_status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


# ----------------------------------------------------------------- packing --

def w4a8_pack_weights(W: torch.Tensor, group: int = 128, symmetric: bool = True,
                      status: Optional[torch.Tensor] = None, out: Optional[PackedWeight] = None,
                      expert: Optional[int] = None) -> PackedWeight:
    """Group-wise 4-bit quantization + packing of W fp32 [K, N] (device).
    With `out` and `expert`, writes expert slot `expert` of a stacked weight."""
    L = load_library()
    _need_cuda(W)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise W4A8Error(1, "W must be fp32 [K, N]")
    W = W.contiguous()
    K, N = W.shape
    G = K // group if group > 0 else 0
    if out is None:
        packed = torch.empty(K * N // 2, dtype=torch.uint8, device=W.device)
        s_w = torch.empty(G, N, dtype=torch.float32, device=W.device)
        z = None if symmetric else torch.empty(G, N, dtype=torch.uint8, device=W.device)
        pk, sw, zz = packed, s_w, z
    else:
        e = int(expert)
        pk, sw = out.packed[e], out.s_w[e]
        zz = None if out.z is None else out.z[e]
    d = WDesc()
    code = L.w4a8_pack_weights(_p(W), K, N, group, int(bool(symmetric)), _p(pk), _p(sw), _p(zz),
                               ctypes.byref(d), _p(status), _stream(W.device))
    _check(code, "w4a8_pack_weights")
    if out is not None:
        return out
    return PackedWeight(packed=pk, s_w=sw, z=zz, desc=d)


def w4a8_pack_expert_weights(make_weight, E: int, K: int, N: int, group: int, symmetric: bool,
                             device, status: Optional[torch.Tensor] = None) -> PackedWeight:
    """Packs E expert matrices (make_weight(e) -> fp32 [K, N] on `device`)
    into one stacked PackedWeight."""
    G = K // group
    packed = torch.empty(E, K * N // 2, dtype=torch.uint8, device=device)
    s_w = torch.empty(E, G, N, dtype=torch.float32, device=device)
    z = None if symmetric else torch.empty(E, G, N, dtype=torch.uint8, device=device)
    pw = PackedWeight(packed=packed, s_w=s_w, z=z,
                      desc=WDesc(4, int(bool(symmetric)), group, K, N, LAYOUT_VERSION), experts=E)
    for e in range(E):
        w4a8_pack_weights(make_weight(e), group, symmetric, status=status, out=pw, expert=e)
    return pw


# ------------------------------------------------------------- activation --

def w4a8_quant_act(X: torch.Tensor, group_for_rowsum: int = 0, status: Optional[torch.Tensor] = None,
                   q_out: Optional[torch.Tensor] = None, s_out: Optional[torch.Tensor] = None):
    """Per-token INT8 quantization of X bf16 [M, K] -> (q int8, s_x fp32, rowsum|None)."""
    L = load_library()
    _need_cuda(X)
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise W4A8Error(1, "X must be bf16 [M, K] with unit column stride")
    M, K = X.shape
    q = q_out if q_out is not None else torch.empty(M, K, dtype=torch.int8, device=X.device)
    s = s_out if s_out is not None else torch.empty(M, dtype=torch.float32, device=X.device)
    rs = (torch.empty(M, K // group_for_rowsum, dtype=torch.int32, device=X.device)
          if group_for_rowsum else None)
    code = L.w4a8_quant_act(_p(X), M, K, X.stride(0), int(group_for_rowsum), _p(q), _p(s), _p(rs),
                            _p(status), _stream(X.device))
    _check(code, "w4a8_quant_act")
    return q, s, rs


# ------------------------------------------------------------------- GEMM ---

def w4a8_gemm_workspace_size(M: int, w: PackedWeight) -> int:
    return int(load_library().w4a8_gemm_workspace_size(int(M), ctypes.byref(w.desc)))


def _gemm(qx, s_x, w: PackedWeight, out, workspace, status, P):
    L = load_library()
    _need_cuda(qx, s_x)
    if qx.dtype != torch.int8 or qx.dim() != 2 or not qx.is_contiguous():
        raise W4A8Error(1, "qx must be contiguous int8 [M, K]")
    M = qx.shape[0]
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=qx.device)
    need = w4a8_gemm_workspace_size(M, w)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=qx.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if P is None:
        code = L.w4a8_gemm(_p(qx), _p(s_x), _p(w.packed), _p(w.s_w), _p(w.z), ctypes.byref(w.desc), M,
                           _p(out), out.stride(0), _p(workspace), ws_bytes, _p(status), _stream(qx.device))
        _check(code, "w4a8_gemm")
    else:
        code = L.w4a8_gemm_debug_partials(_p(qx), _p(s_x), _p(w.packed), _p(w.s_w), _p(w.z),
                                          ctypes.byref(w.desc), M, _p(out), out.stride(0), _p(P),
                                          _p(workspace), ws_bytes, _p(status), _stream(qx.device))
        _check(code, "w4a8_gemm_debug_partials")
    return out


def w4a8_gemm(qx: torch.Tensor, s_x: torch.Tensor, w: PackedWeight, out: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y bf16 [M, N] = W4A8(qx, w)."""
    return _gemm(qx, s_x, w, out, workspace, status, None)


def w4a8_gemm_static_scratch(qx: torch.Tensor, s_x: torch.Tensor, w: PackedWeight, out: torch.Tensor,
                             status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """w4a8_gemm without a workspace: the library's fixed per-device scratch
    buffer holds the split-K partials, and nothing is allocated (``out`` is
    required).  Calls that may overlap on the GPU race on that buffer."""
    L = load_library()
    _need_cuda(qx, s_x)
    if qx.dtype != torch.int8 or qx.dim() != 2 or not qx.is_contiguous():
        raise W4A8Error(1, "qx must be contiguous int8 [M, K]")
    code = L.w4a8_gemm_static_scratch(_p(qx), _p(s_x), _p(w.packed), _p(w.s_w), _p(w.z), ctypes.byref(w.desc),
                                      qx.shape[0], _p(out), out.stride(0), _p(status), _stream(qx.device))
    _check(code, "w4a8_gemm_static_scratch")
    return out


def w4a8_gemm_debug_partials(qx, s_x, w: PackedWeight, out=None, workspace=None, status=None):
    """(Y, P int32 [M, G, N]) — the exact group partials as the tensor cores produced them."""
    M = qx.shape[0]
    P = torch.zeros(M, w.K // w.desc.group, w.N, dtype=torch.int32, device=qx.device)
    Y = _gemm(qx, s_x, w, out, workspace, status, P)
    return Y, P


def w4a8_linear_workspace_size(M: int, w: PackedWeight) -> int:
    return int(load_library().w4a8_linear_workspace_size(int(M), ctypes.byref(w.desc)))


def w4a8_linear(X: torch.Tensor, w: PackedWeight, out=None, workspace=None, status=None) -> torch.Tensor:
    """Y bf16 [M, N] = the quantized Linear layer on X bf16 [M, K]: per-token
    INT8 quantization then the W4A8 GEMM, in one library call."""
    L = load_library()
    _need_cuda(X)
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise W4A8Error(1, "X must be bf16 [M, K] with unit column stride")
    M = X.shape[0]
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    need = w4a8_linear_workspace_size(M, w)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    code = L.w4a8_linear(_p(X), M, X.stride(0), _p(w.packed), _p(w.s_w), _p(w.z), ctypes.byref(w.desc), _p(out),
                         out.stride(0), _p(workspace), ws_bytes, _p(status), _stream(X.device))
    _check(code, "w4a8_linear")
    return out


# -------------------------------------------------------------------- MoE ---

def w4a8_moe_workspace_size(T: int, E: int, topk: int, w1: PackedWeight, w2: PackedWeight) -> int:
    return int(load_library().w4a8_moe_workspace_size(T, E, topk, ctypes.byref(w1.desc),
                                                      ctypes.byref(w2.desc)))


def w4a8_moe_workspace_layout(T: int, E: int, topk: int, w1: PackedWeight, w2: PackedWeight) -> dict:
    lay = MoeWsLayout()
    code = load_library().w4a8_moe_workspace_layout(T, E, topk, ctypes.byref(w1.desc), ctypes.byref(w2.desc),
                                                    ctypes.byref(lay))
    _check(code, "w4a8_moe_workspace_layout")
    return {n: int(getattr(lay, n)) for n, _ in MoeWsLayout._fields_}


def w4a8_moe_grouped_gemm(X: torch.Tensor, logits: torch.Tensor, topk: int, w1: PackedWeight,
                          w2: PackedWeight, workspace: Optional[torch.Tensor] = None,
                          status: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                          stage_events=None, debug_pair_slot: Optional[torch.Tensor] = None):
    """One MoE expert layer (route, dispatch, gate_up + SiLU*up, down, combine).
    Returns dict(out, topk_idx, topk_w, expert_offsets, workspace).
    stage_events: optional list of 8 torch.cuda.Event recorded at the stage
    boundaries (see w4a8_moe_grouped_gemm_profiled).
    debug_pair_slot: optional int32 [T*topk] (test hook, w4a8_moe_debug_partials):
    the result then also holds P1 int32 [S, H/g, 2I] and P2 int32 [S, I/g, H],
    the exact group partials of the pairs with slot >= 0."""
    L = load_library()
    _need_cuda(X, logits)
    if X.dtype != torch.bfloat16 or logits.dtype != torch.float32:
        raise W4A8Error(1, "X must be bf16 and logits fp32")
    X = X.contiguous()
    logits = logits.contiguous()
    T, H = X.shape
    E = logits.shape[1]
    dev = X.device
    need = w4a8_moe_workspace_size(T, E, topk, w1, w2)
    if need == 0 and T > 0:
        raise W4A8Error(2, "w4a8_moe_workspace_size: shape not supported")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(T, topk, dtype=torch.int32, device=dev)
    pw = torch.empty(T, topk, dtype=torch.float32, device=dev)
    offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
    args = [_p(X), _p(logits), T, E, int(topk),
            _p(w1.packed), _p(w1.s_w), _p(w1.z), ctypes.byref(w1.desc),
            _p(w2.packed), _p(w2.s_w), _p(w2.z), ctypes.byref(w2.desc),
            _p(out), _p(idx), _p(pw), _p(offs), _p(workspace),
            workspace.numel() * workspace.element_size(), _p(status), _stream(dev)]
    extra = {}
    if debug_pair_slot is not None:
        S = int(debug_pair_slot.max().item()) + 1 if debug_pair_slot.numel() else 0
        g = w1.desc.group
        I = w1.N // 2
        P1 = torch.zeros(max(S, 1), H // g, 2 * I, dtype=torch.int32, device=dev)
        P2 = torch.zeros(max(S, 1), I // g, H, dtype=torch.int32, device=dev)
        code = L.w4a8_moe_debug_partials(*args, _p(debug_pair_slot.to(dev, torch.int32).contiguous()),
                                         _p(P1), _p(P2))
        extra = dict(P1=P1, P2=P2)
    elif stage_events is None:
        code = L.w4a8_moe_grouped_gemm(*args)
    else:
        evs = (ctypes.c_void_p * 8)(*[None if e is None else ctypes.c_void_p(e.cuda_event) for e in stage_events])
        code = L.w4a8_moe_grouped_gemm_profiled(*args, evs)
    _check(code, "w4a8_moe_grouped_gemm")
    return dict(out=out, topk_idx=idx, topk_w=pw, expert_offsets=offs, workspace=workspace, **extra)


def w4a8_selftest_bounded_wait(status: torch.Tensor, limit_ns: int = 1_000_000) -> None:
    code = load_library().w4a8_selftest_bounded_wait(_p(status), int(limit_ns), _stream(status.device))
    _check(code, "w4a8_selftest_bounded_wait")


# ------------------------------------------------------------------ W8A8 ---

@dataclasses.dataclass
class PackedW8:
    """Per-channel INT8 weight of the W8A8 path: q_w int8 [N, K], s_w fp32 [N]."""
    q_w: torch.Tensor
    s_w: torch.Tensor
    desc: WDesc

    @property
    def K(self):
        return self.desc.K

    @property
    def N(self):
        return self.desc.N


def w8a8_pack_weights(W: torch.Tensor, status: Optional[torch.Tensor] = None) -> PackedW8:
    """Per-channel INT8 quantization of W fp32 [K, N] (device)."""
    L = load_library()
    _need_cuda(W)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise W4A8Error(1, "W must be fp32 [K, N]")
    W = W.contiguous()
    K, N = W.shape
    q = torch.empty(N, K, dtype=torch.int8, device=W.device)
    s = torch.empty(N, dtype=torch.float32, device=W.device)
    d = WDesc()
    _check(L.w8a8_pack_weights(_p(W), K, N, _p(q), _p(s), ctypes.byref(d), _p(status), _stream(W.device)),
           "w8a8_pack_weights")
    return PackedW8(q_w=q, s_w=s, desc=d)


def w8a8_gemm_workspace_size(M: int, w: PackedW8) -> int:
    return int(load_library().w8a8_gemm_workspace_size(int(M), ctypes.byref(w.desc)))


def w8a8_gemm(qx: torch.Tensor, s_x: torch.Tensor, w: PackedW8, out: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y bf16 [M, N] = W8A8(qx, w)."""
    L = load_library()
    _need_cuda(qx, s_x)
    if qx.dtype != torch.int8 or qx.dim() != 2 or not qx.is_contiguous():
        raise W4A8Error(1, "qx must be contiguous int8 [M, K]")
    M = qx.shape[0]
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=qx.device)
    need = w8a8_gemm_workspace_size(M, w)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=qx.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(L.w8a8_gemm(_p(qx), _p(s_x), _p(w.q_w), _p(w.s_w), ctypes.byref(w.desc), M, _p(out), out.stride(0),
                       _p(workspace), ws_bytes, _p(status), _stream(qx.device)), "w8a8_gemm")
    return out


def w8a8_linear_workspace_size(M: int, w: PackedW8) -> int:
    return int(load_library().w8a8_linear_workspace_size(int(M), ctypes.byref(w.desc)))


def w8a8_linear(X: torch.Tensor, w: PackedW8, out=None, workspace=None, status=None) -> torch.Tensor:
    """Y bf16 [M, N] = the W8A8 Linear layer on X bf16 [M, K] (quantization + GEMM)."""
    L = load_library()
    _need_cuda(X)
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise W4A8Error(1, "X must be bf16 [M, K] with unit column stride")
    M = X.shape[0]
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    need = w8a8_linear_workspace_size(M, w)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(L.w8a8_linear(_p(X), M, X.stride(0), _p(w.q_w), _p(w.s_w), ctypes.byref(w.desc), _p(out), out.stride(0),
                         _p(workspace), ws_bytes, _p(status), _stream(X.device)), "w8a8_linear")
    return out


# ------------------------------------------------------------------ W4A16 --

def w4a16_gemm_workspace_size(M: int, w: PackedWeight) -> int:
    return int(load_library().w4a16_gemm_workspace_size(int(M), ctypes.byref(w.desc)))


def w4a16_gemm(X: torch.Tensor, w: PackedWeight, out=None, workspace=None, status=None) -> torch.Tensor:
    """Y bf16 [M, N] = X bf16 [M, K] times the W4A8-packed weight dequantized
    to bf16 inside the kernel (the weight-only W4A16 path)."""
    L = load_library()
    _need_cuda(X)
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise W4A8Error(1, "X must be bf16 [M, K] with unit column stride")
    if w.experts:
        raise W4A8Error(1, "w4a16_gemm takes one weight matrix, not stacked experts")
    M = X.shape[0]
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    need = w4a16_gemm_workspace_size(M, w)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    code = L.w4a16_gemm(_p(X), M, X.stride(0), _p(w.packed), _p(w.s_w), _p(w.z), ctypes.byref(w.desc), _p(out),
                        out.stride(0), _p(workspace), ws_bytes, _p(status), _stream(X.device))
    _check(code, "w4a16_gemm")
    return out


# ------------------------------------------- expert-parallel building blocks --

def w4a8_moe_route(logits: torch.Tensor, topk: int, status: Optional[torch.Tensor] = None):
    """(topk_idx int32 [T, k], topk_w fp32 [T, k]) of logits fp32 [T, E]."""
    L = load_library()
    _need_cuda(logits)
    logits = logits.contiguous()
    T, E = logits.shape
    idx = torch.empty(T, topk, dtype=torch.int32, device=logits.device)
    w = torch.empty(T, topk, dtype=torch.float32, device=logits.device)
    _check(L.w4a8_moe_route(_p(logits), T, E, int(topk), _p(idx), _p(w), _p(status), _stream(logits.device)),
           "w4a8_moe_route")
    return idx, w


def w4a8_moe_experts(X: torch.Tensor, expert_ids: torch.Tensor, w1: PackedWeight, w2: PackedWeight,
                     workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y bf16 [R, H]: row r of X bf16 [R, H] through expert expert_ids[r] (unweighted)."""
    L = load_library()
    _need_cuda(X, expert_ids)
    X = X.contiguous()
    ids = expert_ids.to(torch.int32).contiguous()
    R, H = X.shape
    E = w1.experts
    if out is None:
        out = torch.empty(R, H, dtype=torch.bfloat16, device=X.device)
    if R == 0:
        return out
    need = int(L.w4a8_moe_experts_workspace_size(R, E, ctypes.byref(w1.desc), ctypes.byref(w2.desc)))
    if need == 0:
        raise W4A8Error(2, "w4a8_moe_experts_workspace_size: shape not supported")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    _check(L.w4a8_moe_experts(_p(X), _p(ids), R, E, _p(w1.packed), _p(w1.s_w), _p(w1.z), ctypes.byref(w1.desc),
                              _p(w2.packed), _p(w2.s_w), _p(w2.z), ctypes.byref(w2.desc), _p(out), _p(workspace),
                              workspace.numel() * workspace.element_size(), _p(status), _stream(X.device)),
           "w4a8_moe_experts")
    return out


def w4a8_moe_combine(y_rows: torch.Tensor, topk_w: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out bf16 [T, H] = sum_j topk_w[t, j] * y_rows[t * k + j] (fp32, slot order)."""
    L = load_library()
    _need_cuda(y_rows, topk_w)
    T, k = topk_w.shape
    H = y_rows.shape[1]
    y_rows = y_rows.contiguous()
    topk_w = topk_w.contiguous()
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=y_rows.device)
    _check(L.w4a8_moe_combine(_p(y_rows), _p(topk_w), T, k, H, _p(out), _stream(y_rows.device)), "w4a8_moe_combine")
    return out
