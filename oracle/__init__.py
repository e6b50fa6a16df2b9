"""W4A8 oracle: plain, slow CPU reference of the W4A8 Linear / MoE path.

TEST INFRASTRUCTURE ONLY.  Only `tests/`, the smoke check and the bench's
CPU-baseline / reference arm may import this package.  The product library
never imports it, and this package never imports the product library: the two
share nothing but the seeded input generators in `synth`.

The arithmetic lives in `w4a8_oracle.c` (plain loops, binary64 for float
results, binary32 IEEE division and round-half-to-even for code decisions).
This module only marshals numpy arrays and composes the C stages in the order
the pages give (route -> dispatch -> quantize -> expert GEMM -> SiLU gate ->
quantize -> expert GEMM -> weighted combine).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4a8_oracle.c")
_LIB = os.path.join(_HERE, "liborc_w4a8.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-shared",
          "-fPIC", "-std=c11", "-Wall"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (kept separate from the CUDA build)."""
    need = force or not os.path.exists(_LIB) or (
        os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC),
                                     os.path.getmtime(os.path.join(_HERE, "w4a8_oracle.h"))))
    if need:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.orc_bf16_to_f32.restype = ctypes.c_float
            lib.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
            lib.orc_f64_to_bf16.restype = ctypes.c_uint16
            lib.orc_f64_to_bf16.argtypes = [ctypes.c_double]
            lib.orc_f64_to_bf16_array.argtypes = [P, ctypes.c_size_t, P]
            lib.orc_quant_row_f32.restype = I
            lib.orc_quant_row_f32.argtypes = [P, I, P, P]
            lib.orc_quant_act_bf16.restype = I
            lib.orc_quant_act_bf16.argtypes = [P, I, I, I, I, P, P, P]
            lib.orc_quant_weights.restype = I
            lib.orc_quant_weights.argtypes = [P, I, I, I, I, P, P, P]
            lib.orc_dequant_weights.argtypes = [P, P, P, I, I, I, P]
            lib.orc_pack_canonical.argtypes = [P, I, I, P]
            lib.orc_pack_tiled.argtypes = [P, I, I, I, P]
            lib.orc_partials.argtypes = [P, P, P, I, I, I, I, P]
            lib.orc_scale_partials.argtypes = [P, P, P, I, I, I, P, P]
            lib.orc_dequant_gemm.argtypes = [P, P, P, P, P, I, I, I, I, P]
            lib.orc_route.restype = I
            lib.orc_route.argtypes = [P, I, I, I, P, P]
            lib.orc_dispatch.argtypes = [P, I, I, I, P, P, P]
            lib.orc_silu.restype = ctypes.c_double
            lib.orc_silu.argtypes = [ctypes.c_double]
            lib.orc_silu_mul.argtypes = [P, I, I, P]
            lib.orc_combine.argtypes = [P, P, P, I, I, I, P, P]
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


class OracleError(ValueError):
    pass


# --------------------------------------------------------------------------
# scalar helpers
# --------------------------------------------------------------------------

def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bits (uint16) to binary32."""
    u16 = np.ascontiguousarray(u16, dtype=np.uint16)
    return (u16.astype(np.uint32) << 16).view(np.float32)


def f64_to_bf16(y: np.ndarray) -> np.ndarray:
    """Correctly rounded binary64 -> bf16 bits (uint16)."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, dtype=np.uint16)
    _load().orc_f64_to_bf16_array(_p(y), y.size, _p(out))
    return out


def silu(x: float) -> float:
    return _load().orc_silu(float(x))


# --------------------------------------------------------------------------
# quantization stages
# --------------------------------------------------------------------------

def quant_row_f32(x: np.ndarray):
    """Per-token INT8 quantization of one fp32 row -> (codes int8, s fp32, bad)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    q = np.empty(x.shape, dtype=np.int8)
    s = np.zeros(1, dtype=np.float32)
    bad = _load().orc_quant_row_f32(_p(x), x.size, _p(q), _p(s))
    return q, np.float32(s[0]), bool(bad)


def quant_act(X_bf16: np.ndarray, group: int = 0):
    """X raw bf16 bits [M,K] -> (q int8 [M,K], s_x fp32 [M], rowsum int32 [M,G]
    or None, nonfinite flag)."""
    X = np.ascontiguousarray(X_bf16, dtype=np.uint16)
    M, K = X.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    rs = np.empty((M, K // group), dtype=np.int32) if group else None
    r = _load().orc_quant_act_bf16(_p(X), M, K, K, group, _p(q), _p(s), _p(rs))
    if r < 0:
        raise OracleError("invalid activation shape / group")
    return q, s, rs, bool(r)


def quant_weights(W: np.ndarray, group: int, symmetric: bool):
    """W fp32 [K,N] -> (codes int8 [N,K], s fp32 [G,N], z uint8 [G,N], bad).
    Raises OracleError when the group does not tile K."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    K, N = W.shape
    if group <= 0 or K % group:
        raise OracleError("group size must tile K exactly")
    G = K // group
    codes = np.empty((N, K), dtype=np.int8)
    s = np.empty((G, N), dtype=np.float32)
    z = np.zeros((G, N), dtype=np.uint8)
    r = _load().orc_quant_weights(_p(W), K, N, group, int(bool(symmetric)),
                                  _p(codes), _p(s), _p(z))
    if r < 0:
        raise OracleError("group size must tile K exactly")
    return codes, s, z, bool(r)


def dequant_weights(codes, s, z, group):
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    N, K = codes.shape
    out = np.empty((K, N), dtype=np.float64)
    _load().orc_dequant_weights(_p(codes), _p(np.ascontiguousarray(s, np.float32)),
                                _p(None if z is None else np.ascontiguousarray(z, np.uint8)),
                                K, N, group, _p(out))
    return out


def pack_canonical(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    N, K = codes.shape
    out = np.empty((N, K // 2), dtype=np.uint8)
    _load().orc_pack_canonical(_p(codes), K, N, _p(out))
    return out


def pack_tiled(codes: np.ndarray, group: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    N, K = codes.shape
    assert N % 64 == 0 and K % group == 0
    out = np.empty(N * K // 2, dtype=np.uint8)
    _load().orc_pack_tiled(_p(codes), K, N, group, _p(out))
    return out


# --------------------------------------------------------------------------
# GEMM stages
# --------------------------------------------------------------------------

def partials(qx: np.ndarray, codes: np.ndarray, z, group: int) -> np.ndarray:
    """Exact int32 P[m, g, n] = sum_{k in g} q_x[m,k] (q_w[k,n] - z[g,n])."""
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    M, K = qx.shape
    N = codes.shape[0]
    G = K // group
    P = np.empty((M, G, N), dtype=np.int32)
    zz = None if z is None else np.ascontiguousarray(z, dtype=np.uint8)
    _load().orc_partials(_p(qx), _p(codes), _p(zz), M, K, N, group, _p(P))
    return P


def scale_partials(P: np.ndarray, s_x: np.ndarray, s_w: np.ndarray):
    """(Y_exact binary64 [M,N], sum of |terms| binary64 [M,N])."""
    P = np.ascontiguousarray(P, dtype=np.int32)
    M, G, N = P.shape
    Y = np.empty((M, N), dtype=np.float64)
    A = np.empty((M, N), dtype=np.float64)
    _load().orc_scale_partials(_p(P), _p(np.ascontiguousarray(s_x, np.float32)),
                               _p(np.ascontiguousarray(s_w, np.float32)), M, G, N,
                               _p(Y), _p(A))
    return Y, A


def dequant_gemm(qx, s_x, codes, s_w, z, group):
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    M, K = qx.shape
    N = codes.shape[0]
    Y = np.empty((M, N), dtype=np.float64)
    zz = None if z is None else np.ascontiguousarray(z, dtype=np.uint8)
    _load().orc_dequant_gemm(_p(qx), _p(np.ascontiguousarray(s_x, np.float32)), _p(codes),
                             _p(np.ascontiguousarray(s_w, np.float32)), _p(zz),
                             M, K, N, group, _p(Y))
    return Y


def linear(X_bf16: np.ndarray, codes, s_w, z, group: int):
    """Whole W4A8 Linear: per-token quant, exact partials, binary64 product.
    Returns dict with q, s_x, P, Y (binary64), absY, Ybf16 (RNE of Y)."""
    q, s_x, _, bad = quant_act(X_bf16)
    P = partials(q, codes, z, group)
    Y, A = scale_partials(P, s_x, s_w)
    return dict(q=q, s_x=s_x, P=P, Y=Y, absY=A, Ybf16=f64_to_bf16(Y), nonfinite=bad)


# --------------------------------------------------------------------------
# MoE stages
# --------------------------------------------------------------------------

def route(logits: np.ndarray, topk: int):
    L = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = L.shape
    idx = np.empty((T, topk), dtype=np.int32)
    p = np.empty((T, topk), dtype=np.float64)
    r = _load().orc_route(_p(L), T, E, topk, _p(idx), _p(p))
    if r < 0:
        raise OracleError("invalid routing shape")
    return idx, p, bool(r)


def dispatch(idx: np.ndarray, E: int):
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, topk = idx.shape
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(T * topk, dtype=np.int32)
    inv = np.empty(T * topk, dtype=np.int32)
    _load().orc_dispatch(_p(idx), T, E, topk, _p(offsets), _p(perm), _p(inv))
    return offsets, perm, inv


def silu_mul(H: np.ndarray) -> np.ndarray:
    H = np.ascontiguousarray(H, dtype=np.float64)
    R, twoI = H.shape
    h = np.empty((R, twoI // 2), dtype=np.uint16)
    _load().orc_silu_mul(_p(H), R, twoI // 2, _p(h))
    return h


def combine(Yd_bf16: np.ndarray, p: np.ndarray, inv: np.ndarray):
    Yd = np.ascontiguousarray(Yd_bf16, dtype=np.uint16)
    p = np.ascontiguousarray(p, dtype=np.float64)
    inv = np.ascontiguousarray(inv, dtype=np.int32)
    T, topk = p.shape
    Hd = Yd.shape[1]
    out = np.empty((T, Hd), dtype=np.uint16)
    out64 = np.empty((T, Hd), dtype=np.float64)
    _load().orc_combine(_p(Yd), _p(p), _p(inv), T, topk, Hd, _p(out), _p(out64))
    return out, out64


def expert_linear_rows(q_rows, s_rows, codes, s_w, z, group):
    """Expert GEMM on already-quantized rows: (Y binary64, absY, P)."""
    P = partials(q_rows, codes, z, group)
    Y, A = scale_partials(P, s_rows, s_w)
    return Y, A, P


def moe_forward(X_bf16, logits, topk, experts_w1, experts_w2, group):
    """The MoE layer, stage by stage, as the pages order it.

    experts_w1[e] / experts_w2[e] = (codes [N,K], s [G,N], z [G,N] or None).
    Returns every intermediate so each stage can be compared on its own."""
    T, H = X_bf16.shape
    E = len(experts_w1)
    idx, p, bad_l = route(logits, topk)
    offsets, perm, inv = dispatch(idx, E)
    qx, sx, _, bad_x = quant_act(X_bf16)
    tok = perm // topk
    q_perm = qx[tok]
    s_perm = sx[tok]
    I2 = next(w[0] for w in experts_w1 if w[0] is not None).shape[0]  # any expert present
    I = I2 // 2
    H_gu = np.zeros((T * topk, I2), dtype=np.float64)
    P1 = [None] * E
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            c, s, z = experts_w1[e]
            Y, _, P = expert_linear_rows(q_perm[a:b], s_perm[a:b], c, s, z, group)
            H_gu[a:b] = Y
            P1[e] = P
    h = silu_mul(H_gu)
    qh, sh, _, _ = quant_act(h)
    Yd64 = np.zeros((T * topk, H), dtype=np.float64)
    P2 = [None] * E
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            c, s, z = experts_w2[e]
            Y, _, P = expert_linear_rows(qh[a:b], sh[a:b], c, s, z, group)
            Yd64[a:b] = Y
            P2[e] = P
    Yd = f64_to_bf16(Yd64)
    out, out64 = combine(Yd, p, inv)
    return dict(idx=idx, p=p, offsets=offsets, perm=perm, inv=inv, qx=qx, sx=sx,
                q_perm=q_perm, s_perm=s_perm, H=H_gu, h=h, qh=qh, sh=sh, Yd64=Yd64,
                Yd=Yd, out=out, out64=out64, P1=P1, P2=P2, nonfinite=bad_l or bad_x)


# --------------------------------------------------------------------------
# W8A8: per-channel INT8 weights ("Inference Quantization ch.1" §2, §4, §8.2)
# --------------------------------------------------------------------------

def quant_w8(W: np.ndarray):
    """Per-channel INT8 weight quantization of W fp32 [K,N]: every column n is
    quantized like a token row (the W8A16 worked example of §2 quantizes a
    weight vector with s = max|W| / 127, q = round(W / s)).  Returns
    (q int8 [K,N], s_w fp32 [N], nonfinite flag)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    K, N = W.shape
    q = np.empty((K, N), dtype=np.int8)
    s = np.empty(N, dtype=np.float32)
    bad = False
    for n in range(N):
        qc, sc, b = quant_row_f32(np.ascontiguousarray(W[:, n]))
        q[:, n] = qc
        s[n] = sc
        bad |= b
    return q, s, bad


def w8a8_exact(qx: np.ndarray, s_x: np.ndarray, qw: np.ndarray, s_w: np.ndarray):
    """§4 ideal path, §8.3: Y = s_x[m] s_w[n] sum_k q_x[m,k] q_w[k,n] with the
    integer sum exact (int64 matmul) and the scaling in binary64.  Returns
    (Y fp64 [M,N], sum of |terms| fp64 [M,N] for the tolerance, acc int64)."""
    acc = qx.astype(np.int64) @ qw.astype(np.int64)
    absacc = np.abs(qx.astype(np.int64)) @ np.abs(qw.astype(np.int64))
    sc = s_x.astype(np.float64)[:, None] * s_w.astype(np.float64)[None, :]
    return sc * acc.astype(np.float64), np.abs(sc) * absacc.astype(np.float64), acc


def w8a8_dequant_gemm(qx: np.ndarray, s_x: np.ndarray, qw: np.ndarray, s_w: np.ndarray) -> np.ndarray:
    """The same product computed the other way round (dequantize both operands
    in binary64, then multiply): the identity the factorised form must meet."""
    Xd = s_x.astype(np.float64)[:, None] * qx.astype(np.float64)
    Wd = qw.astype(np.float64) * s_w.astype(np.float64)[None, :]
    return Xd @ Wd


# --------------------------------------------------------------------------
# W4A16: weight-only, dequantized inside the GEMM ("Inference Quantization
# ch.1" §2 and §3.1-3.2: W_fp ~ s_w W_int, Y = X_fp dequant(W_int, s_w))
# --------------------------------------------------------------------------

def w4a16_dequant_f32(codes: np.ndarray, s: np.ndarray, z, group: int) -> np.ndarray:
    """The dequantized weight before its bf16 rounding: fp32 [K, N] with
    w[k, n] = s[g, n] * (q[n, k] - z[g, n]) rounded once to binary32
    (g = k // group; z = 0 for symmetric codes).  q - z is a small integer,
    so the only rounding is that of the product."""
    codes = np.asarray(codes, dtype=np.int8)
    N, K = codes.shape
    g = np.arange(K) // group
    d = codes.T.astype(np.float32)
    if z is not None:
        d = d - np.asarray(z, dtype=np.uint8)[g, :].astype(np.float32)
    sk = np.asarray(s, dtype=np.float32)[g, :]
    return np.multiply(d, sk, dtype=np.float32)


def w4a16_dequant(codes: np.ndarray, s: np.ndarray, z, group: int) -> np.ndarray:
    """The bf16 operand the weight-only GEMM multiplies: raw bf16 bits [K, N]
    = round-to-nearest-even of w4a16_dequant_f32."""
    return f64_to_bf16(w4a16_dequant_f32(codes, s, z, group).astype(np.float64))


def w4a16_gemm(X_bf16: np.ndarray, W_hat_bf16: np.ndarray):
    """Y = X w_hat in binary64 (both operands are bf16 values, every product is
    exact in binary64).  Returns (Y [M, N], sum of |terms| [M, N])."""
    X = bf16_to_f32(X_bf16).astype(np.float64)
    W = bf16_to_f32(W_hat_bf16).astype(np.float64)
    return X @ W, np.abs(X) @ np.abs(W)
