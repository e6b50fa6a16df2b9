"""GPU parity of the W8A8 variant (per-channel INT8 weights, per-token INT8
activations, "Inference Quantization ch.1" §4 / §8.2-8.3) against the oracle:
weight codes and scales bit-exact; bf16 outputs within 1 bf16 ulp of the
correctly rounded exact value, or within the fp32 bound where it nearly
cancels (tests/_util.py check_bf16)."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import gen_linear
from tests._util import bits, check_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    from moe_linear_layers_w4a8_b200 import _build
    _build.build()
    import moe_linear_layers_w4a8_b200 as mm
    mm.load_library()
    return mm


@pytest.mark.parametrize("K,N", [(128, 16), (512, 512), (4096, 1024), (1024, 448)])
def test_w8_pack_bit_exact(m, K, N):
    inp = gen_linear(1, K, N, seed=K + N)
    W = inp.W.clone()
    W[:, 3] = 0.0
    st = m.new_status("cuda")
    pw = m.w8a8_pack_weights(W.cuda(), status=st)
    qo, so, bad = O.quant_w8(W.numpy())
    assert np.array_equal(pw.q_w.cpu().numpy(), qo.T)
    assert np.array_equal(pw.s_w.cpu().numpy(), so)
    assert (pw.desc.bits, pw.desc.symmetric, pw.desc.group, pw.desc.K, pw.desc.N) == (8, 1, K, K, N)
    assert m.w4a8_get_device_status(st) == 0 and not bad


W8_CASES = [
    # (M, K, N)
    (16, 512, 512),       # one k-block range per tile
    (1, 4096, 14336),     # decode shapes: split-K
    (8, 4096, 14336),
    (32, 4096, 14336),
    (37, 1024, 320),      # ragged M (BN=64), N % 128 == 64
    (300, 1024, 448),     # BN=256 tiles, ragged
    (130, 2048, 256),     # BN=256
    (5, 128, 2048),       # one k-block (no split possible)
]


@pytest.mark.parametrize("M,K,N", W8_CASES)
def test_w8a8_gemm_against_oracle(m, M, K, N):
    inp = gen_linear(M, K, N, seed=M * 3 + N, n_outliers=min(8, K // 4), outlier_scale=50.0)
    pw = m.w8a8_pack_weights(inp.W.cuda())
    st = m.new_status("cuda")
    q, sx, _ = m.w4a8_quant_act(inp.X.cuda(), status=st)
    Y = m.w8a8_gemm(q, sx, pw, status=st)
    Y2 = m.w8a8_linear(inp.X.cuda(), pw, status=st)
    assert m.w4a8_get_device_status(st) == 0
    qo, so, _, _ = O.quant_act(bits(inp.X))
    assert np.array_equal(q.cpu().numpy(), qo)
    qw, sw, _ = O.quant_w8(inp.W.numpy())
    Ye, A, _ = O.w8a8_exact(qo, so, qw, sw)
    check_bf16(bits(Y), Ye, A, what=f"w8a8 M={M} K={K} N={N}")
    # the one-call layer gives the two calls' result bit for bit
    assert np.array_equal(bits(Y2), bits(Y))


def test_w8a8_prefill_shape_sampled_rows(m):
    """M=8192, K=4096, N=14336 through the one-call layer (the launch the bench
    times); a seeded sample of rows against the oracle."""
    M, K, N = 8192, 4096, 14336
    inp = gen_linear(M, K, N, seed=0, n_outliers=8, outlier_scale=50.0)
    pw = m.w8a8_pack_weights(inp.W.cuda())
    st = m.new_status("cuda")
    Y = m.w8a8_linear(inp.X.cuda(), pw, status=st)
    assert m.w4a8_get_device_status(st) == 0
    rows = np.unique(np.concatenate([[0, 255, 256, 8191], np.random.default_rng(2).integers(0, M, 20)]))
    qo, so, _, _ = O.quant_act(bits(inp.X)[rows])
    qw, sw, _ = O.quant_w8(inp.W.numpy())
    Ye, A, _ = O.w8a8_exact(qo, so, qw, sw)
    check_bf16(bits(Y)[rows], Ye, A, what="w8a8 prefill rows")


def test_w8a8_zero_rows_and_columns(m):
    M, K, N = 24, 512, 256
    inp = gen_linear(M, K, N, seed=9)
    X = inp.X.clone()
    X[[0, 7]] = 0
    W = inp.W.clone()
    W[:, 100] = 0
    pw = m.w8a8_pack_weights(W.cuda())
    Y = m.w8a8_linear(X.cuda(), pw)
    Yb = bits(Y)
    assert (Yb[[0, 7]] & 0x7FFF == 0).all()
    assert (Yb[:, 100] & 0x7FFF == 0).all()


def test_w8a8_rejects_w4_descriptor(m):
    inp = gen_linear(4, 256, 128, seed=1)
    w4 = m.w4a8_pack_weights(inp.W.cuda(), 128, True)
    w8 = m.w8a8_pack_weights(inp.W.cuda())
    q, sx, _ = m.w4a8_quant_act(inp.X.cuda())
    fake = m.PackedW8(q_w=w8.q_w, s_w=w8.s_w, desc=w4.desc)
    with pytest.raises(m.W4A8Error) as e:
        m.w8a8_gemm(q, sx, fake)
    assert e.value.code == 3
    fake4 = m.PackedWeight(packed=w4.packed, s_w=w4.s_w, z=None, desc=w8.desc)
    with pytest.raises(m.W4A8Error) as e:
        m.w4a8_gemm(q, sx, fake4)
    assert e.value.code == 3
