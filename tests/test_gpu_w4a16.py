"""GPU parity of the weight-only W4A16 path ("Inference Quantization ch.1" §2,
§3.2: bf16 activations, 4-bit group weights dequantized inside the GEMM)
against the oracle:
  * the dequantized bf16 weight is bit-exact (one-hot activation rows return
    it unchanged: one exact product, no rounding);
  * bf16 outputs are within 1 bf16 ulp of the correctly rounded exact value,
    or within the fp32 accumulation bound where it nearly cancels
    (tests/_util.py check_bf16 with the bound below);
  * split-K results are deterministic."""
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


def fp32_bound(K: int) -> float:
    """Relative bound (to sum |x w|) of the fp32 accumulation: the tensor core
    adds K / 16 blocks of 16 exact bf16 products into an fp32 accumulator,
    split-K adds at most a few partial tiles; each addition rounds by at most
    2^-24 of the running magnitude, and the running magnitude never exceeds
    sum |terms|.  Doubled for the block-internal sums."""
    return 2.0 * (K / 16 + 64) * 2.0 ** -24


def oracle_weight(W: np.ndarray, group: int, sym: bool):
    codes, s, z, bad = O.quant_weights(W, group, sym)
    assert not bad
    return codes, s, (None if sym else z)


@pytest.mark.parametrize("K,N,group,sym", [
    (256, 192, 128, True), (256, 192, 128, False), (512, 320, 64, True), (512, 320, 64, False),
])
def test_w4a16_dequant_bit_exact_one_hot_rows(m, K, N, group, sym):
    """X = the K x K identity: row k of Y is the dequantized weight row k,
    bf16 for bf16 (every nibble position, both halves of a 128-column tile,
    the N % 128 == 64 tail)."""
    inp = gen_linear(1, K, N, seed=K + N + int(sym))
    W = inp.W.clone()
    W.view(-1)[:: 997] *= 20.0                      # a few outliers: wider scales
    w = m.w4a8_pack_weights(W.cuda(), group, sym)
    codes, s, z = oracle_weight(W.numpy(), group, sym)
    assert np.array_equal(w.s_w.cpu().numpy(), s)
    X = torch.eye(K, dtype=torch.bfloat16, device="cuda")
    st = m.new_status("cuda")
    Y = m.w4a16_gemm(X, w, status=st)
    assert m.w4a8_get_device_status(st) == 0
    Wh = O.w4a16_dequant(codes, s, z, group)
    assert np.array_equal(bits(Y), Wh)


W16_CASES = [
    # (M, K, N, group, symmetric)
    (16, 512, 512, 128, True),        # the small symmetric linear
    (1, 4096, 14336, 128, True),      # decode shapes: split-K
    (8, 4096, 14336, 128, True),
    (32, 4096, 14336, 128, True),
    (37, 1024, 320, 64, False),       # ragged M (BN=64), N % 128 == 64
    (300, 1024, 448, 128, False),     # BN=256 tiles, ragged
    (130, 2048, 256, 64, True),
    (5, 128, 2048, 128, False),       # one group, one k-block pair
    (64, 7168, 4096, 64, False),      # expert gate_up shape, asymmetric group 64
]


@pytest.mark.parametrize("M,K,N,group,sym", W16_CASES)
def test_w4a16_gemm_against_oracle(m, M, K, N, group, sym):
    inp = gen_linear(M, K, N, seed=M * 7 + N + group, n_outliers=min(8, K // 4), outlier_scale=50.0)
    w = m.w4a8_pack_weights(inp.W.cuda(), group, sym)
    st = m.new_status("cuda")
    Y = m.w4a16_gemm(inp.X.cuda(), w, status=st)
    assert m.w4a8_get_device_status(st) == 0
    codes, s, z = oracle_weight(inp.W.numpy(), group, sym)
    Ye, A = O.w4a16_gemm(bits(inp.X), O.w4a16_dequant(codes, s, z, group))
    check_bf16(bits(Y), Ye, A, rel=fp32_bound(K), what=f"w4a16 M={M} K={K} N={N} g={group} sym={sym}")
    # deterministic: a second call gives the same bits
    Y2 = m.w4a16_gemm(inp.X.cuda(), w, status=st)
    assert np.array_equal(bits(Y2), bits(Y))


def test_w4a16_prefill_shape_sampled_rows(m):
    """M=8192, K=4096, N=14336 (the launch the bench times); a seeded sample
    of rows against the oracle."""
    M, K, N = 8192, 4096, 14336
    inp = gen_linear(M, K, N, seed=0, n_outliers=8, outlier_scale=50.0)
    w = m.w4a8_pack_weights(inp.W.cuda(), 128, True)
    st = m.new_status("cuda")
    Y = m.w4a16_gemm(inp.X.cuda(), w, status=st)
    assert m.w4a8_get_device_status(st) == 0
    rows = np.unique(np.concatenate([[0, 255, 256, 8191], np.random.default_rng(2).integers(0, M, 20)]))
    codes, s, z = oracle_weight(inp.W.numpy(), 128, True)
    Ye, A = O.w4a16_gemm(bits(inp.X)[rows], O.w4a16_dequant(codes, s, z, 128))
    check_bf16(bits(Y)[rows], Ye, A, rel=fp32_bound(K), what="w4a16 prefill rows")


def test_w4a16_strided_rows_and_output(m):
    """X rows with a stride wider than K and Y written into a wider buffer."""
    M, K, N = 20, 1024, 384
    inp = gen_linear(M, K, N, seed=11)
    Xw = torch.zeros(M, K + 64, dtype=torch.bfloat16)
    Xw[:, :K] = inp.X
    Xd = Xw.cuda()[:, :K]
    w = m.w4a8_pack_weights(inp.W.cuda(), 128, False)
    out = torch.full((M, N + 8), 7.0, dtype=torch.bfloat16, device="cuda")
    m.w4a16_gemm(Xd, w, out=out[:, :N])
    Y0 = m.w4a16_gemm(inp.X.cuda(), w)
    assert np.array_equal(bits(out[:, :N]), bits(Y0))
    assert (out[:, N:].float() == 7.0).all()


def test_w4a16_zero_rows_and_columns(m):
    M, K, N = 24, 512, 256
    inp = gen_linear(M, K, N, seed=9)
    X = inp.X.clone()
    X[[0, 7]] = 0
    W = inp.W.clone()
    W[:, 100] = 0
    w = m.w4a8_pack_weights(W.cuda(), 64, True)
    Yb = bits(m.w4a16_gemm(X.cuda(), w))
    assert (Yb[[0, 7]] & 0x7FFF == 0).all()
    assert (Yb[:, 100] & 0x7FFF == 0).all()


def test_w4a16_rejects_bad_arguments(m):
    inp = gen_linear(4, 256, 128, seed=1)
    w = m.w4a8_pack_weights(inp.W.cuda(), 128, True)
    X = inp.X.cuda()
    bad = m.PackedWeight(packed=w.packed, s_w=w.s_w, z=w.s_w.to(torch.uint8), desc=w.desc)
    with pytest.raises(m.W4A8Error) as e:
        m.w4a16_gemm(X, bad)
    assert e.value.code == 3
    Xodd = torch.zeros(4, 260, dtype=torch.bfloat16, device="cuda")[:, :256]  # ldx % 8 != 0
    with pytest.raises(m.W4A8Error) as e:
        m.w4a16_gemm(Xodd, w)
    assert e.value.code == 1
