"""GPU parity of the Linear path against the CPU oracle (element by element).

Codes, scales, zero-points, packed bytes and the int32 group partials must be
bit-exact; bf16 outputs within 1 bf16 ulp of the correctly rounded exact
value, or, where the exact value nearly cancels, within the fp32 accumulation
bound 1e-5 * sum|s_x s_w P| (see tests/_util.py check_bf16)."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import gen_linear
from synth.inputs import _gen, _weight
from tests._util import bits, check_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    from moe_linear_layers_w4a8_b200 import _build
    _build.build()
    import moe_linear_layers_w4a8_b200 as mm
    mm.load_library()
    return mm


def _weights(K, N, seed, symmetric, outlier_p=0.0):
    g = _gen(1000 + seed)
    W = _weight(g, K, N, 0.02, outlier_p, 20.0)
    if not symmetric:  # give every column a different offset so zero-points vary
        W = W + torch.linspace(-0.02, 0.03, N)[None, :]
    return W


# ----------------------------------------------------------------- quant ---

@pytest.mark.parametrize("M,K", [(16, 512), (1, 4096), (37, 1408), (8, 7168), (300, 2048), (3, 8), (2, 8192),
                                 (1000, 1408), (129, 2056), (70, 4104),
                                 (9000, 2048),                                  # one CTA per row
                                 (8192, 8), (8200, 512), (8193, 1408), (8192, 1536)])  # one warp per row
def test_quant_act_bit_exact(m, M, K):
    inp = gen_linear(M, K, 64, seed=M + K, n_outliers=min(8, K // 2), outlier_scale=50.0)
    st = m.new_status("cuda")
    grp = 64 if K % 64 == 0 else 0
    q, s, rs = m.w4a8_quant_act(inp.X.cuda(), group_for_rowsum=grp, status=st)
    qo, so, rso, bad = O.quant_act(bits(inp.X), group=grp)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy(), so)
    if grp:
        assert np.array_equal(rs.cpu().numpy(), rso)
    assert m.w4a8_get_device_status(st) == 0 and not bad


def test_quant_act_strided_rows_zero_rows_and_ties(m):
    # a row of zeros, a row of exact ties (x/s = k + 0.5 in binary32), and a
    # padded row pitch
    K = 64
    X = torch.zeros(4, 128, dtype=torch.bfloat16)
    X[1, :K] = torch.arange(K, dtype=torch.float32).to(torch.bfloat16) - 32
    X[2, 0] = 127.0
    X[2, 1:K] = torch.tensor([0.5 + i for i in range(K - 1)], dtype=torch.float32).to(torch.bfloat16)
    X[3, :K] = -1e-30
    Xd = X.cuda()[:, :K]
    q, s, _ = m.w4a8_quant_act(Xd)
    qo, so, _, _ = O.quant_act(np.ascontiguousarray(bits(X)[:, :K]))
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy(), so)
    assert s[0].item() == 0.0 and (q[0] == 0).all()


@pytest.mark.parametrize("bad", [0x7FC0, 0x7F80, 0xFF80])
@pytest.mark.parametrize("rows", [3, 8200])  # one CTA per row / one warp per row
def test_quant_act_flags_nonfinite(m, bad, rows):
    X = torch.ones(rows, 256, dtype=torch.bfloat16)
    X.view(torch.int16)[rows - 2, 17] = np.int16(np.uint16(bad).view(np.int16))
    st = m.new_status("cuda")
    m.w4a8_quant_act(X.cuda(), status=st)
    assert m.w4a8_get_device_status(st) == 4


# ------------------------------------------------------------------ pack ---

@pytest.mark.parametrize("K,N,g,sym", [(512, 512, 128, True), (256, 192, 64, False), (1408, 2816, 128, True),
                                       (2048, 448, 64, False), (4096, 14336, 128, True), (128, 64, 128, False)])
def test_pack_bit_exact(m, K, N, g, sym):
    W = _weights(K, N, K + N, sym, outlier_p=0.001)
    W[:, 3] = 0.0  # an all-zero column: scale 0, codes 0
    st = m.new_status("cuda")
    pw = m.w4a8_pack_weights(W.cuda(), g, sym, status=st)
    codes, s, z, bad = O.quant_weights(W.numpy(), g, sym)
    assert np.array_equal(pw.packed.cpu().numpy(), O.pack_tiled(codes, g))
    assert np.array_equal(pw.s_w.cpu().numpy(), s)
    if not sym:
        assert np.array_equal(pw.z.cpu().numpy(), z)
    assert (pw.desc.bits, pw.desc.symmetric, pw.desc.group, pw.desc.K, pw.desc.N, pw.desc.layout_version) == \
        (4, int(sym), g, K, N, 1)
    assert m.w4a8_get_device_status(st) == 0


def test_pack_flags_nonfinite(m):
    W = torch.zeros(128, 64)
    W[5, 7] = float("nan")
    st = m.new_status("cuda")
    m.w4a8_pack_weights(W.cuda(), 128, True, status=st)
    assert m.w4a8_get_device_status(st) == 4


# ------------------------------------------------------------------ GEMM ---

GEMM_CASES = [
    # (M, K, N, group, symmetric): the correctness config first
    (16, 512, 512, 128, True),
    (1, 512, 512, 128, True),
    (37, 1408, 320, 64, False),     # ragged M, N % 128 == 64 tail, asym g=64
    (200, 1024, 448, 128, False),   # several m-tiles (BN=128) + a ragged one
    (130, 768, 256, 64, True),
    (64, 256, 64, 128, True),       # a single half tile
    (513, 512, 1024, 128, True),    # many tiles, ragged last row block
    (33, 4096, 1024, 128, True),    # BN=64, split-K
    (20, 128, 256, 128, True),      # one group (G = 1)
    (9, 64, 192, 64, False),        # one group, asymmetric, half tile
    (8, 4096, 1024, 128, True),     # split-K: 8 tiles over the SMs, every tile summed from ~16 CTAs
    (5, 2048, 1024, 64, False),     # split-K, asymmetric g=64, ragged M
]


def _gemm_case(m, M, K, N, g, sym, seed, outliers=8):
    inp = gen_linear(M, K, N, seed=seed, n_outliers=min(outliers, K // 4), outlier_scale=50.0)
    W = inp.W if sym else _weights(K, N, seed, sym)
    pw = m.w4a8_pack_weights(W.cuda(), g, sym)
    codes, s, z, _ = O.quant_weights(W.numpy(), g, sym)
    qo, so, _, _ = O.quant_act(bits(inp.X))
    return inp, pw, codes, s, (None if sym else z), qo, so


@pytest.mark.parametrize("M,K,N,g,sym", GEMM_CASES)
def test_gemm_partials_bit_exact_and_output(m, M, K, N, g, sym):
    inp, pw, codes, s, z, qo, so = _gemm_case(m, M, K, N, g, sym, seed=M * 7 + N)
    st = m.new_status("cuda")
    q, sx, _ = m.w4a8_quant_act(inp.X.cuda(), status=st)
    Y, P = m.w4a8_gemm_debug_partials(q, sx, pw, status=st)
    assert m.w4a8_get_device_status(st) == 0
    Po = O.partials(qo, codes, z, g)
    Pg = P.cpu().numpy()
    assert np.array_equal(Pg, Po), f"{int((Pg != Po).sum())} partials differ"
    Ye, A = O.scale_partials(Po, so, s)
    check_bf16(bits(Y), Ye, A)
    # the plain call agrees bit for bit with the debug call
    Y2 = m.w4a8_gemm(q, sx, pw)
    assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16))


def test_gemm_config1_exact_scales(m):
    # X = d R, W = c Q with power-of-two scales: every code and scale is exact,
    # so the bf16 output must be the correctly rounded X @ W.
    rng = np.random.default_rng(0)
    M, K, N, g = 16, 512, 512, 128
    R = rng.integers(-127, 128, size=(M, K)); R[:, 0] = 127
    Q = rng.integers(-7, 8, size=(K, N)); Q[::g, :] = 7
    X = torch.tensor(R * 2.0 ** -3, dtype=torch.float32).to(torch.bfloat16)
    W = torch.tensor(Q * 2.0 ** -6, dtype=torch.float32)
    pw = m.w4a8_pack_weights(W.cuda(), g, True)
    Y = m.w4a8_linear(X.cuda(), pw)
    exact = (R * 2.0 ** -3) @ (Q * 2.0 ** -6)
    assert np.array_equal(bits(Y), O.f64_to_bf16(exact))


@pytest.mark.parametrize("M", [1, 8, 32])
def test_gemm_decode_shapes_full(m, M):
    # Decode-shaped linear: K=4096, N=14336, 8 outlier channels x50, full output.
    K, N, g = 4096, 14336, 128
    inp = gen_linear(M, K, N, seed=0, n_outliers=8, outlier_scale=50.0)
    pw = m.w4a8_pack_weights(inp.W.cuda(), g, True)
    codes, s, _, _ = O.quant_weights(inp.W.numpy(), g, True)
    qo, so, _, _ = O.quant_act(bits(inp.X))
    q, sx, _ = m.w4a8_quant_act(inp.X.cuda())
    assert np.array_equal(q.cpu().numpy(), qo)
    Y, P = m.w4a8_gemm_debug_partials(q, sx, pw)
    Po = O.partials(qo, codes, None, g)
    assert np.array_equal(P.cpu().numpy(), Po)
    Ye, A = O.scale_partials(Po, so, s)
    check_bf16(bits(Y), Ye, A)


@pytest.mark.parametrize("M", [1, 8, 32])
def test_linear_decode_shapes_against_oracle(m, M):
    """The product path itself (w4a8_linear: quantization + the GEMM
    instantiation without the debug write, launched as the bench launches it)
    at the decode shapes, every output element against the oracle."""
    K, N, g = 4096, 14336, 128
    inp = gen_linear(M, K, N, seed=0, n_outliers=8, outlier_scale=50.0)
    pw = m.w4a8_pack_weights(inp.W.cuda(), g, True)
    st = m.new_status("cuda")
    ws = torch.empty(m.w4a8_linear_workspace_size(M, pw), dtype=torch.uint8, device="cuda")
    Y = m.w4a8_linear(inp.X.cuda(), pw, workspace=ws, status=st)
    Y2 = m.w4a8_linear(inp.X.cuda(), pw, workspace=ws, status=st)  # the same workspace again
    assert m.w4a8_get_device_status(st) == 0
    codes, s, _, _ = O.quant_weights(inp.W.numpy(), g, True)
    res = O.linear(bits(inp.X), codes, s, None, g)
    check_bf16(bits(Y), res["Y"], res["absY"], what=f"w4a8_linear M={M}")
    assert np.array_equal(bits(Y2), bits(Y))


def test_gemm_prefill_shape_sampled_rows(m):
    # Prefill-shaped linear at full size (M=8192, K=4096, N=14336): the GPU
    # computes everything in the launch configuration the bench times; the
    # oracle checks a seeded sample of rows (every m-tile position class).
    M, K, N, g = 8192, 4096, 14336, 128
    inp = gen_linear(M, K, N, seed=0, n_outliers=8, outlier_scale=50.0)
    pw = m.w4a8_pack_weights(inp.W.cuda(), g, True)
    st = m.new_status("cuda")
    Y = m.w4a8_linear(inp.X.cuda(), pw, status=st)
    assert m.w4a8_get_device_status(st) == 0
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 4095, 8190, 8191],
                                     np.random.default_rng(1).integers(0, M, 25)]))
    codes, s, _, _ = O.quant_weights(inp.W.numpy(), g, True)
    Xs = bits(inp.X)[rows]
    res = O.linear(Xs, codes, s, None, g)
    check_bf16(bits(Y)[rows], res["Y"], res["absY"])


def test_bounded_wait_reports_timeout(m):
    st = m.new_status("cuda")
    m.w4a8_selftest_bounded_wait(st, limit_ns=2_000_000)
    assert m.w4a8_get_device_status(st) == 5
    # the context is still usable afterwards
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


@pytest.mark.parametrize("M,K,N,group,sym", [(32, 4096, 14336, 128, True), (1, 4096, 14336, 128, True),
                                             (300, 2048, 1024, 128, True), (17, 1024, 512, 64, False)])
def test_linear_one_call_equals_quant_then_gemm(m, M, K, N, group, sym):
    """w4a8_linear (quantization and GEMM in one call, the GEMM launched to
    overlap the quantization) gives bit for bit what the two calls give."""
    inp = gen_linear(M, K, N, seed=M + N)
    W = inp.W if sym else _weights(K, N, 5, False)
    pw = m.w4a8_pack_weights(W.cuda(), group, sym)
    X = inp.X.cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y1 = m.w4a8_linear(X, pw, status=st)
    Y1b = m.w4a8_linear(X, pw, status=st)  # again: the split-K flags of the first call must not leak
    q, s, _ = m.w4a8_quant_act(X)
    Y2 = m.w4a8_gemm(q, s, pw)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(bits(Y1), bits(Y2))
    assert np.array_equal(bits(Y1b), bits(Y2))


def test_gemm_zero_rows_and_zero_groups(m):
    """All-zero activation rows give s_x = 0 and exactly zero outputs; an
    all-zero weight group gives s_w = 0 and contributes nothing (the zero-scale
    reading of "Quantization: formats, error and the real execution path")."""
    M, K, N, g = 24, 1024, 384, 128
    inp = gen_linear(M, K, N, seed=77)
    X = inp.X.clone()
    X[[0, 5, 23]] = 0
    W = inp.W.clone()
    W[128:256, 64:80] = 0          # group 1 of columns 64..79
    W[:, 300] = 0                   # every group of column 300
    pw = m.w4a8_pack_weights(W.cuda(), g, True)
    codes, s, z, _ = O.quant_weights(W.numpy(), g, True)
    assert (s[1, 64:80] == 0).all() and (s[:, 300] == 0).all()
    st = m.new_status("cuda")
    q, sx, _ = m.w4a8_quant_act(X.cuda(), status=st)
    Y, P = m.w4a8_gemm_debug_partials(q, sx, pw, status=st)
    assert m.w4a8_get_device_status(st) == 0
    qo, so, _, _ = O.quant_act(bits(X))
    assert np.array_equal(P.cpu().numpy(), O.partials(qo, codes, None, g))
    Ye, A = O.scale_partials(O.partials(qo, codes, None, g), so, s)
    check_bf16(bits(Y), Ye, A)
    Yb = bits(Y)
    assert (Yb[[0, 5, 23]] & 0x7FFF == 0).all()
    assert (Yb[:, 300] & 0x7FFF == 0).all()


@pytest.mark.parametrize("M", [3, 33, 130])
def test_gemm_strided_output(m, M):
    """Y with a row pitch of N + 3 elements (no 16-byte row stores) holds the
    same bits as a contiguous Y, and the padding is left untouched."""
    K, N = 1024, 512
    inp = gen_linear(M, K, N, seed=M)
    pw = m.w4a8_pack_weights(inp.W.cuda(), 128, True)
    q, sx, _ = m.w4a8_quant_act(inp.X.cuda())
    Yc = m.w4a8_gemm(q, sx, pw)
    big = torch.full((M, N + 3), -7.0, dtype=torch.bfloat16, device="cuda")
    Ys = m.w4a8_gemm(q, sx, pw, out=big[:, :N])
    torch.cuda.synchronize()
    assert Ys.stride(0) == N + 3
    assert np.array_equal(bits(Ys), bits(Yc))
    assert (big[:, N:] == -7.0).all()


@pytest.mark.parametrize("M,K,N,g,sym", [(5, 16384, 384, 128, True), (3, 12288, 320, 64, False)])
def test_gemm_long_k(m, M, K, N, g, sym):
    """Long rows (K = 16384 / 12288: 128 / 192 groups per tile, split-K): the
    quantization reads each row twice (absmax, then codes) and must give the
    oracle's codes bit for bit; the one-call layer gives what quantization +
    GEMM give; partials bit-exact."""
    inp = gen_linear(M, K, N, seed=K + M, n_outliers=8, outlier_scale=50.0)
    W = inp.W if sym else _weights(K, N, 9, False)
    pw = m.w4a8_pack_weights(W.cuda(), g, sym)
    codes, s, z, _ = O.quant_weights(W.numpy(), g, sym)
    qo, so, rso, _ = O.quant_act(bits(inp.X), group=g)
    st = m.new_status("cuda")
    q, sx, rs = m.w4a8_quant_act(inp.X.cuda(), group_for_rowsum=g, status=st)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(sx.cpu().numpy(), so)
    assert np.array_equal(rs.cpu().numpy(), rso)
    Y, P = m.w4a8_gemm_debug_partials(q, sx, pw, status=st)
    Y1 = m.w4a8_linear(inp.X.cuda(), pw, status=st)
    assert m.w4a8_get_device_status(st) == 0
    Po = O.partials(qo, codes, None if sym else z, g)
    assert np.array_equal(P.cpu().numpy(), Po)
    Ye, A = O.scale_partials(Po, so, s)
    check_bf16(bits(Y), Ye, A)
    assert np.array_equal(bits(Y1), bits(Y))


@pytest.mark.parametrize("M,K", [(3, 8200), (70, 16384), (2, 32768)])
def test_quant_act_long_rows_bit_exact(m, M, K):
    """Rows beyond 8192 elements (two passes over the row), with code sums."""
    inp = gen_linear(M, K, 64, seed=M + K, n_outliers=8, outlier_scale=50.0)
    st = m.new_status("cuda")
    q, s, rs = m.w4a8_quant_act(inp.X.cuda(), group_for_rowsum=64 if K % 64 == 0 else 0, status=st)
    qo, so, rso, bad = O.quant_act(bits(inp.X), group=64 if K % 64 == 0 else 0)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy(), so)
    if K % 64 == 0:
        assert np.array_equal(rs.cpu().numpy(), rso)
    assert m.w4a8_get_device_status(st) == 0 and not bad
