"""Pins for the CPU oracle, independent of the oracle itself.

Each test ties the oracle to something the pages or the mathematics fix:
values printed on the pages (tests/golden/*), closed forms, exact special
cases, invariants, brute force on tiny inputs.  The cases are chosen so that a
plausible slip in the oracle (a dropped zero-point term, a wrong sign, a
transposed operand, a wrong group index, multiplying by a reciprocal instead
of dividing) fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle as O
from oracle import OracleError


def _bf16_bits(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- INT8 act --

def test_worked_int8_example_linear_s2(orc, golden):
    g = golden("lin_s2_worked_int8.txt")
    x = np.array([float(v) for v in g["input"]], np.float32)
    q, s, bad = orc.quant_row_f32(x)
    assert not bad
    assert q.tolist() == [int(v) for v in g["codes"]]
    assert round(float(s), 4) == float(g["scale_printed"][0])
    # The page's dequantized values come from its rounded scale 0.0063 (with
    # half-up printing: 95 * 0.0063 = 0.5985 -> 0.599); with the exact scale
    # the values agree with the printed ones to the printed precision.
    from decimal import Decimal, ROUND_HALF_UP
    printed = [Decimal(v) for v in g["dequant_printed"]]
    s_pr = Decimal(g["scale_printed"][0])
    assert [(int(c) * s_pr).quantize(Decimal("0.001"), ROUND_HALF_UP) for c in q] == printed
    deq = q.astype(np.float64) * float(s)
    assert np.all(np.abs(deq - np.array([float(v) for v in printed])) <= 1e-3)


def test_worked_int8_example_survives_bf16_inputs(orc, golden):
    # The act path takes bf16 rows; the page's values rounded to bf16 keep
    # the printed codes (the quotients move by < 0.1, far from a .5 tie).
    g = golden("lin_s2_worked_int8.txt")
    xb = _bf16_bits([float(v) for v in g["input"]])
    q, s, _, bad = orc.quant_act(xb[None, :])
    assert q[0].tolist() == [int(v) for v in g["codes"]]
    assert round(float(s[0]), 4) == float(g["scale_printed"][0])


def test_outlier_example_linear_s5(orc, golden):
    g = golden("lin_s5_outlier.txt")
    x = np.array([float(v) for v in g["input"]], np.float32)
    q, s, _ = orc.quant_row_f32(x)
    assert round(float(s), 3) == float(g["scale_printed"][0])
    quo = x / np.float32(s)
    assert [round(float(v), 3) for v in quo] == [float(v) for v in g["quotients_printed"]]
    assert q.tolist() == [int(v) for v in g["codes"]]


def test_act_quant_brute_force_small():
    # Brute force: the code is the integer c in [-127,127] nearest to the fp32
    # quotient x/s, ties to even; checked against an enumeration.
    import oracle
    rng = np.random.default_rng(1)
    for _ in range(50):
        x = (rng.standard_normal(7) * rng.choice([1e-3, 1, 50])).astype(np.float32)
        q, s, _ = oracle.quant_row_f32(x)
        assert s == np.float32(np.max(np.abs(x))) / np.float32(127)
        for xi, qi in zip(x, q):
            t = np.float32(xi) / np.float32(s)
            best = min(range(-127, 128), key=lambda c: (abs(float(t) - c), c % 2))
            assert qi == best


def test_act_quant_zero_row_and_nonfinite(orc):
    q, s, _, bad = orc.quant_act(np.zeros((2, 8), np.uint16))
    assert not bad and np.all(q == 0) and np.all(s == 0)
    X = _bf16_bits(np.ones((2, 8)))
    X[1, 3] = 0x7FC0  # NaN
    _, _, _, bad = orc.quant_act(X)
    assert bad
    X[1, 3] = 0x7F80  # +Inf
    _, _, _, bad = orc.quant_act(X)
    assert bad


def test_act_quant_clamp_never_needed():
    # s = amax/127 exactly rounded: |x/s| <= 127 (1 + 2^-23) so the RNE code
    # of the largest element is exactly +-127.
    rng = np.random.default_rng(2)
    for _ in range(200):
        x = rng.standard_normal(33).astype(np.float32) * np.float32(rng.uniform(1e-30, 1e30))
        q, s, _ = O.quant_row_f32(x)
        assert abs(int(q[np.argmax(np.abs(x))])) == 127


def test_rowsum_zero_point_expansion_identity(orc):
    # "Inference Quantization ch.1" §7: sum q_x (q_w - z) = sum q_x q_w - z sum q_x.
    rng = np.random.default_rng(3)
    M, K, N, g = 5, 128, 64, 64
    X = _bf16_bits(rng.standard_normal((M, K)))
    W = (rng.standard_normal((K, N)) * 0.02 + 0.01).astype(np.float32)
    q, s, rs, _ = orc.quant_act(X, group=g)
    codes, sw, z, _ = orc.quant_weights(W, g, symmetric=False)
    P = orc.partials(q, codes, z, g)
    for gi in range(K // g):
        sl = slice(gi * g, (gi + 1) * g)
        raw = q[:, sl].astype(np.int64) @ codes[:, sl].astype(np.int64).T
        assert np.array_equal(rs[:, gi], q[:, sl].astype(np.int64).sum(1))
        expanded = raw - rs[:, gi][:, None].astype(np.int64) * z[gi][None, :].astype(np.int64)
        assert np.array_equal(P[:, gi, :], expanded)


# ------------------------------------------------------------- 4-bit wts ---

def test_qfmt_group_reference_invariants(orc, golden):
    gd = golden("qfmt_group_reference.txt")
    x = np.array([[float(v) for v in gd["row0"]], [float(v) for v in gd["row1"]]], np.float32)
    group = int(gd["group"][0])
    # oracle groups along K of W[K, N]: the page's rows are output columns.
    codes, s, z, bad = orc.quant_weights(x.T.copy(), group, symmetric=True)
    assert not bad
    assert codes.min() >= -7 and codes.max() <= 7
    num0, den0 = map(float, gd["scale_row0_max_over_qmax"])
    num1, den1 = map(float, gd["scale_row1_max_over_qmax"])
    assert s[0, 0] == np.float32(num0) / np.float32(den0)
    assert s[0, 1] == np.float32(num1) / np.float32(den1)
    xhat = codes.astype(np.float32) * s[0][:, None]
    slack = float(gd["error_bound_slack"][0])
    assert np.all(np.abs(x - xhat) <= s[0][:, None] / 2 + slack)


def test_qfmt_zero_group_and_reject(orc, golden):
    gd = golden("qfmt_group_reference.txt")
    codes, s, z, bad = orc.quant_weights(np.zeros((4, 1), np.float32), 4, True)
    assert np.all(codes == 0) and s[0, 0] == 0.0
    assert np.all(orc.dequant_weights(codes, s, None, 4) == 0.0)
    rows, cols = map(int, gd["reject_shape"])
    with pytest.raises(OracleError):
        orc.quant_weights(np.ones((cols, rows), np.float32), int(gd["reject_group"][0]), True)


def test_fp32_quotient_decides_the_code():
    # 0.5 / fp32(1/7) is 3.4999998 in binary32, so the code is 3; a real-number
    # quotient (3.5) would round to 4.  The oracle follows the binary32 form.
    x = np.array([[0.0, -1.0, 0.5, 0.25]], np.float32)
    codes, s, _, _ = O.quant_weights(x.T.copy(), 4, True)
    assert np.float32(0.5) / s[0, 0] < np.float32(3.5)
    assert codes[0].tolist() == [0, -7, 3, 2]


def test_symmetric_invariants_random():
    rng = np.random.default_rng(4)
    for g in (64, 128):
        W = (rng.standard_normal((256, 96)) * 0.02).astype(np.float32)
        W[rng.random(W.shape) < 0.001] *= 20
        codes, s, z, _ = O.quant_weights(W, g, True)
        assert codes.min() >= -7 and codes.max() <= 7
        What = O.dequant_weights(codes, s, None, g)
        sk = np.repeat(s, g, axis=0)
        assert np.all(np.abs(W - What) <= sk / 2 * (1 + 1e-6) + 1e-12)
        # absmax element of every group maps to +-7
        for gi in range(256 // g):
            blk = W[gi * g:(gi + 1) * g]
            am = np.argmax(np.abs(blk), axis=0)
            assert np.all(np.abs(codes[np.arange(96), gi * g + am]) == 7)


def test_per_channel_special_case_group_equals_K():
    # "Inference Quantization ch.1" §8.2: per-channel weight scale s_w in R^N is
    # the group-wise scheme with one group spanning K.
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((128, 40)) * 0.02).astype(np.float32)
    codes, s, _, _ = O.quant_weights(W, 128, True)
    assert s.shape == (1, 40)
    assert np.array_equal(s[0], np.max(np.abs(W), axis=0) / np.float32(7))


def test_asymmetric_invariants_random():
    rng = np.random.default_rng(6)
    g = 64
    W = (rng.standard_normal((256, 80)) * 0.02 + rng.uniform(-0.03, 0.03, 80)).astype(np.float32)
    W[rng.random(W.shape) < 0.001] *= 20
    codes, s, z, _ = O.quant_weights(W, g, False)
    assert codes.min() >= 0 and codes.max() <= 15 and z.max() <= 15
    What = O.dequant_weights(codes, s, z, g)
    sk = np.repeat(s, g, axis=0)
    assert np.all(np.abs(W - What) <= sk * (1 + 1e-6))
    for gi in range(256 // g):
        blk = W[gi * g:(gi + 1) * g]
        lo_k = np.argmin(blk, axis=0) + gi * g
        hi_k = np.argmax(blk, axis=0) + gi * g
        n = np.arange(80)
        neg = blk.min(0) < 0
        assert np.all(codes[n, lo_k][neg] == 0)  # the group minimum maps to 0
        pos = blk.max(0) > 0
        assert np.all(codes[n, hi_k][pos] >= 14)
        # Cross-check with the deployment page's float-offset form
        # (q = round((w - min)/s), w_hat = q s + min): both within s of w.
        lo = np.minimum(blk.min(0), 0)
        qf = np.clip(np.rint((blk - lo) / s[gi]), 0, 15)
        assert np.all(np.abs(qf * s[gi] + lo - blk) <= s[gi] * (0.5 + 1e-6))


def test_asymmetric_constant_group():
    W = np.full((64, 3), 0.37, np.float32)
    W[:, 1] = -0.5
    W[:, 2] = 0.0
    codes, s, z, _ = O.quant_weights(W, 64, False)
    What = O.dequant_weights(codes, s, z, 64)
    assert np.allclose(What[:, :2], W[:, :2], rtol=1e-6, atol=0)
    assert np.all(What[:, 2] == 0) and s[0, 2] == 0 and z[0, 2] == 0


# ----------------------------------------------------------------- packing --

def _unpack_canonical(b, K):
    lo = (b & 0xF).astype(np.int16)
    hi = (b >> 4).astype(np.int16)
    out = np.empty((b.shape[0], K), np.int16)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def test_pack_canonical_bijection():
    rng = np.random.default_rng(7)
    codes = rng.integers(-7, 8, size=(64, 256)).astype(np.int8)
    b = O.pack_canonical(codes)
    nib = _unpack_canonical(b, 256)
    signed = np.where(nib >= 8, nib - 16, nib)
    assert np.array_equal(signed, codes)
    u = rng.integers(0, 16, size=(64, 256)).astype(np.int8)
    assert np.array_equal(_unpack_canonical(O.pack_canonical(u), 256), u)


def test_pack_tiled_positions_by_hand():
    # Written-out positions of the device layout for g = 128, K = 256, N = 128:
    # block (nb, gi) at (nb*G + gi)*4096, chunk (c, r) at (c*64 + r)*16,
    # byte b: low nibble k = gi*128 + 32c + b, high nibble k + 16.
    K, N, g = 256, 128, 128
    codes = np.zeros((N, K), np.int8)
    codes[70, 128 + 32 * 2 + 5] = 3       # nb=1, r=6, gi=1, c=2, b=5 (low)
    codes[70, 128 + 32 * 2 + 16 + 5] = -2  # same byte, high nibble
    codes[1, 31] = 7                       # nb=0, r=1, gi=0, c=0, b=15 (high)
    t = O.pack_tiled(codes, g)
    G = K // g
    off1 = (1 * G + 1) * 4096 + (2 * 64 + 6) * 16 + 5
    off2 = (0 * G + 0) * 4096 + (0 * 64 + 1) * 16 + 15
    assert t[off1] == (3 | (0xE << 4))
    assert t[off2] == (7 << 4)
    nz = np.nonzero(t)[0]
    assert sorted(nz.tolist()) == sorted([off1, off2])


def test_pack_tiled_is_a_permutation_of_codes():
    rng = np.random.default_rng(8)
    for g in (64, 128):
        K, N = 256, 192
        codes = rng.integers(0, 16, size=(N, K)).astype(np.int8)
        t = O.pack_tiled(codes, g)
        assert t.size == N * K // 2
        hist_t = np.bincount(np.concatenate([t & 0xF, t >> 4]), minlength=16)
        hist_c = np.bincount(codes.ravel(), minlength=16)
        assert np.array_equal(hist_t, hist_c)


# ------------------------------------------------------------------- GEMM ---

def _exact_case(rng, M, K, N, g, symmetric):
    """X = d R, W = c (Q - z) built so that every scale comes out exact and the
    codes are R and Q: then the oracle's Y must equal X @ W exactly."""
    R = rng.integers(-127, 128, size=(M, K))
    R[np.arange(M), rng.integers(0, K, M)] = rng.choice([-127, 127], M)
    d = np.float32(2.0 ** -3)
    G = K // g
    cexp = rng.integers(-9, -3, size=(G, N))
    c = (2.0 ** cexp).astype(np.float32)
    if symmetric:
        Q = rng.integers(-7, 8, size=(N, K))
        z = np.zeros((G, N), np.int64)
        for gi in range(G):
            Q[np.arange(N), gi * g + rng.integers(0, g, N)] = rng.choice([-7, 7], N)
    else:
        Q = rng.integers(0, 16, size=(N, K))
        z = rng.integers(0, 16, size=(G, N))
        for gi in range(G):
            pos = rng.permutation(g)[:2] + gi * g
            Q[np.arange(N), pos[0]] = 0
            Q[np.arange(N), pos[1]] = 15
    X = (R * d).astype(np.float32)
    zk = np.repeat(z, g, axis=0).T  # [N, K]
    W = (np.repeat(c, g, axis=0).T * (Q - zk)).T.astype(np.float32)  # [K, N]
    return X, W, R, Q, z


@pytest.mark.parametrize("symmetric,g", [(True, 128), (True, 64), (False, 64), (False, 128)])
def test_linear_exact_when_scales_are_exact(symmetric, g):
    rng = np.random.default_rng(9 + g + symmetric)
    M, K, N = 6, 256, 64
    X, W, R, Q, z = _exact_case(rng, M, K, N, g, symmetric)
    Xb = _bf16_bits(X)
    assert np.array_equal(O.bf16_to_f32(Xb), X)  # exact in bf16
    codes, s, zz, _ = O.quant_weights(W, g, symmetric)
    assert np.array_equal(codes, Q)
    if not symmetric:
        assert np.array_equal(zz, z)
    res = O.linear(Xb, codes, s, None if symmetric else zz, g)
    assert np.array_equal(res["q"], R)
    truth = X.astype(np.float64) @ W.astype(np.float64)
    assert np.array_equal(res["Y"], truth)


def test_factorised_equals_dequantize_then_gemm():
    # spec identity: the binary64 dequantize-then-GEMM form equals the
    # factorised per-group scale form up to binary64 rounding.
    rng = np.random.default_rng(10)
    for symmetric, g in ((True, 128), (False, 64)):
        M, K, N = 7, 384, 64
        Xb = _bf16_bits(rng.standard_normal((M, K)) * np.array([1] * 380 + [50] * 4))
        W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
        codes, s, z, _ = O.quant_weights(W, g, symmetric)
        zz = None if symmetric else z
        res = O.linear(Xb, codes, s, zz, g)
        Yd = O.dequant_gemm(res["q"], res["s_x"], codes, s, zz, g)
        assert np.all(np.abs(res["Y"] - Yd) <= 1e-12 * res["absY"] + 1e-300)


def test_partials_brute_force_tiny():
    rng = np.random.default_rng(11)
    M, K, N, g = 2, 64, 64, 32
    qx = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    codes = rng.integers(0, 16, size=(N, K)).astype(np.int8)
    z = rng.integers(0, 16, size=(K // g, N)).astype(np.uint8)
    P = O.partials(qx, codes, z, g)
    for m, gi, n in itertools.product(range(M), range(K // g), range(0, N, 7)):
        ref = sum(int(qx[m, k]) * (int(codes[n, k]) - int(z[gi, n])) for k in range(gi * g, gi * g + g))
        assert P[m, gi, n] == ref


def test_accumulator_bound_fits_int32():
    # "Correctness contract": the accumulator must cover the reduction range.
    qx = np.full((1, 128), -127, np.int8)
    codes = np.full((64, 128), 0, np.int8)
    z = np.full((1, 64), 15, np.uint8)
    P = O.partials(qx, codes, z, 128)
    assert P[0, 0, 0] == 128 * 127 * 15 < 2 ** 22


# ------------------------------------------------------------------ bf16 ----

def test_bf16_rounding_matches_torch_for_binary32_values():
    rng = np.random.default_rng(12)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(1e3),
        (rng.standard_normal(2000) * 1e-38).astype(np.float32),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.3895314e38, 3.39e38, -3.39e38,
                  1e-45, 9.2e-41, np.inf, -np.inf], np.float32)])
    ours = O.f64_to_bf16(x.astype(np.float64))
    ref = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert O.f64_to_bf16(np.array([np.nan]))[0] & 0x7F80 == 0x7F80


def test_bf16_rounding_is_single_rounding_from_binary64():
    # 1 + 2^-8 + 2^-30 is just above a bf16 tie: correct rounding goes up,
    # while rounding through binary32 first would land on the tie and go down.
    y = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert O.f64_to_bf16(np.array([y]))[0] == 0x3F81
    assert O.f64_to_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80


# ---------------------------------------------------------------- routing ---

def test_route_brute_force_and_softmax():
    rng = np.random.default_rng(13)
    T, E, k = 9, 6, 3
    L = rng.standard_normal((T, E)).astype(np.float32)
    L[2, 1] = L[2, 4] = L[2].max() + 1  # a tie for the top slot
    idx, p, bad = O.route(L, k)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(L[t, e]), e))[:k]
        assert idx[t].tolist() == order
        ex = np.exp(L[t].astype(np.float64) - L[t].max())
        assert np.allclose(p[t], ex[order] / ex.sum(), rtol=1e-14, atol=0)
    assert idx[2, 0] == 1 and idx[2, 1] == 4


def test_dispatch_invariants_and_order():
    rng = np.random.default_rng(14)
    T, E, k = 37, 8, 3
    L = rng.standard_normal((T, E)).astype(np.float32)
    idx, _, _ = O.route(L, k)
    off, perm, inv = O.dispatch(idx, E)
    assert off[0] == 0 and off[-1] == T * k and np.all(np.diff(off) >= 0)
    assert np.array_equal(perm[inv], np.arange(T * k))
    assert np.array_equal(np.bincount(perm // k, minlength=T), np.full(T, k))
    keys = [(int(idx.ravel()[pid]), int(pid // k), int(pid % k)) for pid in perm]
    assert keys == sorted(keys)
    for e in range(E):
        assert np.all(idx.ravel()[perm[off[e]:off[e + 1]]] == e)


def test_combine_uniform_weights_is_a_mean():
    # k = E with equal logits: every weight is 1/E, so the combine is the plain
    # mean of the E expert rows of each token.
    rng = np.random.default_rng(15)
    T, E, Hd = 5, 4, 16
    idx, p, _ = O.route(np.zeros((T, E), np.float32), E)
    assert np.all(p == 0.25)
    off, perm, inv = O.dispatch(idx, E)
    Yd = _bf16_bits(rng.standard_normal((T * E, Hd)))
    out, out64 = O.combine(Yd, p, inv)
    rows = O.bf16_to_f32(Yd).astype(np.float64)[inv.reshape(T, E)]
    assert np.allclose(out64, rows.mean(1), rtol=1e-15, atol=1e-300)
    assert np.array_equal(out, O.f64_to_bf16(rows.mean(1)))


def test_silu_closed_forms():
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(1.0) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-16
    for x in (0.3, 2.0, 7.5):
        assert abs((O.silu(x) - O.silu(-x)) - x) < 1e-14
    assert abs(O.silu(40.0) - 40.0) < 1e-12
    h = O.silu_mul(np.array([[1.0, -2.0, 3.0, 0.5]]))
    assert np.array_equal(h, O.f64_to_bf16(np.array([[O.silu(1.0) * 3.0, O.silu(-2.0) * 0.5]])))


def test_moe_forward_tiny_against_dense_dequant():
    # Tiny MoE through the oracle; each token's output equals the weighted sum
    # of its experts, each computed by dequantize-then-GEMM on the same codes.
    rng = np.random.default_rng(16)
    T, H, E, k, I, g = 6, 128, 4, 2, 64, 64
    Xb = _bf16_bits(rng.standard_normal((T, H)))
    L = rng.standard_normal((T, E)).astype(np.float32)
    w1, w2 = [], []
    for e in range(E):
        c, s, z, _ = O.quant_weights((rng.standard_normal((H, 2 * I)) * 0.02).astype(np.float32), g, False)
        w1.append((c, s, z))
        c, s, z, _ = O.quant_weights((rng.standard_normal((I, H)) * 0.02).astype(np.float32), g, False)
        w2.append((c, s, z))
    r = O.moe_forward(Xb, L, k, w1, w2, g)
    for t in range(T):
        acc = np.zeros(H)
        for j in range(k):
            e = r["idx"][t, j]
            pos = r["inv"][t * k + j]
            Hg = O.dequant_gemm(r["qx"][t:t + 1], r["sx"][t:t + 1], *w1[e], g)[0]
            assert np.allclose(Hg, r["H"][pos], rtol=1e-12, atol=1e-12)
            hh = O.silu_mul(Hg[None])
            qh, sh, _, _ = O.quant_act(hh)
            yd = O.dequant_gemm(qh, sh, *w2[e], g)[0]
            acc += r["p"][t, j] * O.bf16_to_f32(O.f64_to_bf16(yd)).astype(np.float64)
        assert np.allclose(acc, r["out64"][t], rtol=1e-12, atol=1e-12)


# ------------------------------------------------------- W8A8 per-channel --

def test_w8_per_channel_worked_example_linear_s2(orc, golden):
    """The §2 worked example quantizes a weight vector: as one output column
    of W it must give the printed codes and scale."""
    g = golden("lin_s2_worked_int8.txt")
    W = np.array([[float(v)] for v in g["input"]], np.float32)  # [K=4, N=1]
    q, s, bad = orc.quant_w8(W)
    assert not bad
    assert q[:, 0].tolist() == [int(v) for v in g["codes"]]
    assert round(float(s[0]), 4) == float(g["scale_printed"][0])


def test_w8_columns_are_independent_and_zero_column():
    """Per-channel: scaling one column by a power of two scales its s_w and
    leaves its codes and every other column unchanged; an all-zero column
    gives s = 0 and codes 0 (the zero-scale reading)."""
    import oracle as O
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((256, 5)) * 0.02).astype(np.float32)
    W[:, 2] = 0.0
    q, s, _ = O.quant_w8(W)
    W2 = W.copy()
    W2[:, 1] *= 8.0
    q2, s2, _ = O.quant_w8(W2)
    assert np.array_equal(q, q2)
    assert s2[1] == np.float32(8.0) * s[1]
    assert np.array_equal(np.delete(s, 1), np.delete(s2, 1))
    assert s[2] == 0.0 and not q[:, 2].any()
    assert np.abs(q).max() <= 127 and (np.abs(q).max(axis=0)[[0, 1, 3, 4]] == 127).all()


def test_w8a8_factorised_equals_dequantize_then_gemm():
    """§4: s_x s_w (X_int8 W_int8) equals the product of the dequantized
    operands (both in binary64; the integer sum is exact)."""
    import oracle as O
    rng = np.random.default_rng(4)
    qx = rng.integers(-127, 128, size=(7, 384)).astype(np.int8)
    qw = rng.integers(-127, 128, size=(384, 33)).astype(np.int8)
    sx = rng.uniform(1e-3, 1e-1, size=7).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-2, size=33).astype(np.float32)
    Y, A, _ = O.w8a8_exact(qx, sx, qw, sw)
    Yd = O.w8a8_dequant_gemm(qx, sx, qw, sw)
    assert np.all(np.abs(Y - Yd) <= 1e-12 * A)


def test_w8a8_integer_sum_brute_force():
    import oracle as O
    rng = np.random.default_rng(5)
    qx = rng.integers(-127, 128, size=(3, 20)).astype(np.int8)
    qw = rng.integers(-127, 128, size=(20, 4)).astype(np.int8)
    _, _, acc = O.w8a8_exact(qx, np.ones(3, np.float32), qw, np.ones(4, np.float32))
    for m in range(3):
        for n in range(4):
            assert acc[m, n] == sum(int(qx[m, k]) * int(qw[k, n]) for k in range(20))


# ------------------------------------------------------- W4A16 weight-only --

def test_w4a16_dequant_worked_example_linear_s2(orc, golden):
    """§2 dequantizes the worked example's codes as s_w * W_int; the weight-only
    dequant (codes as one column, one group) gives the printed values before
    its bf16 rounding, and its bf16 rounding is within half a bf16 ulp."""
    g = golden("lin_s2_worked_int8.txt")
    codes = np.array([[int(v) for v in g["codes"]]], np.int8)          # [N=1, K=4]
    s = np.array([[np.float32(0.8) / np.float32(127.0)]], np.float32)    # [G=1, N=1]
    w32 = orc.w4a16_dequant_f32(codes, s, None, 4)[:, 0]
    # the page prints its values from the rounded scale 0.0063, so the exact
    # scale's values agree with them to the printed precision
    printed = np.array([float(v) for v in g["dequant_printed"]])
    assert np.all(np.abs(w32.astype(np.float64) - printed) <= 1e-3)
    assert np.array_equal(w32, codes[0].astype(np.float32) * s[0, 0])
    wb = orc.bf16_to_f32(orc.w4a16_dequant(codes, s, None, 4))[:, 0].astype(np.float64)
    assert np.all(np.abs(wb - w32) <= np.abs(w32) * 2.0 ** -8)  # half a bf16 ulp


def test_w4a16_dequant_by_hand_asymmetric_groups():
    """Asymmetric, group 2, K = 4: q = [0, 15, 7, 8], z = [7, 8], s = [0.5, 0.25]
    -> s (q - z) = [-3.5, 4.0, -0.25, 0.0] (all exact in bf16); the group
    index follows k, never the column."""
    import oracle as O
    codes = np.array([[0, 15, 7, 8], [8, 7, 15, 0]], np.int8)           # [N=2, K=4]
    z = np.array([[7, 8], [8, 7]], np.uint8)                             # [G=2, N=2]
    s = np.array([[0.5, 1.0], [0.25, 2.0]], np.float32)
    w = O.bf16_to_f32(O.w4a16_dequant(codes, s, z, 2)).astype(np.float64)
    assert w[:, 0].tolist() == [-3.5, 4.0, -0.25, 0.0]
    # column 1: s = 1 on k 0-1, 2 on k 2-3; q - z = [0, -1, 8, -7]
    assert w[:, 1].tolist() == [0.0, -1.0, 16.0, -14.0]


def test_w4a16_dequant_rounds_the_fp32_product_then_to_bf16():
    """The reading: one binary32 product, then bf16.  s = 0x3F95AAAB
    (1.16927087306976318359375), q - z = 3: the exact product is
    3.5078125 + 2^-23, a binary32 tie that rounds to even, 3.5078125; that
    is the bf16 midpoint of 3.5 and 3.515625, which rounds to even: 3.5
    (0x4060).  Rounding the exact product straight to bf16 would give
    3.515625 (0x4061)."""
    import oracle as O
    s = np.array([0x3F95AAAB], np.uint32).view(np.float32).reshape(1, 1)
    codes = np.array([[3]], np.int8)
    assert float(O.w4a16_dequant_f32(codes, s, None, 1)[0, 0]) == 3.5078125
    assert int(O.w4a16_dequant(codes, s, None, 1)[0, 0]) == 0x4060


def test_w4a16_gemm_by_hand_and_zero_codes():
    """Y = X w_hat: X = [1, 2, -1, 0.5] against the column [-3.5, 4, -0.25, 0]
    gives -3.5 + 8 + 0.25 = 4.75; codes equal to their zero-points give 0."""
    import oracle as O
    codes = np.array([[0, 15, 7, 8]], np.int8)
    z = np.array([[7], [8]], np.uint8)
    s = np.array([[0.5], [0.25]], np.float32)
    Wh = O.w4a16_dequant(codes, s, z, 2)
    X = O.f64_to_bf16(np.array([[1.0, 2.0, -1.0, 0.5]]))
    Y, A = O.w4a16_gemm(X, Wh)
    assert Y[0, 0] == 4.75 and A[0, 0] == 3.5 + 8.0 + 0.25
    Wz = O.w4a16_dequant(np.array([[7, 7, 8, 8]], np.int8), s, z, 2)
    assert not O.w4a16_gemm(X, Wz)[0].any()


def test_w4a16_within_bf16_rounding_of_the_exact_dequant():
    """The weight-only product differs from X times the exact dequantized
    weight (the W4A8 oracle's binary64 s (q - z)) only by the weights' bf16
    rounding: |Y - Y_exact| <= 2^-8 sum |x| |w| (fp32 then bf16 rounding,
    each at most half an ulp)."""
    import oracle as O
    rng = np.random.default_rng(6)
    K, N = 256, 64
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    for sym in (True, False):
        codes, s, z, _ = O.quant_weights(W, 64, sym)
        zz = None if sym else z
        Wh = O.w4a16_dequant(codes, s, zz, 64)
        Wx = O.dequant_weights(codes, s, zz, 64)                    # binary64 [K, N]
        X = O.f64_to_bf16(rng.standard_normal((5, K)))
        Xf = O.bf16_to_f32(X).astype(np.float64)
        Y, _ = O.w4a16_gemm(X, Wh)
        Yx = Xf @ Wx
        assert np.all(np.abs(Y - Yx) <= 2.0 ** -8 * (np.abs(Xf) @ np.abs(Wx)) + 1e-30)
