"""GPU parity of the MoE layer against the CPU oracle, stage by stage.

Each stage is checked on the GPU's own input to that stage:
  routing indices, dispatch offsets / order: bit-exact;
  routing weights: within the fp32 softmax bound (E + 4) * 2^-24 relative;
  quantized activations in dispatch order: bit-exact;
  h = silu(gate) * up: 1 bf16 ulp, or the propagated fp32 accumulation bound;
  quantized h: bit-exact (given the GPU's h);
  expert outputs (bf16): 1 bf16 ulp, or the fp32 accumulation bound;
  combine: 1 bf16 ulp of the combine of the GPU's expert outputs, or the fp32
  bound relative to sum_j |p y|;
  end to end against the all-binary64 oracle: relative RMS <= 1e-2.
"""
import numpy as np
import pytest
import torch

import oracle as O
from synth import gen_moe_activations, gen_expert_weight
from tests._util import bf16_ordinal, bf16_ulp, bits, check_bf16, record_fallback

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    from moe_linear_layers_w4a8_b200 import _build
    _build.build()
    import moe_linear_layers_w4a8_b200 as mm
    mm.load_library()
    return mm


def _ws_view(ws, off, count, dtype, width=1):
    nbytes = count * width * torch.tensor([], dtype=dtype).element_size()
    return ws[off:off + nbytes].view(dtype).view(count, width) if width > 1 else ws[off:off + nbytes].view(dtype)


class Layer:
    """A MoE layer's weights: packed on the GPU, oracle codes on demand."""

    def __init__(self, m, seed, E, H, I, group, sym, w_outlier_p, device="cuda"):
        self.seed, self.E, self.H, self.I, self.group, self.sym = seed, E, H, I, group, sym
        self.p = w_outlier_p
        self.w1 = m.w4a8_pack_expert_weights(lambda e: self.W(e, 0, device), E, H, 2 * I, group, sym, device)
        self.w2 = m.w4a8_pack_expert_weights(lambda e: self.W(e, 1, device), E, I, H, group, sym, device)
        self._codes = {}

    def W(self, e, which, device="cuda"):
        K, N = (self.H, 2 * self.I) if which == 0 else (self.I, self.H)
        W = gen_expert_weight(self.seed, e, which, K, N, outlier_p=self.p, device=device)
        if not self.sym:
            W = W + 0.01  # offset distributions exercise the zero-point
        return W

    def codes(self, e, which):
        key = (e, which)
        if key not in self._codes:
            W = self.W(e, which, "cuda").cpu().numpy()
            c, s, z, _ = O.quant_weights(W, self.group, self.sym)
            self._codes[key] = (c, s, None if self.sym else z)
        return self._codes[key]


def pair_slots(T, topk, tokens):
    """int32 [T*topk]: the partials row of every pair of the sampled tokens
    (token tokens[i], slot j -> i*topk + j), -1 elsewhere."""
    ps = torch.full((T * topk,), -1, dtype=torch.int32)
    for i, t in enumerate(tokens):
        for j in range(topk):
            ps[int(t) * topk + j] = i * topk + j
    return ps


def run_layer(m, layer, inp, topk, tokens=None):
    """Runs the layer; with `tokens`, through the debug entry that also returns
    the exact int32 group partials of those tokens' pairs (P1, P2)."""
    st = m.new_status("cuda")
    T = inp.X.shape[0]
    ps = None if tokens is None else pair_slots(T, topk, tokens).cuda()
    res = m.w4a8_moe_grouped_gemm(inp.X.cuda(), inp.logits.cuda(), topk, layer.w1, layer.w2, status=st,
                                  debug_pair_slot=ps)
    assert m.w4a8_get_device_status(st) == 0
    return res


def sample_tokens(T, n, seed, extra=()):
    """Sorted unique token indices: `extra` plus n seeded draws."""
    t = np.random.default_rng(seed).choice(T, min(n, T), replace=False)
    return np.asarray(sorted(set(int(x) for x in np.concatenate([np.asarray(extra, dtype=np.int64), t]))))


def check_layer(m, layer, inp, topk, res, tokens=None):
    T, H = inp.X.shape
    E, I, g = layer.E, layer.I, layer.group
    R = T * topk
    lay = m.w4a8_moe_workspace_layout(T, E, topk, layer.w1, layer.w2)
    ws = res["workspace"]

    # routing + dispatch (all tokens)
    idx_o, p_o, _ = O.route(inp.logits.numpy(), topk)
    idx = res["topk_idx"].cpu().numpy()
    assert np.array_equal(idx, idx_o)
    p = res["topk_w"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(p - p_o) <= (E + 4) * 2.0 ** -24 * p_o + 1e-30)
    off_o, perm_o, inv_o = O.dispatch(idx_o, E)
    assert np.array_equal(res["expert_offsets"].cpu().numpy(), off_o)
    perm = _ws_view(ws, lay["perm"], R, torch.int32).cpu().numpy()
    inv = _ws_view(ws, lay["inv"], R, torch.int32).cpu().numpy()
    assert np.array_equal(perm, perm_o) and np.array_equal(inv, inv_o)

    if tokens is None:
        tokens = np.arange(T)
    tokens = np.asarray(sorted(set(int(t) for t in tokens)))
    rows = np.array([inv[t * topk + j] for t in tokens for j in range(topk)])
    expert_of_row = np.searchsorted(off_o, rows, side="right") - 1
    # partials row of each dispatch row (the debug entry's pair slots)
    tok_pos = {int(t): i for i, t in enumerate(tokens)}
    slot_of_row = np.array([tok_pos[int(perm[r]) // topk] * topk + int(perm[r]) % topk for r in rows])
    P1 = res["P1"].cpu().numpy() if "P1" in res else None
    P2 = res["P2"].cpu().numpy() if "P2" in res else None

    # quantized X in dispatch order
    qx_o, sx_o, _, _ = O.quant_act(bits(inp.X)[tokens])
    qx = _ws_view(ws, lay["qx"], R, torch.int8, H).cpu().numpy()
    sx = _ws_view(ws, lay["sx"], R, torch.float32).cpu().numpy()
    for r in rows:
        i = tok_pos[int(perm[r] // topk)]
        assert np.array_equal(qx[r], qx_o[i]) and sx[r] == sx_o[i]

    h = _ws_view(ws, lay["h"], R, torch.int16, I).cpu().numpy().view(np.uint16)
    qh = _ws_view(ws, lay["qh"], R, torch.int8, I).cpu().numpy()
    sh = _ws_view(ws, lay["sh"], R, torch.float32).cpu().numpy()
    yd = _ws_view(ws, lay["yd"], R, torch.int16, H).cpu().numpy().view(np.uint16)
    n_fallback = 0
    for e in np.unique(expert_of_row):
        sel = expert_of_row == e
        rs = rows[sel]
        c1, s1, z1 = layer.codes(int(e), 0)
        c2, s2, z2 = layer.codes(int(e), 1)
        # gate_up partials, bit for bit
        if P1 is not None:
            Po1 = O.partials(qx[rs], c1, z1, g)
            Pg1 = P1[slot_of_row[sel]]
            assert np.array_equal(Pg1, Po1), f"gate_up partials: {int((Pg1 != Po1).sum())} differ (expert {e})"
        # gate_up, then h = silu(gate) * up
        Hx, Ha, _ = O.expert_linear_rows(qx[rs], sx[rs], c1, s1, z1, g)
        h_exact = O.silu_mul(Hx)
        gt, up = Hx[:, :I], Hx[:, I:]
        sig = 1.0 / (1.0 + np.exp(-gt))
        hx = gt * sig * up
        dsilu = np.abs(sig * (1 + gt * (1 - sig)))
        bound = (dsilu * 1e-5 * Ha[:, :I] * np.abs(up) + np.abs(gt * sig) * 1e-5 * Ha[:, I:]
                 + 0.5 * bf16_ulp(hx) + 1e-30)
        d = np.abs(bf16_ordinal(h[rs]) - bf16_ordinal(h_exact))
        hv = O.bf16_to_f32(h[rs]).astype(np.float64)
        ok = (d <= 1) | (np.abs(hv - hx) <= bound)
        assert ok.all(), f"h: {int((~ok).sum())} elements out of tolerance (expert {e})"
        record_fallback(f"h (expert {e})", int(((d > 1) & ok).sum()), d.size)
        # quantization of the GPU's h
        qh_o, sh_o, _, _ = O.quant_act(np.ascontiguousarray(h[rs]))
        assert np.array_equal(qh[rs], qh_o) and np.array_equal(sh[rs], sh_o)
        # down partials, bit for bit, then the bf16 expert rows
        if P2 is not None:
            Po2 = O.partials(qh[rs], c2, z2, g)
            Pg2 = P2[slot_of_row[sel]]
            assert np.array_equal(Pg2, Po2), f"down partials: {int((Pg2 != Po2).sum())} differ (expert {e})"
        Yx, Ya, _ = O.expert_linear_rows(qh[rs], sh[rs], c2, s2, z2, g)
        n_fallback += check_bf16(yd[rs], Yx, Ya, what=f"expert {e} down output")

    # combine of the GPU's expert outputs with the GPU's weights
    out = bits(res["out"])[tokens]
    inv_t = inv.reshape(T, topk)[tokens]
    y = O.bf16_to_f32(yd).astype(np.float64)
    acc = np.zeros((len(tokens), H))
    aabs = np.zeros((len(tokens), H))
    for j in range(topk):
        term = p[tokens, j][:, None] * y[inv_t[:, j]]
        acc += term
        aabs += np.abs(term)
    check_bf16(out, acc, aabs, what="combine")
    return n_fallback, tokens


def end_to_end_rms(layer, inp, topk, res, tokens):
    """Relative RMS of the GPU output against the all-binary64 oracle."""
    T = inp.X.shape[0]
    idx_o, p_o, _ = O.route(inp.logits.numpy(), topk)
    qx, sx, _, _ = O.quant_act(bits(inp.X)[tokens])
    ref = np.zeros((len(tokens), layer.H))
    for i, t in enumerate(tokens):
        for j in range(topk):
            e = int(idx_o[t, j])
            Hx, _, _ = O.expert_linear_rows(qx[i:i + 1], sx[i:i + 1], *layer.codes(e, 0), layer.group)
            hh = O.silu_mul(Hx)
            qh, sh, _, _ = O.quant_act(hh)
            Yx, _, _ = O.expert_linear_rows(qh, sh, *layer.codes(e, 1), layer.group)
            ref[i] += p_o[t, j] * O.bf16_to_f32(O.f64_to_bf16(Yx[0])).astype(np.float64)
    got = O.bf16_to_f32(bits(res["out"])[tokens]).astype(np.float64)
    return float(np.sqrt(np.mean((got - ref) ** 2)) / np.sqrt(np.mean(ref ** 2)))


SMALL = [
    # (T, H, E, topk, I, group, sym, zipf)
    (50, 256, 8, 2, 192, 64, False, None),
    (64, 512, 16, 4, 128, 128, True, None),
    (33, 128, 4, 4, 64, 64, True, 1.1),     # topk == E: every token visits every expert
    (200, 256, 64, 6, 128, 128, True, 1.1),  # many experts with 0 tokens
    (1, 256, 8, 2, 128, 64, False, None),    # a single token
    (40, 128, 512, 16, 64, 64, True, 1.1),   # the largest E and top-k the dispatch supports
]


@pytest.mark.parametrize("T,H,E,topk,I,g,sym,zipf", SMALL)
def test_moe_small_stagewise(m, T, H, E, topk, I, g, sym, zipf):
    layer = Layer(m, seed=T + E, E=E, H=H, I=I, group=g, sym=sym, w_outlier_p=0.001)
    inp = gen_moe_activations(T, H, E, seed=T * 3 + E, zipf=zipf)
    res = run_layer(m, layer, inp, topk, tokens=np.arange(T))
    _, tokens = check_layer(m, layer, inp, topk, res)
    assert end_to_end_rms(layer, inp, topk, res, tokens[:16]) <= 1e-2


def test_moe_one_expert_takes_every_token(m):
    T, H, E, topk, I = 300, 256, 8, 1, 128
    layer = Layer(m, seed=5, E=E, H=H, I=I, group=128, sym=True, w_outlier_p=0.0)
    inp = gen_moe_activations(T, H, E, seed=5)
    inp.logits[:, 3] += 100.0
    res = run_layer(m, layer, inp, topk, tokens=np.arange(T))
    offs = res["expert_offsets"].cpu().numpy()
    assert offs[3] == 0 and offs[4] == T
    check_layer(m, layer, inp, topk, res)


def test_moe_flags_nonfinite_logits(m):
    T, H, E, topk, I = 8, 128, 4, 2, 64
    layer = Layer(m, seed=6, E=E, H=H, I=I, group=64, sym=True, w_outlier_p=0.0)
    inp = gen_moe_activations(T, H, E, seed=6)
    inp.logits[2, 1] = float("nan")
    st = m.new_status("cuda")
    m.w4a8_moe_grouped_gemm(inp.X.cuda(), inp.logits.cuda(), topk, layer.w1, layer.w2, status=st)
    assert m.w4a8_get_device_status(st) == 4


def test_moe_symmetric_config_sampled(m):
    # T=4096, hidden 2048, 64 experts, top-6, gate_up 2048->2816, down 1408->2048,
    # int4 group 128 symmetric; routing checked for all tokens, the expert
    # path for a seeded sample of tokens.
    T, H, E, topk, I = 4096, 2048, 64, 6, 1408
    layer = Layer(m, seed=0, E=E, H=H, I=I, group=128, sym=True, w_outlier_p=0.0)
    inp = gen_moe_activations(T, H, E, seed=0, zipf=None)
    tokens = sample_tokens(T, 12, 0, extra=[0, T - 1])
    res = run_layer(m, layer, inp, topk, tokens=tokens)
    _, tokens = check_layer(m, layer, inp, topk, res, tokens=tokens)
    assert end_to_end_rms(layer, inp, topk, res, tokens[:4]) <= 1e-2


def test_moe_asym_decode_config(m):
    # T=64, hidden 7168, 256 experts, top-8 with Zipf(1.1) logits, I=2048,
    # asymmetric uint4 + zero-point, group 64, 0.1% weight outliers x20.
    T, H, E, topk, I = 64, 7168, 256, 8, 2048
    layer = Layer(m, seed=0, E=E, H=H, I=I, group=64, sym=False, w_outlier_p=0.001)
    inp = gen_moe_activations(T, H, E, seed=0, zipf=1.1)
    tokens = sample_tokens(T, 3, 1)
    res = run_layer(m, layer, inp, topk, tokens=tokens)
    check_layer(m, layer, inp, topk, res, tokens=tokens)


@pytest.mark.parametrize("T,H,E,topk,I,g,sym,zipf", [
    (3000, 128, 256, 8, 64, 64, False, 1.1),   # dispatch over 12 CTAs, skewed experts
    (270000, 64, 16, 1, 64, 64, True, None),   # 528 CTAs of 512 tokens each
])
def test_moe_dispatch_many_tokens(m, T, H, E, topk, I, g, sym, zipf):
    """Many tokens: the dispatch runs over several CTAs (count, scan, scatter);
    offsets, permutation and inverse must equal the oracle's for every token,
    and the expert path is checked on a sample."""
    layer = Layer(m, seed=T % 1000 + E, E=E, H=H, I=I, group=g, sym=sym, w_outlier_p=0.001)
    inp = gen_moe_activations(T, H, E, seed=5, zipf=zipf)
    tokens = sample_tokens(T, 16, 1, extra=[0, T - 1])
    res = run_layer(m, layer, inp, topk, tokens=tokens)
    check_layer(m, layer, inp, topk, res, tokens=tokens)


def test_moe_asym_prefill_config(m):
    """The asymmetric prefill configuration at full size: T=8192, hidden 7168,
    256 experts, top-8 with Zipf(1.1) logits, I=2048, uint4 + zero-point,
    group 64 (112 groups per gate_up tile, BN=128), 0.1% weight outliers x20.
    Routing and dispatch are checked for every token; quantized X, the int32
    partials of both grouped GEMMs, h, q_h and the expert rows for a seeded
    sample of tokens; the combine for those tokens."""
    T, H, E, topk, I = 8192, 7168, 256, 8, 2048
    layer = Layer(m, seed=0, E=E, H=H, I=I, group=64, sym=False, w_outlier_p=0.001)
    inp = gen_moe_activations(T, H, E, seed=0, zipf=1.1)
    tokens = sample_tokens(T, 10, 2, extra=[0, 4095, T - 1])
    res = run_layer(m, layer, inp, topk, tokens=tokens)
    check_layer(m, layer, inp, topk, res, tokens=tokens)


@pytest.mark.parametrize("T,H,E,topk,I,g,sym,zipf", [(200, 256, 16, 4, 128, 128, True, 1.1),
                                                      (64, 512, 8, 2, 192, 64, False, None)])
def test_moe_building_blocks_equal_layer(m, T, H, E, topk, I, g, sym, zipf):
    """Routing, pre-routed experts and combine run as separate calls (the
    expert-parallel layer with one rank) give w4a8_moe_grouped_gemm's result
    bit for bit."""
    from moe_linear_layers_w4a8_b200.ep import ExpertParallelMoE
    layer = Layer(m, seed=T + E, E=E, H=H, I=I, group=g, sym=sym, w_outlier_p=0.001)
    inp = gen_moe_activations(T, H, E, seed=T * 5 + E, zipf=zipf)
    X, L = inp.X.cuda(), inp.logits.cuda()
    res = run_layer(m, layer, inp, topk)
    ep = ExpertParallelMoE(E, layer.w1, layer.w2)
    out, idx, w = ep.forward(X, L, topk)
    torch.cuda.synchronize()
    assert torch.equal(idx, res["topk_idx"])
    assert torch.equal(w, res["topk_w"])
    assert np.array_equal(bits(out), bits(res["out"]))


def test_moe_experts_rejects_out_of_range_ids(m):
    T, H, E, I = 16, 128, 4, 64
    layer = Layer(m, seed=3, E=E, H=H, I=I, group=64, sym=True, w_outlier_p=0.0)
    X = gen_moe_activations(T, H, E, seed=3).X.cuda()
    ids = torch.full((T,), 1, dtype=torch.int32, device="cuda")
    ids[5] = E + 3
    st = m.new_status("cuda")
    m.w4a8_moe_experts(X, ids, layer.w1, layer.w2, status=st)
    assert m.w4a8_get_device_status(st) == 1
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0  # the context is still usable
