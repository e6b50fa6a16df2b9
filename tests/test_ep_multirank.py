"""Expert-parallel MoE (moe_linear_layers_w4a8_b200.ep): the token exchange
between ranks, checked on CPU with two gloo ranks.  Each rank owns half of
the experts and its own tokens; the per-rank compute steps are the oracle's
(route, one expert per row, combine), passed in as the layer's callables, so
the test isolates what the exchange must get right: every (token, slot) row
reaches its expert's rank and its result comes back to the right place.  The
result must equal the one-process oracle layer bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

E, H, I, TOPK, GROUP = 8, 128, 64, 2, 64


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _codes(sym):
    import oracle as O
    from synth import gen_expert_weight
    w1, w2 = [], []
    for e in range(E):
        W1 = gen_expert_weight(7, e, 0, H, 2 * I, outlier_p=0.01).numpy()
        W2 = gen_expert_weight(7, e, 1, I, H, outlier_p=0.01).numpy()
        if not sym:
            W1, W2 = W1 + 0.01, W2 + 0.01
        c1, s1, z1, _ = O.quant_weights(W1, GROUP, sym)
        c2, s2, z2, _ = O.quant_weights(W2, GROUP, sym)
        w1.append((c1, s1, None if sym else z1))
        w2.append((c2, s2, None if sym else z2))
    return w1, w2


def _oracle_callables(w1, w2, e0):
    import oracle as O

    def route_fn(logits, topk):
        idx, p, _ = O.route(logits.numpy(), topk)
        return torch.from_numpy(idx), torch.from_numpy(p)

    def experts_fn(rows, ids):
        x = rows.numpy().view(np.uint16)
        ids = ids.numpy()
        out = np.zeros_like(x)
        if len(x) == 0:
            return torch.from_numpy(out.view(np.int16))
        q, s, _, _ = O.quant_act(x)
        for el in np.unique(ids):
            sel = np.nonzero(ids == el)[0]
            e = e0 + int(el)
            Hx, _, _ = O.expert_linear_rows(q[sel], s[sel], *w1[e], GROUP)
            h = O.silu_mul(Hx)
            qh, sh, _, _ = O.quant_act(h)
            Yx, _, _ = O.expert_linear_rows(qh, sh, *w2[e], GROUP)
            out[sel] = O.f64_to_bf16(Yx)
        return torch.from_numpy(out.view(np.int16))

    def combine_fn(rows, p):
        T, k = p.shape
        o, _ = O.combine(rows.numpy().view(np.uint16), p.numpy(), np.arange(T * k, dtype=np.int32))
        return torch.from_numpy(o.view(np.int16))
    return route_fn, experts_fn, combine_fn


def _rank_main(rank, world, port, sym, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import oracle as O
        from moe_linear_layers_w4a8_b200.ep import ExpertParallelMoE
        from synth import gen_moe_activations
        w1, w2 = _codes(sym)
        e_local = E // world
        fns = _oracle_callables(w1, w2, rank * e_local)
        layer = ExpertParallelMoE(E, route_fn=fns[0], experts_fn=fns[1], combine_fn=fns[2])
        T = 24 + 9 * rank  # ranks hold different numbers of tokens
        inp = gen_moe_activations(T, H, E, seed=100 + rank, zipf=1.1)
        Xb = inp.X.view(torch.int16)
        got, idx, _ = layer.forward(Xb.view(torch.bfloat16), inp.logits, TOPK)
        ref = O.moe_forward(Xb.numpy().view(np.uint16), inp.logits.numpy(), TOPK, w1, w2, GROUP)
        out[rank] = (bool(np.array_equal(got.numpy().view(np.uint16), ref["out"])),
                     bool(np.array_equal(idx.numpy(), ref["idx"])),
                     int((idx.numpy() // e_local != rank).sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,sym", [(2, True), (2, False), (4, True)])
def test_ranks_equal_one_process_layer(world, sym):
    """2 and 4 ranks (4 experts / 2 experts per rank): every rank's output
    equals the one-process layer on its tokens, and rows really travel."""
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, sym, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    for r in range(world):
        same_out, same_idx, remote_pairs = res[r]
        assert same_idx
        assert remote_pairs > 0  # some rows really travelled to the other rank
        assert same_out


def test_plan_groups_pairs_by_owner_in_token_order():
    from moe_linear_layers_w4a8_b200.ep import ExpertParallelMoE
    layer = ExpertParallelMoE.__new__(ExpertParallelMoE)
    layer.world, layer.E_local = 4, 2
    idx = torch.tensor([[7, 0], [2, 3], [0, 6], [5, 1]], dtype=torch.int32)
    order, counts = layer.plan(idx)
    owner = (idx.reshape(-1) // 2)[order]
    assert counts.tolist() == [3, 2, 1, 2]
    assert owner.tolist() == sorted(owner.tolist())
    # inside each owner, pairs keep their (token, slot) order
    for o in range(4):
        pos = order[owner == o].tolist()
        assert pos == sorted(pos)
