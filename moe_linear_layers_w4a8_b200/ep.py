"""Expert-parallel MoE layer over a torch.distributed process group.

"Kimi 2.7 MoE W4A8 deployment in practice" §5.4 scales the MoE layer by
spreading the experts over GPUs and exchanging tokens between them.  Here
rank r of a group of P ranks holds experts [r*E/P, (r+1)*E/P) (packed as for
w4a8_moe_grouped_gemm) and its own tokens; one forward pass is

  1. route the rank's tokens (w4a8_moe_route);
  2. order the (token, slot) pairs by the rank that owns their expert and
     exchange the activation rows and local expert ids (all-to-all);
  3. run the received rows through the local experts (w4a8_moe_experts:
     dispatch, quantization, gate_up + SiLU*up, quantization of h, down);
  4. send every expert output row back to its token's rank (all-to-all, the
     reverse split);
  5. combine in (token, slot) order (w4a8_moe_combine).

Every row is computed by the same kernels with the same arithmetic as in the
one-GPU layer, and the combine adds the same values in the same order, so the
result equals w4a8_moe_grouped_gemm's bit for bit.  The exchanges are plain
NCCL all-to-alls (bf16 rows travel as raw bit patterns); nothing reads
another GPU's memory directly.  With one rank (or no process group) the
exchanges are skipped.

The three compute steps are the library's by default; a caller may pass other
callables with the same contracts (route_fn(logits, topk) -> (idx [T,k] int32,
weights [T,k]); experts_fn(rows int16 [R,H], ids int32 [R]) -> rows int16
[R,H]; combine_fn(rows int16 [T*k,H], weights) -> out), which is how the
exchange itself is tested on CPU ranks.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch


def _a2a(t: torch.Tensor, out_splits, in_splits, group) -> torch.Tensor:
    """all_to_all_single along dim 0 with the given split sizes.  16-bit rows
    travel as int32 pairs (every backend moves int32; the bits are kept)."""
    import torch.distributed as dist
    src = t.contiguous()
    if src.element_size() == 2:
        src = src.view(torch.int32)
    out = torch.empty((sum(out_splits),) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    dist.all_to_all_single(out, src, output_split_sizes=list(out_splits), input_split_sizes=list(in_splits),
                           group=group)
    return out.view(t.dtype) if t.element_size() == 2 else out


class ExpertParallelMoE:
    """One MoE layer whose experts are spread over the ranks of `group`."""

    def __init__(self, num_experts: int, w1_local=None, w2_local=None, group=None,
                 route_fn: Optional[Callable] = None, experts_fn: Optional[Callable] = None,
                 combine_fn: Optional[Callable] = None):
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group) if (dist.is_available() and dist.is_initialized()) else 1
        self.rank = dist.get_rank(group) if self.world > 1 else 0
        if num_experts % self.world != 0:
            raise ValueError("the number of experts must be a multiple of the number of ranks")
        self.E = num_experts
        self.E_local = num_experts // self.world
        self.w1, self.w2 = w1_local, w2_local
        if route_fn is None or experts_fn is None or combine_fn is None:
            import moe_linear_layers_w4a8_b200 as m
            if w1_local is None or w2_local is None or w1_local.experts != self.E_local:
                raise ValueError("w1_local / w2_local must stack this rank's E / world experts")

            def _route(logits, topk):
                return m.w4a8_moe_route(logits, topk)

            def _experts(rows, ids):
                x = rows.view(torch.bfloat16)
                return m.w4a8_moe_experts(x, ids, self.w1, self.w2).view(torch.int16)

            def _combine(rows, weights):
                return m.w4a8_moe_combine(rows.view(torch.bfloat16), weights)
            route_fn = route_fn or _route
            experts_fn = experts_fn or _experts
            combine_fn = combine_fn or _combine
        self.route_fn, self.experts_fn, self.combine_fn = route_fn, experts_fn, combine_fn

    def plan(self, idx: torch.Tensor):
        """Send order and counts of the (token, slot) pairs: pairs grouped by
        the rank that owns their expert, (token, slot) order inside a group."""
        owner = (idx.to(torch.int64) // self.E_local).reshape(-1)
        order = torch.argsort(owner, stable=True)
        counts = torch.bincount(owner, minlength=self.world)
        return order, counts

    def forward(self, X: torch.Tensor, logits: torch.Tensor, topk: int):
        """X bf16 [T, H] and logits [T, E] of this rank's tokens -> (out [T, H],
        topk_idx, topk_w)."""
        T, H = X.shape
        idx, w = self.route_fn(logits, topk)
        order, send_counts = self.plan(idx)
        tok = order // topk
        rows = X.view(torch.int16)[tok]                       # [T*k, H] bf16 bits
        eids = (idx.reshape(-1).to(torch.int64)[order] % self.E_local).to(torch.int32)
        if self.world > 1:
            sc = send_counts.to(X.device if X.is_cuda else "cpu")
            rc = torch.empty_like(sc)
            import torch.distributed as dist
            dist.all_to_all_single(rc, sc, group=self.group)
            send_l, recv_l = sc.tolist(), rc.tolist()
            rows_in = _a2a(rows, recv_l, send_l, self.group)
            eids_in = _a2a(eids, recv_l, send_l, self.group)
            y_in = self.experts_fn(rows_in, eids_in)
            y_back = _a2a(y_in, send_l, recv_l, self.group)
        else:
            y_back = self.experts_fn(rows, eids)
        y_rows = torch.empty_like(y_back)
        y_rows[order] = y_back                                 # back to (token, slot) order
        out = self.combine_fn(y_rows, w)
        return out, idx, w
