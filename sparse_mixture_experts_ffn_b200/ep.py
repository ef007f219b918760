"""Expert parallelism over a process group: one process per GPU, each holding a contiguous
range of the routed experts (``expert_range``), the router and the shared expert.

One forward of G ranks, each with T tokens of its own:
  1. all-gather the tokens, so that every rank holds the group's G*T tokens;
  2. each rank routes all G*T tokens over all E experts and computes the contributions of
     the experts it holds, plus the shared expert on its own T tokens
     (``moe_layer_forward_ep``: fp32 share of the output, G*T rows);
  3. reduce-scatter the shares: rank r receives the sum over the ranks of rows
     [r*T, (r+1)*T), its own tokens' full output;
  4. store it in the working dtype (``moe_layer_sum_partials`` with one part).
Steps 1 and 3 are the collectives (NCCL over NVLink on GPUs); 2 and 4 run in the library's
kernels.  For a decode batch each GPU streams only the touched experts it holds, about 1/G
of the layer's weight bytes.  The source pages mention multi-GPU serving only in passing
(q4km.ai model page, hardware section); this split is the library's.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import expert_range, moe_layer_forward_ep, sum_partials


class ExpertParallelMoE:
    """This rank's part of the layer.  ``W_gate_up`` / ``W_down`` hold the routed experts
    ``expert_range(E, world, rank)`` only (``[n, 2I, H]``, ``[n, H, I]``); ``W_router`` all E.

    ``local_forward(X, expert_begin, shared_rows) -> fp32 [G*T, H]`` and
    ``finish(own fp32 [T, H]) -> y`` default to the library's kernels; they are parameters so
    that the exchange logic can be exercised on CPU process groups."""

    def __init__(self, W_router, W_gate_up, W_down, Ws_gate_up=None, Ws_down=None, *, top_k: int,
                 router_bias=None, group=None, local_forward=None, finish=None, **layer_options):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E = W_router.shape[0]
        self.expert_begin, self.expert_end = expert_range(self.E, self.world, self.rank)
        if W_gate_up.shape[0] != self.expert_end - self.expert_begin:
            raise ValueError(f"rank {self.rank} holds experts [{self.expert_begin}, {self.expert_end}), "
                             f"got {W_gate_up.shape[0]}")
        self.W_router, self.W_gate_up, self.W_down = W_router, W_gate_up, W_down
        self.Ws_gate_up, self.Ws_down = Ws_gate_up, Ws_down
        self.top_k = top_k
        self.router_bias = router_bias
        self.options = layer_options
        self.local_forward = local_forward or self._library_forward
        self.finish = finish or self._library_finish

    def _library_forward(self, X, expert_begin, shared_rows):
        y_part, _ = moe_layer_forward_ep(X, self.W_router, self.W_gate_up, self.W_down, self.Ws_gate_up,
                                         self.Ws_down, top_k=self.top_k, expert_begin=expert_begin,
                                         shared_rows=shared_rows, router_bias=self.router_bias, **self.options)
        return y_part

    @staticmethod
    def _library_finish(own, dtype):
        return sum_partials([own], torch.empty(own.shape, dtype=dtype, device=own.device))

    def forward(self, x):
        """x [T, H]: this rank's tokens (the same T on every rank).  Returns y [T, H] in x's dtype."""
        T, H = x.shape
        G, r = self.world, self.rank
        X = torch.empty((G * T, H), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(X, x.contiguous(), group=self.group)
        part = self.local_forward(X, self.expert_begin, (r * T, (r + 1) * T))
        own = torch.empty((T, H), dtype=part.dtype, device=part.device)
        dist.reduce_scatter_tensor(own, part, op=dist.ReduceOp.SUM, group=self.group)
        return self.finish(own, x.dtype)
