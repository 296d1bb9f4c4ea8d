"""Expert parallelism: the layer spread over the ranks of a torch.distributed process group.

The model's configuration supports expert-parallel layouts in which the experts are placed
on the devices and the rest is replicated, with a device count that divides the 256 experts
("Reflection releases Beam ...", section "Tool calling and multi-node setups").  Here rank r
of G holds experts [r E/G, (r+1) E/G) and the whole router, and one step is:

  1. all-gather of the ranks' BF16 token rows (every rank then holds the same T_all = G T rows);
  2. nvfp4moe_forward_partial on all gathered tokens with the rank's experts: FP32 sums
     [T_all][H] of the contributions of those experts;
  3. reduce-scatter (sum) of the FP32 sums, which leaves each rank the rows of its own tokens;
  4. nvfp4moe_finalize: BF16 rounding.

Every rank routes the same gathered rows with the same kernels, so the ranks agree on every
routing decision and on the input's global scale with no further exchange, and the result
equals the single-GPU layer up to the order of the FP32 additions.  Per GPU the expert
weights streamed at decode fall from the experts hit by its own tokens to its share of the
experts hit by all tokens.  The two collectives are NCCL's (all_gather_into_tensor,
reduce_scatter_tensor); every rank passes the same number of tokens.
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist

from . import _lib


def expert_range(E: int, rank: int, world: int) -> tuple[int, int]:
    """(first expert, count) held by ``rank`` of ``world``; E must be a multiple of world."""
    if world < 1 or E % world != 0:
        raise ValueError(f"{E} experts cannot be split evenly over {world} ranks")
    n = E // world
    return rank * n, n


class ExpertParallelLayer:
    """The layer on one rank of a process group (world 1: the whole layer on one GPU).

    ``partial`` and ``finalize`` default to the library's calls (nvfp4moe_forward_partial on
    this rank's experts, nvfp4moe_finalize); they can be replaced to exercise the exchange
    logic without a GPU."""

    def __init__(self, cfg: _lib.Cfg, group=None,
                 partial: Callable[[torch.Tensor, torch.Tensor, torch.Tensor | None], torch.Tensor] | None = None,
                 finalize: Callable[[torch.Tensor], torch.Tensor] | None = None):
        self.cfg = cfg
        self.group = group
        initialized = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if initialized else 1
        self.rank = dist.get_rank(group) if initialized else 0
        self.e_begin, self.e_count = expert_range(cfg.E, self.rank, self.world)
        self._partial = partial
        self._finalize = finalize if finalize is not None else (lambda acc: _lib.finalize(acc))
        self.experts: _lib.Experts | None = None
        self._ws: torch.Tensor | None = None

    # ---------------------------------------------------------------- experts ----
    def create_experts(self) -> _lib.Experts:
        """This rank's expert handle (experts e_begin .. e_begin + e_count - 1)."""
        if self.experts is None:
            self.experts = _lib.Experts(self.cfg, self.e_begin, self.e_count)
        return self.experts

    def owns(self, e: int) -> bool:
        return self.e_begin <= e < self.e_begin + self.e_count

    def _partial_cuda(self, x_all: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None) -> torch.Tensor:
        ex = self.create_experts()
        need = _lib.forward_workspace_bytes(self.cfg, x_all.shape[0])
        if self._ws is None or self._ws.numel() < need or self._ws.device != x_all.device:
            self._ws = torch.empty(need, dtype=torch.uint8, device=x_all.device)
        return _lib.forward_partial(ex, x_all, w_router, bias, ws=self._ws)

    # ---------------------------------------------------------------- forward ----
    def gather(self, x: torch.Tensor) -> torch.Tensor:
        if self.world == 1:
            return x
        x_all = torch.empty((self.world * x.shape[0], x.shape[1]), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(x_all, x.contiguous(), group=self.group)
        return x_all

    def scatter_sum(self, acc: torch.Tensor, T: int) -> torch.Tensor:
        if self.world == 1:
            return acc
        mine = torch.empty((T, acc.shape[1]), dtype=acc.dtype, device=acc.device)
        dist.reduce_scatter_tensor(mine, acc.contiguous(), op=dist.ReduceOp.SUM, group=self.group)
        return mine

    def forward(self, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None = None) -> torch.Tensor:
        """x [T, H] BF16: this rank's tokens (T equal on every rank) -> out [T, H] BF16."""
        x_all = self.gather(x)
        partial = self._partial if self._partial is not None else self._partial_cuda
        acc = partial(x_all, w_router, bias)
        return self._finalize(self.scatter_sum(acc, x.shape[0]))

    def close(self):
        if self.experts is not None:
            self.experts.close()
            self.experts = None
