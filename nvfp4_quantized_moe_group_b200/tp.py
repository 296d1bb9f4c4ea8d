"""Tensor parallelism: every expert's intermediate dimension split over the ranks of a group.

The quantised checkpoint is validated with four-way tensor parallelism ("NVFP4
quantization", section "Hardware compatibility and serving").  For the MoE layer that means
rank r of G holds, of every expert, the gate and up rows of features [r I/G, (r+1) I/G) and
the matching columns of the down projection, and every rank holds all tokens and the whole
router.  One step:

  1. nvfp4moe_forward_partial on the rank's tokens with its slice of every expert: FP32 sums
     [T][H] of the slice's contributions;
  2. all-reduce (sum) of the FP32 sums;
  3. nvfp4moe_finalize: BF16 rounding.

The slices are cut from the single-GPU quantisation of each whole weight tensor (its codes,
its E4M3 block scales and its global scale), so each rank's operands are exactly the
single-GPU operands of its features: the gate and up rows keep their blocks of 16 along H,
and the down columns split on block boundaries because I/G is a multiple of 128.  Every rank
routes the same tokens with the same kernels, so the ranks agree on every routing decision
and on the input's global scale; the SwiGLU product of a feature depends on that feature's
gate and up rows only, so its requantisation (static scale g_h of the expert, blocks of 16
features) is the single-GPU one; the down projection over the slice's features gives partial
sums whose total equals the single-GPU layer's sums up to the order of the FP32 additions.

Per step and rank: one all-reduce of T H 4 bytes; the expert weights streamed per rank fall
to 1/G of the experts hit.
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist

from . import _lib


def intermediate_range(I: int, rank: int, world: int) -> tuple[int, int]:
    """(first feature, count) of ``rank`` of ``world``: I must split into slices that are
    multiples of 128 features (the library's shape rule for the intermediate size)."""
    if world < 1 or I % (128 * world) != 0:
        raise ValueError(f"an intermediate size of {I} cannot be split into {world} slices of a multiple of 128")
    n = I // world
    return rank * n, n


def slice_expert(gate, up, down, i0: int, n: int):
    """Features [i0, i0 + n) of one quantised expert.  gate, up: (codes [I, H/2], linear scales
    [I, H/16], global scale); down: (codes [H, I/2], linear scales [H, I/16], global scale).
    Returns the same triples for the slice, the global scales unchanged."""
    if i0 % 16 or n % 16:
        raise ValueError("a slice must start and end on a 16-feature block boundary")

    def rows(t):
        return t[0][i0:i0 + n].contiguous(), t[1][i0:i0 + n].contiguous(), t[2]

    dc, ds, dg = down
    return (rows(gate), rows(up),
            (dc[:, i0 // 2:(i0 + n) // 2].contiguous(), ds[:, i0 // 16:(i0 + n) // 16].contiguous(), dg))


class TensorParallelLayer:
    """The layer on one rank of a tensor-parallel group (world 1: the whole layer on one GPU).

    ``partial`` and ``finalize`` default to the library's calls (nvfp4moe_forward_partial
    with this rank's slice of every expert, nvfp4moe_finalize); they can be replaced to
    exercise the logic without a GPU."""

    def __init__(self, cfg: _lib.Cfg, group=None,
                 partial: Callable[[torch.Tensor, torch.Tensor, torch.Tensor | None], torch.Tensor] | None = None,
                 finalize: Callable[[torch.Tensor], torch.Tensor] | None = None):
        self.cfg = cfg
        self.group = group
        initialized = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if initialized else 1
        self.rank = dist.get_rank(group) if initialized else 0
        self.i0, self.n = intermediate_range(cfg.I, self.rank, self.world)
        self.cfg_local = _lib.Cfg(cfg.E, cfg.n_groups, cfg.topk_groups, cfg.topk, cfg.H, self.n, cfg.routed_scale)
        self._partial = partial
        self._finalize = finalize if finalize is not None else (lambda acc: _lib.finalize(acc))
        self.experts: _lib.Experts | None = None
        self._ws: torch.Tensor | None = None

    # ---------------------------------------------------------------- experts ----
    def create_experts(self) -> _lib.Experts:
        """This rank's handle: every expert, with intermediate size I / world."""
        if self.experts is None:
            self.experts = _lib.Experts(self.cfg_local)
        return self.experts

    def set_expert(self, e: int, gate, up, down, g_h: float, stream=None):
        """Expert e from its whole-tensor quantisation (triples as from ``quantize``, linear
        scales, global scales as floats): this rank's slice goes into the handle."""
        sg, su, sd = slice_expert(gate, up, down, self.i0, self.n)
        self.create_experts().set(e, sg, su, sd, g_h, stream=stream)

    def set_expert_from_bf16(self, e: int, gate: torch.Tensor, up: torch.Tensor, down: torch.Tensor, g_h: float,
                             stream=None):
        """Quantise the whole BF16 tensors gate [I, H], up [I, H], down [H, I] (dynamic global
        scales, as the single-GPU layer) and keep this rank's slice; returns the global scales."""
        q = [_lib.quantize(w, stream=stream) for w in (gate, up, down)]
        gs = torch.cat([t[2] for t in q]).cpu().tolist()
        self.set_expert(e, (q[0][0], q[0][1], gs[0]), (q[1][0], q[1][1], gs[1]), (q[2][0], q[2][1], gs[2]), g_h,
                        stream=stream)
        return gs

    def _partial_cuda(self, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None) -> torch.Tensor:
        ex = self.create_experts()
        need = _lib.forward_workspace_bytes(self.cfg_local, x.shape[0])
        if self._ws is None or self._ws.numel() < need or self._ws.device != x.device:
            self._ws = torch.empty(need, dtype=torch.uint8, device=x.device)
        return _lib.forward_partial(ex, x, w_router, bias, ws=self._ws)

    # ---------------------------------------------------------------- forward ----
    def forward(self, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None = None) -> torch.Tensor:
        """x [T, H] BF16, the same tokens on every rank -> out [T, H] BF16 (the same on every rank)."""
        partial = self._partial if self._partial is not None else self._partial_cuda
        acc = partial(x, w_router, bias)
        if self.world > 1:
            dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=self.group)
        return self._finalize(acc)

    def close(self):
        if self.experts is not None:
            self.experts.close()
            self.experts = None
