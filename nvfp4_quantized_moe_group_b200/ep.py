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

With ``exchange="all_to_all"`` (large batches) the pairs travel instead of the tokens:

  1. nvfp4moe_amax of the rank's tokens, all-reduced with a maximum (the global scale of the
     concatenated batch, so every rank quantises as the single-GPU layer would);
  2. nvfp4moe_ep_dispatch: the rank routes and quantises its own tokens and lays out its
     T * topk pairs' quantised rows (2,880 bytes each for Beam) in destination-rank order;
  3. an all-to-all of the per-rank counts, then of the rows, their local expert and weight;
  4. nvfp4moe_ep_experts on the received rows: weighted FP32 output rows;
  5. an all-to-all returns the rows to their tokens' ranks;
  6. nvfp4moe_ep_combine adds each token's topk rows in slot order and rounds to BF16.

Per step and rank that moves T topk (H/2 + H/16 + 8) bytes out and T topk H 4 bytes back,
against G T H 2 gathered and G T H 4 reduce-scattered bytes for the gather exchange, and each
rank routes and quantises T tokens instead of G T.

With ``exchange="peer"`` the gather exchange's reduce-scatter disappears into the down GEMM:
every rank maps the other ranks' FP32 accumulators into its address space once (CUDA
inter-process handles exchanged through the process group), and each step

  1. all-gathers the ranks' BF16 token rows, zeroes its own accumulator, and waits for every
     rank to have done so (a collective on the stream);
  2. nvfp4moe_forward_partial_peer: the rank's experts on all gathered tokens, the down
     GEMM's epilogue adding each weighted row straight into the owning rank's accumulator
     (over NVLink for other ranks' tokens), overlapped with the MMAs;
  3. waits for every rank's additions (a second collective) and rounds its own rows to BF16.
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
                 finalize: Callable[[torch.Tensor], torch.Tensor] | None = None,
                 exchange: str = "gather", a2a_ops: dict | None = None, peer_ops: dict | None = None):
        """``exchange``: "gather" (all-gather the tokens, reduce-scatter FP32 sums), "peer" (the
        same gather, the sums added into the owners' accumulators by the down GEMM) or
        "all_to_all" (send each pair's quantised row to its expert's rank and its weighted
        output row back).  ``a2a_ops`` / ``peer_ops`` replace those paths' library calls (keys
        amax, dispatch, experts, combine / alloc, handle, open, close, partial_peer; the
        signatures of the default methods below), to exercise the exchanges without a GPU.
        The peer exchange maps the accumulators through CUDA inter-process handles, which cover
        memory from cudaMalloc only: torch's caching allocator without expandable segments
        (with them the handle call fails and raises)."""
        if exchange not in ("gather", "all_to_all", "peer"):
            raise ValueError(f"unknown exchange {exchange!r}")
        self.cfg = cfg
        self.group = group
        self.exchange = exchange
        self._a2a = {"amax": self._amax_cuda, "dispatch": self._dispatch_cuda, "experts": self._experts_cuda,
                     "combine": self._combine_cuda}
        self._a2a.update(a2a_ops or {})
        self._p = {"alloc": self._peer_alloc_cuda, "handle": _lib.ipc_handle, "open": _lib.ipc_open,
                   "close": _lib.ipc_close, "partial_peer": self._partial_peer_cuda}
        self._p.update(peer_ops or {})
        self._peer = None
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

    # ------------------------------------------------------ all-to-all library calls ----
    def _amax_cuda(self, x: torch.Tensor) -> torch.Tensor:
        return _lib.amax(x)

    def _dispatch_cuda(self, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None,
                       amax_bits: torch.Tensor) -> dict:
        return _lib.ep_dispatch(self.cfg, self.world, x, w_router, bias, amax_bits)

    def _experts_cuda(self, codes, scales, expert, w, amax_bits) -> torch.Tensor:
        return _lib.ep_experts(self.create_experts(), codes, scales, expert, w, amax_bits)

    def _combine_cuda(self, rows: torch.Tensor, pos: torch.Tensor, T: int) -> torch.Tensor:
        return _lib.ep_combine(rows, pos, T, self.cfg.topk)

    def _all_to_all(self, out: torch.Tensor, inp: torch.Tensor, out_splits: list, in_splits: list):
        if self.world == 1:
            out.copy_(inp)
            return
        dist.all_to_all_single(out, inp, output_split_sizes=out_splits, input_split_sizes=in_splits,
                               group=self.group)

    def forward_all_to_all(self, x: torch.Tensor, w_router: torch.Tensor,
                           bias: torch.Tensor | None = None) -> torch.Tensor:
        """The all-to-all exchange: x [T, H] BF16 (T equal on every rank) -> out [T, H] BF16."""
        T, H = x.shape
        amax_bits = self._a2a["amax"](x)
        if self.world > 1:
            dist.all_reduce(amax_bits, op=dist.ReduceOp.MAX, group=self.group)
        send = self._a2a["dispatch"](x, w_router, bias, amax_bits)
        send_counts = send["rank_counts"]
        recv_counts = torch.empty_like(send_counts)
        self._all_to_all(recv_counts, send_counts, [1] * self.world, [1] * self.world)
        sc = [int(v) for v in send_counts.cpu().tolist()]
        rc = [int(v) for v in recv_counts.cpu().tolist()]
        n = sum(rc)
        recv = {}
        for key in ("codes", "scales", "expert", "w"):
            t = send[key]
            recv[key] = torch.empty((n,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
            self._all_to_all(recv[key], t, rc, sc)
        rows = self._a2a["experts"](recv["codes"], recv["scales"], recv["expert"], recv["w"], amax_bits)
        back = torch.empty((T * self.cfg.topk, rows.shape[1]), dtype=rows.dtype, device=rows.device)
        self._all_to_all(back, rows, sc, rc)
        return self._a2a["combine"](back, send["pos"], T)

    # ----------------------------------------------- combine into the owners' memory ----
    def _peer_alloc_cuda(self, T: int, H: int, device) -> torch.Tensor:
        return torch.zeros((T, H), dtype=torch.float32, device=device)

    def _partial_peer_cuda(self, x_all: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None,
                           table: torch.Tensor, rows_per_peer: int):
        ex = self.create_experts()
        need = _lib.forward_workspace_bytes(self.cfg, x_all.shape[0])
        if self._ws is None or self._ws.numel() < need or self._ws.device != x_all.device:
            self._ws = torch.empty(need, dtype=torch.uint8, device=x_all.device)
        _lib.forward_partial_peer(ex, x_all, w_router, bias, table, rows_per_peer, ws=self._ws)

    def _peer_setup(self, T: int, H: int, device) -> dict:
        """This rank's accumulator [T, H] FP32 and the table of every rank's accumulator address
        in this process (the other ranks' mapped through inter-process handles), made once per
        token count."""
        if self._peer is not None and self._peer["T"] == T:
            return self._peer
        self._peer_close()
        acc = self._p["alloc"](T, H, device)
        addrs, opened = [], []
        if self.world == 1:
            addrs = [acc.data_ptr()]
        else:
            mine = self._p["handle"](acc)
            every = [None] * self.world
            dist.all_gather_object(every, mine, group=self.group)
            for r, (handle, offset) in enumerate(every):
                if r == self.rank:
                    addrs.append(acc.data_ptr())
                else:
                    base = self._p["open"](handle)
                    opened.append(base)
                    addrs.append(base + offset)
        table = torch.tensor(addrs, dtype=torch.int64, device=device)
        self._peer = {"T": T, "acc": acc, "table": table, "opened": opened}
        return self._peer

    def _peer_close(self):
        if self._peer is not None:
            for base in self._peer["opened"]:
                self._p["close"](base)
            self._peer = None

    def _ranks_reached(self, device):
        """Every rank's stream has reached this point (a collective ordered on the stream)."""
        if self.world > 1:
            dist.all_reduce(torch.zeros(1, device=device), group=self.group)

    def forward_peer(self, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None = None) -> torch.Tensor:
        """The gather exchange with the combine in the down GEMM: x [T, H] BF16 (T equal on every
        rank) -> out [T, H] BF16."""
        T, H = x.shape
        p = self._peer_setup(T, H, x.device)
        x_all = self.gather(x)
        p["acc"].zero_()
        self._ranks_reached(x.device)          # every owner's accumulator is zeroed
        self._p["partial_peer"](x_all, w_router, bias, p["table"], T)
        self._ranks_reached(x.device)          # every rank's additions are done
        return self._finalize(p["acc"])

    def forward(self, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None = None) -> torch.Tensor:
        """x [T, H] BF16: this rank's tokens (T equal on every rank) -> out [T, H] BF16."""
        if self.exchange == "all_to_all":
            return self.forward_all_to_all(x, w_router, bias)
        if self.exchange == "peer":
            return self.forward_peer(x, w_router, bias)
        x_all = self.gather(x)
        partial = self._partial if self._partial is not None else self._partial_cuda
        acc = partial(x_all, w_router, bias)
        return self._finalize(self.scatter_sum(acc, x.shape[0]))

    def close(self):
        self._peer_close()
        if self.experts is not None:
            self.experts.close()
            self.experts = None
