"""Token Parallel forward of a TokenMixer-Large stack over P ranks.

TokenMixer-Large digest, section 2.5.3 ("Token Parallel"): instead of holding every per-token
weight on every GPU, the per-token parameters are split across the GPUs and the activations are
exchanged at the Mix / Revert boundary of each block.  Here rank p holds

  * the mixing banks of its H/P heads (heads p*H/P .. (p+1)*H/P - 1; their columns of the token
    tensor are D/P consecutive columns, since a head owns dh = D/H consecutive columns),
  * the reverting banks of its T/P tokens (tokens p*T/P .. (p+1)*T/P - 1),
  * the activations of its T/P tokens for all B samples, x_p [B, T/P, D].

One block then runs as

  1. token -> head exchange (all-to-all): rank p receives from every rank q the columns of p's heads
     of q's tokens, and so holds G_p = X[:, :, columns of p's heads], a [B, T, D/P] token tensor;
  2. the mixing sub-layer on G_p through the Mix layout with H/P heads: its rows are exactly the
     mixed rows (b, h) of p's heads, and its output, written through Revert, is
     R_p = X_revert[:, :, columns of p's heads];
  3. head -> token exchange: rank p receives from every rank q the rows of p's tokens of q's head
     columns, i.e. X_revert[:, tokens of p, :];
  4. the reverting sub-layer on p's tokens (row layout, T/P banks), with the block input x_p as the
     residual and, where the stack's rule applies, X_{l-gap} of p's tokens as the inter-residual.

Two exchanges per block, each moving (P-1)/P of B * T/P * D elements per rank in each direction.
Every row is computed by the same kernels on the same data as in the unsharded stack, and the
library's per-row results do not depend on the batch or bank composition around a row, so the
sharded stack gives the same bits as tm_stack_forward.

The exchange is a callable send [P, ...] -> recv [P, ...] (chunk q of send goes to rank q; chunk q
of recv came from rank q): torch.distributed's all_to_all_single between processes, or a local
transpose of all ranks' chunks when every shard lives in one process.  The packing of a rank's
tensors into the exchange layout and back is the library's tm_tp_exchange_layout (a permutation
kernel); `layouts` may stand in another implementation of the same four maps (the CPU tests pass
a host one, since their ranks compute on the CPU).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence

import torch

from . import _abi as A
from . import api


@dataclass(frozen=True)
class ShardPlan:
    """Heads and tokens of each of P ranks (H and T must be multiples of P)."""
    T: int
    D: int
    H: int
    P: int

    def __post_init__(self):
        if self.P < 1 or self.T % self.P or self.H % self.P or self.D % self.H:
            raise ValueError(f"Token Parallel needs T ({self.T}) and H ({self.H}) divisible by P ({self.P}) "
                             f"and D ({self.D}) by H")

    @property
    def Tp(self) -> int:
        return self.T // self.P

    @property
    def Hp(self) -> int:
        return self.H // self.P

    @property
    def Dp(self) -> int:
        return self.D // self.P

    def heads(self, rank: int):
        return rank * self.Hp, (rank + 1) * self.Hp

    def tokens(self, rank: int):
        return rank * self.Tp, (rank + 1) * self.Tp


# ------------------------------------------------------------------ exchange layout
def _tp_layout(src: torch.Tensor, dst: torch.Tensor, plan: "ShardPlan", B: int, local_layout: int,
               to_exchange: bool) -> torch.Tensor:
    dt = A.TM_BF16 if src.dtype == torch.bfloat16 else A.TM_F32
    A.check(api.lib().tm_tp_exchange_layout(api._p(src), api._p(dst), plan.P, B, plan.Tp, plan.Dp, dt, local_layout,
                                            1 if to_exchange else 0, api._s(torch.cuda.current_stream())),
            "tm_tp_exchange_layout")
    return dst


class LibraryLayouts:
    """The four packing maps of the two exchanges, on the device (tm_tp_exchange_layout)."""

    @staticmethod
    def pack_for_heads(plan: "ShardPlan", x_local: torch.Tensor) -> torch.Tensor:
        """x_p [B, T/P, D] -> send [P, B, T/P, D/P]: chunk q = the columns of rank q's heads."""
        B = x_local.shape[0]
        out = torch.empty((plan.P, B, plan.Tp, plan.Dp), dtype=x_local.dtype, device=x_local.device)
        return _tp_layout(x_local.contiguous(), out, plan, B, A.TM_TP_TOKEN_SHARD, True)

    @staticmethod
    def unpack_heads(plan: "ShardPlan", recv: torch.Tensor) -> torch.Tensor:
        """recv [P, B, T/P, D/P] (chunk q: q's tokens) -> G_p [B, T, D/P] in token order."""
        B = recv.shape[1]
        out = torch.empty((B, plan.T, plan.Dp), dtype=recv.dtype, device=recv.device)
        return _tp_layout(recv.contiguous(), out, plan, B, A.TM_TP_HEAD_SHARD, False)

    @staticmethod
    def pack_for_tokens(plan: "ShardPlan", r_local: torch.Tensor) -> torch.Tensor:
        """R_p [B, T, D/P] -> send [P, B, T/P, D/P]: chunk q = rank q's tokens."""
        B = r_local.shape[0]
        out = torch.empty((plan.P, B, plan.Tp, plan.Dp), dtype=r_local.dtype, device=r_local.device)
        return _tp_layout(r_local.contiguous(), out, plan, B, A.TM_TP_HEAD_SHARD, True)

    @staticmethod
    def unpack_tokens(plan: "ShardPlan", recv: torch.Tensor) -> torch.Tensor:
        """recv [P, B, T/P, D/P] (chunk q: the columns of q's heads) -> X_revert of p's tokens [B, T/P, D]."""
        B = recv.shape[1]
        out = torch.empty((B, plan.Tp, plan.D), dtype=recv.dtype, device=recv.device)
        return _tp_layout(recv.contiguous(), out, plan, B, A.TM_TP_TOKEN_SHARD, False)


def skip_index(l: int, L: int, gap: int) -> Optional[int]:
    """Block l (1-based) adds X_{l-gap} when gap > 0, l % gap == 0 and l < L ([digest] 2.3.4)."""
    return l - gap if (gap > 0 and l % gap == 0 and l < L) else None


# ------------------------------------------------------------------ one rank's share
class RankStage:
    """Rank p's banks of every block and its two local computations, on the library's kernels."""

    def __init__(self, blocks: Sequence[api.Block], plan: ShardPlan, rank: int, sh: A.tm_shape, device):
        self.plan = plan
        self.rank = rank
        self.mix = [api.slice_banks(b.mix, *plan.heads(rank)) for b in blocks]
        self.rev = [api.slice_banks(b.rev, *plan.tokens(rank)) for b in blocks]
        # G_p is a [B, T, D/P] token tensor with H/P heads of the original head width; the reverting
        # rows are [B, T/P, D] (row layout: banks and width come from the weights)
        self.sh_mix = A.tm_shape(sh.B, plan.T, plan.Dp, plan.Hp, sh.dtype, sh.eps)
        self.sh_rev = A.tm_shape(sh.B, plan.Tp, plan.D, plan.H, sh.dtype, sh.eps)
        n = max([api.sublayer_workspace_bytes(self.sh_mix, A.TM_LAYOUT_MIXED, s) for s in self.mix] +
                [api.sublayer_workspace_bytes(self.sh_rev, A.TM_LAYOUT_ROWS, s) for s in self.rev])
        self.ws = torch.empty(n, dtype=torch.uint8, device=device)

    @staticmethod
    def _rows(sh: A.tm_shape, B: int) -> A.tm_shape:
        return sh if B == sh.B else A.tm_shape(B, sh.T, sh.D, sh.H, sh.dtype, sh.eps)

    def mixing(self, l: int, G: torch.Tensor) -> torch.Tensor:
        """Mixing sub-layer of block l on p's heads: R_p = Revert(FFN(Norm(Mix(G_p))) + Mix(G_p)) (any
        number of samples up to the stage's B)."""
        return api.sublayer_forward(G, G, None, A.TM_LAYOUT_MIXED, self._rows(self.sh_mix, G.shape[0]), self.mix[l],
                                    workspace=self.ws)

    def reverting(self, l: int, Xr: torch.Tensor, x: torch.Tensor, extra: Optional[torch.Tensor]) -> torch.Tensor:
        """Reverting sub-layer of block l on p's tokens: FFN(Norm(X_rev)) + x (+ inter-residual)."""
        return api.sublayer_forward(Xr, x, extra, A.TM_LAYOUT_ROWS, self._rows(self.sh_rev, Xr.shape[0]), self.rev[l],
                                    workspace=self.ws)


# ------------------------------------------------------------------ drivers
def forward_rank(stage, plan: ShardPlan, x_local: torch.Tensor, L: int, gap: int,
                 exchange: Callable[[torch.Tensor], torch.Tensor], layouts=LibraryLayouts) -> torch.Tensor:
    """The stack on one rank: x_p [B, T/P, D] -> Y_p [B, T/P, D]; exchange(send) -> recv is the
    all-to-all between the ranks (every rank calls this with the same L and gap, so the exchanges
    pair up)."""
    lay = layouts
    hist: List[torch.Tensor] = [x_local]
    for l in range(1, L + 1):
        G = lay.unpack_heads(plan, exchange(lay.pack_for_heads(plan, hist[-1])))
        R = stage.mixing(l - 1, G)
        Xr = lay.unpack_tokens(plan, exchange(lay.pack_for_tokens(plan, R)))
        s = skip_index(l, L, gap)
        hist.append(stage.reverting(l - 1, Xr, hist[-1], hist[s] if s is not None else None))
    return hist[-1]


def forward_rank_overlapped(stage, plan: ShardPlan, x_local: torch.Tensor, L: int, gap: int, exchange_async,
                            chunks: int = 2, layouts=LibraryLayouts) -> torch.Tensor:
    """forward_rank with each block's two exchanges split into sample chunks and overlapped with the
    compute: every chunk's token->head exchange is issued at once; chunk c's mixing sub-layer runs
    as soon as its exchange has landed, while the later chunks' exchanges are in flight, and its
    head->token exchange is issued right after it, in flight while chunk c+1 mixes; the reverting
    sub-layer of chunk c follows its exchange.  exchange_async(send) -> (recv, handle), handle.wait()
    before recv is used (torch_exchange_async: NCCL's own stream beside the compute).  Samples are
    independent, so the result is the bits of forward_rank; every rank issues the same exchanges in
    the same order."""
    lay = layouts
    B = x_local.shape[0]
    n = max(1, min(chunks, B))
    bounds = [B * i // n for i in range(n + 1)]
    spans = [(bounds[i], bounds[i + 1]) for i in range(n) if bounds[i + 1] > bounds[i]]
    hist: List[torch.Tensor] = [x_local]
    for l in range(1, L + 1):
        x = hist[-1]
        first = [exchange_async(lay.pack_for_heads(plan, x[a:b])) for a, b in spans]
        second = []
        for recv, h in first:
            h.wait()
            R = stage.mixing(l - 1, lay.unpack_heads(plan, recv))
            second.append(exchange_async(lay.pack_for_tokens(plan, R)))
        s = skip_index(l, L, gap)
        outs = []
        for (a, b), (recv, h) in zip(spans, second):
            h.wait()
            Xr = lay.unpack_tokens(plan, recv)
            outs.append(stage.reverting(l - 1, Xr, x[a:b], hist[s][a:b] if s is not None else None))
        hist.append(torch.cat(outs, dim=0))
    return hist[-1]


def forward_all_ranks(stages: Sequence, plan: ShardPlan, x_locals: Sequence[torch.Tensor], L: int,
                      gap: int, layouts=LibraryLayouts) -> List[torch.Tensor]:
    """Every rank's share in one process (the exchange becomes a transpose of the ranks' chunks)."""
    P = plan.P
    lay = layouts
    hist = [list(x_locals)]
    for l in range(1, L + 1):
        sends = [lay.pack_for_heads(plan, hist[-1][p]) for p in range(P)]
        G = [lay.unpack_heads(plan, torch.stack([sends[q][p] for q in range(P)])) for p in range(P)]
        R = [stages[p].mixing(l - 1, G[p]) for p in range(P)]
        sends = [lay.pack_for_tokens(plan, R[p]) for p in range(P)]
        Xr = [lay.unpack_tokens(plan, torch.stack([sends[q][p] for q in range(P)])) for p in range(P)]
        s = skip_index(l, L, gap)
        hist.append([stages[p].reverting(l - 1, Xr[p], hist[-1][p], hist[s][p] if s is not None else None)
                     for p in range(P)])
    return hist[-1]


def torch_exchange_async(group=None):
    """The all-to-all of torch.distributed issued asynchronously: send -> (recv, handle)."""
    import torch.distributed as dist

    def ex(send: torch.Tensor):
        recv = torch.empty_like(send)
        return recv, dist.all_to_all_single(recv, send, group=group, async_op=True)
    return ex


def torch_exchange(group=None) -> Callable[[torch.Tensor], torch.Tensor]:
    """The all-to-all of torch.distributed (NCCL between GPUs; gloo on the CPU) as an exchange."""
    import torch.distributed as dist

    def ex(send: torch.Tensor) -> torch.Tensor:
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=group)
        return recv
    return ex
