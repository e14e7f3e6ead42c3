"""Token-sharded stack forward: G ranks, each owning T / G consecutive tokens
(their rows of every sample and their per-token FFN weights); the token
mixing becomes an all-to-all between the ranks ("特征交叉 —— RankMixer 精读笔记"
draws the analogy; "重新理解 RankMixer" section 3.3 discusses model sharding).

Every step of the path runs in the library's kernels through the C ABI
(rm_tokshard_pack, rm_tokshard_mix_ln, rm_pffn_forward, rm_tokshard_pool);
this module allocates the buffers, slices the rank's weights and performs the
two exchanges: an equal-split all-to-all of the packed rows per block and a
mean of the ranks' pooled parts at the end.  A rank's forward is a generator
that yields at each exchange, so the same code runs

  * one rank per GPU (`run_distributed`, torch.distributed: NCCL all-to-all
    and all-reduce over NVLink), or
  * G ranks in one process on one device (`run_local`), the exchanges done by
    device copies between the ranks' buffers (no kernel waits for another).
"""
from __future__ import annotations

from typing import Dict, Iterator, List, Sequence, Tuple

import torch

from . import rankmixer as rm
from .synth import Workload


class TokenShardedRank:
    """One rank's share of a dense bf16 stack (blocks: the full weights)."""

    def __init__(self, wl: Workload, blocks: Sequence[Dict[str, torch.Tensor]], rank: int, world: int,
                 device="cuda"):
        if wl.n_experts or wl.dtype != "bf16" or not wl.mix_addnorm or wl.T % world:
            raise ValueError("token sharding covers dense bf16 stacks with the Add & Norm, T % world == 0")
        self.wl, self.rank, self.world = wl, rank, world
        self.Tl = wl.T // world
        t0, t1 = rank * self.Tl, (rank + 1) * self.Tl
        self.h = rm.rm_create(wl.B, self.Tl, wl.D, wl.hidden, wl.L, n_experts=0, dtype="bf16", act=wl.act,
                              mix_addnorm=True)
        self.blocks = []
        for blk in blocks:
            b = {k: v.to(device) for k, v in blk.items() if k.startswith("ln")}
            for k in ("W1", "b1", "W2", "b2"):   # the rank's tokens: leading dimension T
                b[k] = blk[k][t0:t1].contiguous().to(device)
            self.blocks.append(b)
        B, D = wl.B, wl.D
        act = dict(dtype=torch.bfloat16, device=device)
        self.Xh = torch.empty(B, self.Tl, D, **act)
        self.send = torch.empty(B * self.Tl * D, **act)
        self.recv = torch.empty(B * self.Tl * D, **act)
        self.S = torch.empty(B, self.Tl, D, **act)
        self.V = torch.empty(B, self.Tl, D, **act)
        self.pooled = torch.empty(B, D, dtype=torch.float32, device=device)

    def close(self) -> None:
        if self.h is not None:
            self.h.close()
            self.h = None

    def forward_steps(self, X0_local: torch.Tensor, B: int) -> Iterator[Tuple]:
        """The rank's forward on its rows X0_local [B, Tl, D]; yields
        ("a2a", send, recv) and ("mean", pooled) exchange requests; when it
        returns, self.pooled holds the pooled output [B, D]."""
        h, W = self.h, self.world
        for l, blk in enumerate(self.blocks):
            if l == 0:
                rm.rm_tokshard_pack(h, X0_local, None, None, None, self.Xh, self.send, B, W)
            else:
                prev = self.blocks[l - 1]
                rm.rm_tokshard_pack(h, self.V, self.S, prev["ln2_g"], prev["ln2_b"], self.Xh, self.send, B, W)
            yield ("a2a", self.send, self.recv)
            rm.rm_tokshard_mix_ln(h, self.recv, self.Xh, blk["ln1_g"], blk["ln1_b"], self.S, B, W)
            rm.rm_pffn_forward(h, blk, self.S, self.V, B)
        last = self.blocks[-1]
        rm.rm_tokshard_pool(h, self.V, self.S, last["ln2_g"], last["ln2_b"], self.pooled, B)
        yield ("mean", self.pooled)


def shard_rows(X0: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """The rank's token rows [B, T / world, D] of a full input [B, T, D]."""
    Tl = X0.shape[1] // world
    return X0[:, rank * Tl:(rank + 1) * Tl].contiguous()


def run_local(ranks: List[TokenShardedRank], X0_locals: List[torch.Tensor], B: int) -> torch.Tensor:
    """All ranks in this process (one device): the exchanges are device copies."""
    gens = [r.forward_steps(x, B) for r, x in zip(ranks, X0_locals)]
    reqs = [next(g) for g in gens]
    W = len(ranks)
    while True:
        kind = reqs[0][0]
        if kind == "a2a":
            n = reqs[0][1].numel() // W
            for r in range(W):
                for q in range(W):   # recv of rank r, block q  <-  send of rank q, block r
                    reqs[r][2][q * n:(q + 1) * n].copy_(reqs[q][1][r * n:(r + 1) * n])
        elif kind == "mean":
            mean = torch.stack([req[1] for req in reqs]).sum(0) / W
            for req in reqs:
                req[1].copy_(mean)
        nxt = []
        for g in gens:
            try:
                nxt.append(next(g))
            except StopIteration:
                return ranks[0].pooled
        reqs = nxt


def run_distributed(rank_obj: TokenShardedRank, X0_local: torch.Tensor, B: int, group=None) -> torch.Tensor:
    """This process's rank under torch.distributed (NCCL on GPUs)."""
    import torch.distributed as dist
    for req in rank_obj.forward_steps(X0_local, B):
        if req[0] == "a2a":
            exchange(req[1], req[2], group)
        else:
            dist.all_reduce(req[1], group=group)
            req[1].div_(dist.get_world_size(group))
    return rank_obj.pooled


def exchange(send: torch.Tensor, recv: torch.Tensor, group=None) -> None:
    """Equal-split all-to-all: block q of recv <- block r of rank q's send."""
    import torch.distributed as dist
    dist.all_to_all_single(recv, send, group=group)
