"""The token-sharded forward's exchange (tokshard.exchange: an equal-split
all-to-all of the packed rows) between two CPU ranks over gloo: block q of a
rank's receive buffer must hold block r of rank q's send buffer, which is the
layout rm_tokshard_pack writes ([dest][b][tq][D / G]) and rm_tokshard_mix_ln
reads ([src][b][tq][D / G])."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, B: int, Tl: int, D: int, q):
    import torch.distributed as dist
    from token_mixing_feature_b200 import tokshard
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    seg = D // world
    # send[dest][b][tq][c] = a value naming (src rank, dest, b, tq, c)
    idx = torch.arange(world * B * Tl * seg, dtype=torch.float32).reshape(world, B, Tl, seg)
    send = (idx + 1e6 * rank).reshape(-1)
    recv = torch.empty_like(send)
    tokshard.exchange(send, recv)
    got = recv.reshape(world, B, Tl, seg)
    ok = True
    for src in range(world):
        expect = (idx[rank] + 1e6 * src)
        ok = ok and torch.equal(got[src], expect)
    q.put((rank, ok))
    dist.destroy_process_group()


def test_exchange_layout_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, 3, 2, 64, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res == {0: True, 1: True}
