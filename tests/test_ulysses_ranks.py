"""Head-sharded (Ulysses) re-sharding on CPU: two gloo ranks, one process
each. Each rank holds a token shard of the same full tensors; after
exchange_heads (of the shard laid out as vdn_pack_head_groups lays it out)
it must hold exactly its heads over every token, in the
library's [B, H/world, L, d] layout, and after z_heads_to_groups exactly its
tokens, with head group g coming from rank g (integers, so the comparison is
exact). One shape is video-only, the other has context tokens after the video
tokens (L = T*N + n_ctx split over the ranks like any other tokens)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SHAPES = [
    dict(B=2, T=3, N=4, n_ctx=0, H=6, w=5),     # 12 video tokens
    dict(B=1, T=5, N=3, n_ctx=7, H=4, w=3),     # 15 video + 7 context tokens
]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from softmax_attention_video_vdn_b200.ulysses import exchange_heads, z_heads_to_groups
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = []
        for sh in SHAPES:
            B, H, w = sh["B"], sh["H"], sh["w"]
            L = sh["T"] * sh["N"] + sh["n_ctx"]
            Ls, Hs = L // world, H // world
            full = torch.arange(B * L * H * w, dtype=torch.float32).reshape(B, L, H, w)
            shard = full[:, rank * Ls:(rank + 1) * Ls]
            # the layout of vdn_pack_head_groups: [b, h, g] = head g*Hs + h
            send = shard.reshape(B, Ls, world, Hs, w).permute(0, 3, 2, 1, 4).contiguous()
            mine = exchange_heads(send)
            # the asynchronous form gives the same tensor once its works end
            mine2, works = exchange_heads(send, async_op=True)
            for work in works:
                work.wait()
            ok_async = torch.equal(mine2, mine)
            want = full[:, :, rank * Hs:(rank + 1) * Hs].permute(0, 2, 1, 3)
            ok_heads = mine.shape == want.shape and torch.equal(mine, want) and ok_async
            zf = torch.arange(B * L * 2 * H * w, dtype=torch.float32).reshape(B, L, 2, H, w)
            got = z_heads_to_groups(zf[:, :, :, rank * Hs:(rank + 1) * Hs].contiguous())
            # [B, src, Ls, 2, Hs, w]: group src holds heads [src*Hs, (src+1)*Hs)
            zwant = zf[:, rank * Ls:(rank + 1) * Ls].reshape(B, Ls, 2, world, Hs, w)
            ok_tokens = got.shape == (B, world, Ls, 2, Hs, w) and torch.equal(
                got, zwant.permute(0, 3, 1, 2, 4, 5))
            res.append((ok_heads, ok_tokens))
        out.put((rank, res))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_reshard_exactly():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(r, [(True, True)] * len(SHAPES)) for r in range(2)]
