"""Head-sharded (Ulysses) re-sharding on CPU: two gloo ranks, one process
each. Each rank holds a token shard of the same full tensors; after
seq_to_heads it must hold exactly its heads over every token, and
z_heads_to_seq must give exactly its tokens over every head (integers, so
the comparison is exact)."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from softmax_attention_video_vdn_b200.ulysses import seq_to_heads, z_heads_to_seq
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, L, H, w = 2, 12, 6, 5
        Ls, Hs = L // world, H // world
        full = torch.arange(B * L * H * w, dtype=torch.float32).reshape(B, L, H, w)
        mine = seq_to_heads(full[:, rank * Ls:(rank + 1) * Ls].contiguous())
        want = full[:, :, rank * Hs:(rank + 1) * Hs].permute(0, 2, 1, 3)
        ok_heads = mine.shape == want.shape and torch.equal(mine, want)
        zf = torch.arange(B * L * 2 * H * w, dtype=torch.float32).reshape(B, L, 2, H, w)
        back = z_heads_to_seq(zf[:, :, :, rank * Hs:(rank + 1) * Hs].contiguous())
        ok_tokens = torch.equal(back, zf[:, rank * Ls:(rank + 1) * Ls])
        out.put((rank, ok_heads, ok_tokens))
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
    assert res == [(0, True, True), (1, True, True)]
