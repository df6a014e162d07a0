"""Head-sharded layer over several GPUs (Ulysses sequence parallelism).

The pages report their fastest runs with branch-specific Ulysses sequence
parallelism on 8 B200 ("Performance Results"). Every (b, h) is independent
through the frame statistics, the scan, the softmax and the readout; only
the output projections mix heads. So, with one process per GPU:

1. tokens arrive sequence-sharded, [B, L/world, H, d] per rank (token-major,
   as a projection produces them);
2. one all-to-all per tensor re-shards q, k and v by head: each rank gets
   H/world heads over the whole sequence, in the library's [B, H, L, d]
   layout;
3. each rank runs the hybrid path on its heads through the C ABI (gated Z
   for its heads, every token);
4. one all-to-all re-shards Z back by sequence: [B, L/world, 2, H, dv];
5. each rank runs the merge GEMM on its tokens with the full projections.

The collectives are torch.distributed all-to-alls (NCCL on GPUs); the
layout changes around them are tensor copies. This module is plumbing: every
computation of the layer is one of the library's entry points.
"""
import torch
import torch.distributed as dist

from . import (VDN_WS_SCAN, VDN_WS_SOFTMAX, make_config, vda_bidir_scan, vda_frame_stats,
               vdn_gated_merge, vdn_softmax_window, vdn_workspace_size)

__all__ = ["seq_to_heads", "z_heads_to_seq", "UlyssesLayer"]


def seq_to_heads(x, group=None):
    """[B, Ls, H, w] (this rank's tokens, all heads) -> [B, H/world, world*Ls, w]
    (this rank's heads, all tokens). Rank r receives heads [r*Hs, (r+1)*Hs)."""
    world = dist.get_world_size(group)
    B, Ls, H, w = x.shape
    if H % world:
        raise ValueError(f"{H} heads do not split over {world} ranks")
    Hs = H // world
    send = x.reshape(B, Ls, world, Hs, w).permute(2, 0, 1, 3, 4).contiguous()  # [dst, B, Ls, Hs, w]
    recv = torch.empty_like(send)                                             # [src, B, Ls, Hs, w]
    dist.all_to_all_single(recv, send, group=group)
    # token index = src * Ls + l
    return recv.permute(1, 3, 0, 2, 4).reshape(B, Hs, world * Ls, w).contiguous()


def z_heads_to_seq(z, group=None):
    """[B, L, 2, Hs, dv] (this rank's heads, all tokens) -> [B, L/world, 2, world*Hs, dv]
    (this rank's tokens, all heads). Rank r receives tokens [r*Ls, (r+1)*Ls)."""
    world = dist.get_world_size(group)
    B, L, two, Hs, dv = z.shape
    if L % world:
        raise ValueError(f"{L} tokens do not split over {world} ranks")
    Ls = L // world
    send = z.reshape(B, world, Ls, two, Hs, dv).permute(1, 0, 2, 3, 4, 5).contiguous()
    recv = torch.empty_like(send)                                  # [src, B, Ls, 2, Hs, dv]
    dist.all_to_all_single(recv, send, group=group)
    # head index = src * Hs + h
    return recv.permute(1, 2, 3, 0, 4, 5).reshape(B, Ls, two, world * Hs, dv).contiguous()


class UlyssesLayer:
    """The hybrid layer with its heads sharded over the ranks of `group`.

    cfg: the full layer's configuration (all H heads, L = T*N tokens), bf16
    or fp32 as the inputs. forward() takes this rank's token shard of q, k,
    v ([B, L/world, H, d]), the full gate logits [H] and projections W1, W2
    [H*dv, d_out], and returns this rank's rows of Y [B, L/world, d_out].
    """

    def __init__(self, cfg, group=None, device="cuda"):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        L = cfg.T * cfg.N
        if cfg.H % self.world or L % self.world:
            raise ValueError("heads and tokens must split evenly over the ranks")
        if cfg.w_per_head:
            raise ValueError("head-shared projections are per head: shard them with the heads")
        self.cfg = cfg
        self.Hs, self.Ls = cfg.H // self.world, L // self.world
        common = dict(B=cfg.B, d=cfg.d, dv=cfg.dv, dtype=cfg.dtype, lam=cfg.lambda_,
                      beta=cfg.beta, block_frames=cfg.block_frames,
                      window_blocks=cfg.window_blocks, anchors=cfg.anchors, d_out=cfg.d_out,
                      softmax_scale=cfg.softmax_scale)
        # this rank's heads over every frame; the merge over this rank's tokens
        self.cfg_heads = make_config(H=self.Hs, T=cfg.T, N=cfg.N, **common)
        self.cfg_tokens = make_config(H=cfg.H, T=1, N=self.Ls, **common)
        dev = torch.device(device)
        f32 = dict(dtype=torch.float32, device=dev)
        c = self.cfg_heads
        self.G = torch.empty((c.B, c.H, c.T, c.d, c.d), **f32)
        self.C = torch.empty((c.B, c.H, c.T, c.dv, c.d), **f32)
        self.S_fwd = torch.empty((c.B, c.H, c.nb, c.dv, c.d), **f32)
        self.S_bwd = torch.empty_like(self.S_fwd)
        u8 = dict(dtype=torch.uint8, device=dev)
        self.scan_ws = torch.empty(vdn_workspace_size(c, VDN_WS_SCAN), **u8)
        self.sm_ws = torch.empty(vdn_workspace_size(c, VDN_WS_SOFTMAX), **u8)
        io = torch.bfloat16 if cfg.dtype == 1 else torch.float32
        self.Z = torch.empty((c.B, L, 2, self.Hs, c.dv), dtype=io, device=dev)
        self.Y = torch.empty((cfg.B, self.Ls, cfg.d_out), dtype=io, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def forward(self, q_seq, k_seq, v_seq, gate_logits, W1, W2, stream=None):
        c = self.cfg_heads
        q, k, v = (seq_to_heads(t, self.group) for t in (q_seq, k_seq, v_seq))
        g = gate_logits[self.rank * self.Hs:(self.rank + 1) * self.Hs].contiguous()
        vda_frame_stats(c, k, v, self.G, self.C, stream)
        vda_bidir_scan(c, self.G, self.C, self.S_fwd, self.S_bwd, self.scan_ws, self.status, stream)
        vdn_softmax_window(c, q, k, v, self.S_fwd, self.S_bwd, g, self.Z, self.sm_ws, self.status,
                           stream)
        z = z_heads_to_seq(self.Z, self.group)
        vdn_gated_merge(self.cfg_tokens, z, W1, W2, self.Y, stream)
        return self.Y
