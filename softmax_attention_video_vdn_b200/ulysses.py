"""Head-sharded layer over several GPUs (Ulysses sequence parallelism).

The pages report their fastest runs with branch-specific Ulysses sequence
parallelism on 8 B200 ("Performance Results"). Every (b, h) is independent
through the frame statistics, the scan, the softmax and the readout; only
the output projections mix heads. So, with one process per GPU:

1. tokens arrive sequence-sharded, [B, Ls, H, d] per rank (token-major, as a
   projection produces them; Ls = L / world, L = T*N video tokens followed by
   n_ctx context tokens);
2. q, k and v are re-sharded by head: one layout copy per tensor
   (vdn_pack_head_groups) puts each destination's heads in a contiguous run,
   then one all-to-all per (batch item, local head) lands every rank's tokens
   straight in the library's [B, H/world, L, d] layout (no copy after the
   exchange); q's exchange runs asynchronously while the frame statistics,
   the solve and the scan (which need only k and v) compute;
3. each rank runs the hybrid path on its heads through the C ABI, which
   writes the gated Z of its heads, token-major [B, L, 2, H/world, dv]; the
   tokens of destination rank r are the contiguous rows [r*Ls, (r+1)*Ls);
4. one all-to-all per batch item sends those rows as they are; each rank
   receives [B, world, Ls, 2, H/world, dv] (its tokens, one head group per
   source rank);
5. vdn_gated_merge_head_groups multiplies that layout by the full
   projections directly, with no copy back to [B, Ls, 2, H, dv].

Per rank that is one layout copy of each of q, k and v and none of Z. The
collectives are torch.distributed all-to-alls (NCCL over NVLink on GPUs, gloo
in the CPU tests of the exchange); every computation of the layer is one of
the library's entry points.
"""
import torch
import torch.distributed as dist

from . import (VDN_WS_SCAN, VDN_WS_SOFTMAX, make_config, vda_bidir_scan, vda_frame_stats,
               vda_readout_gated, vdn_gated_merge_head_groups, vdn_pack_head_groups,
               vdn_softmax_window, vdn_workspace_size)

__all__ = ["exchange_heads", "z_heads_to_groups", "UlyssesLayer", "STAGES"]

# stage names of UlyssesLayer.forward's events
STAGES = ("reshard_qkv", "frame_stats", "solve_scan", "softmax_window", "readout", "reshard_z",
          "gated_merge")


def exchange_heads(send, group=None, async_op=False):
    """[B, Hs, world, Ls, w] (this rank's tokens; [b, h, g] = head g*Hs + h,
    as vdn_pack_head_groups lays them out) -> [B, Hs, world*Ls, w] (this
    rank's heads, all tokens; token index = source rank * Ls + l). Rank r
    receives heads [r*Hs, (r+1)*Hs). With async_op, returns (out, works):
    out is valid once every work has been waited for."""
    world = dist.get_world_size(group)
    B, Hs, g, Ls, w = send.shape
    if g != world:
        raise ValueError(f"{g} head groups for {world} ranks")
    out = torch.empty((B, Hs, world * Ls, w), dtype=send.dtype, device=send.device)
    works = []
    for b in range(B):
        for h in range(Hs):
            works.append(dist.all_to_all_single(out[b, h], send[b, h], group=group,
                                                async_op=async_op))
    return (out, works) if async_op else out


def z_heads_to_groups(z, group=None):
    """[B, L, 2, Hs, dv] (this rank's heads, all tokens) ->
    [B, world, L/world, 2, Hs, dv] (this rank's tokens; index 1 = the source
    rank, i.e. the head group [src*Hs, (src+1)*Hs)). Rank r receives tokens
    [r*Ls, (r+1)*Ls)."""
    world = dist.get_world_size(group)
    B, L, two, Hs, dv = z.shape
    if L % world:
        raise ValueError(f"{L} tokens do not split over {world} ranks")
    Ls = L // world
    out = torch.empty((B, world, Ls, two, Hs, dv), dtype=z.dtype, device=z.device)
    for b in range(B):
        dist.all_to_all_single(out[b], z[b].contiguous(), group=group)
    return out


class UlyssesLayer:
    """The hybrid layer with its heads sharded over the ranks of `group`.

    cfg: the full layer's configuration (all H heads, L = T*N + n_ctx tokens),
    bf16. forward() takes this rank's token shard of q, k, v ([B, L/world, H,
    d]), the full gate logits [H] and projections W1, W2 [H*dv, d_out], and
    returns this rank's rows of Y [B, L/world, d_out].
    """

    def __init__(self, cfg, group=None, device="cuda"):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        L = cfg.T * cfg.N + cfg.n_ctx
        if cfg.H % self.world or L % self.world:
            raise ValueError("heads and tokens must split evenly over the ranks")
        if cfg.w_per_head:
            raise ValueError("head-shared projections are per head: shard them with the heads")
        if cfg.dtype != 1:
            raise ValueError("the head-sharded merge takes bf16 inputs")
        self.cfg = cfg
        self.Hs, self.Ls = cfg.H // self.world, L // self.world
        common = dict(B=cfg.B, d=cfg.d, dv=cfg.dv, dtype=cfg.dtype, lam=cfg.lambda_,
                      beta=cfg.beta, block_frames=cfg.block_frames,
                      window_blocks=cfg.window_blocks, anchors=cfg.anchors, d_out=cfg.d_out,
                      softmax_scale=cfg.softmax_scale)
        # this rank's heads over every token; the merge over this rank's tokens
        self.cfg_heads = make_config(H=self.Hs, T=cfg.T, N=cfg.N, n_ctx=cfg.n_ctx, **common)
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
        self.Z = torch.empty((c.B, L, 2, self.Hs, c.dv), dtype=torch.bfloat16, device=dev)
        self.Y = torch.empty((cfg.B, self.Ls, cfg.d_out), dtype=torch.bfloat16, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def _to_heads(self, x, stream, async_op=False):
        """This rank's token shard [B, Ls, H, d] -> its heads over every token
        (with async_op: (heads, works), valid once the works are waited for)."""
        send = torch.empty((self.cfg.B, self.Hs, self.world, self.Ls, self.cfg.d),
                           dtype=x.dtype, device=x.device)
        vdn_pack_head_groups(self.cfg_tokens, self.world, x, send, stream)
        return exchange_heads(send, self.group, async_op=async_op)

    def forward(self, q_seq, k_seq, v_seq, gate_logits, W1, W2, stream=None, Y=None,
                events=None):
        """Y (this rank's token rows). The collectives and the kernels run in
        `stream` (default: the current stream). `Y` optionally names the output
        buffer; `events`, if given, is a list of len(STAGES) + 1 CUDA events
        recorded before the first stage and after each stage."""
        if stream is not None:
            with torch.cuda.stream(stream):
                return self._forward(q_seq, k_seq, v_seq, gate_logits, W1, W2, Y, events)
        return self._forward(q_seq, k_seq, v_seq, gate_logits, W1, W2, Y, events)

    def _forward(self, q_seq, k_seq, v_seq, gate_logits, W1, W2, Y, events):
        c = self.cfg_heads
        Y = self.Y if Y is None else Y
        stream = torch.cuda.current_stream()

        def mark(i):
            if events is not None:
                events[i].record(stream)

        mark(0)
        # k and v first; q travels while the linear branch (which needs only
        # k and v) runs, and the softmax waits for it
        k, v = (self._to_heads(t, stream) for t in (k_seq, v_seq))
        q, q_works = self._to_heads(q_seq, stream, async_op=True)
        mark(1)
        g = gate_logits[self.rank * self.Hs:(self.rank + 1) * self.Hs].contiguous()
        vda_frame_stats(c, k, v, self.G, self.C, stream)
        mark(2)
        vda_bidir_scan(c, self.G, self.C, self.S_fwd, self.S_bwd, self.scan_ws, self.status, stream)
        for w in q_works:
            w.wait()
        mark(3)
        # the two halves of the gated Z (the kernels vdn_softmax_window runs
        # when given the states, one entry point each so that each is timed)
        vdn_softmax_window(c, q, k, v, None, None, g, self.Z, self.sm_ws, self.status, stream)
        mark(4)
        vda_readout_gated(c, q, self.S_fwd, self.S_bwd, g, self.Z, stream)
        mark(5)
        z = z_heads_to_groups(self.Z, self.group)
        mark(6)
        vdn_gated_merge_head_groups(self.cfg_tokens, self.world, z, W1, W2, Y, stream)
        mark(7)
        return Y
