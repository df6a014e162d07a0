"""Allocation helpers around the C ABI: output and workspace tensors are
torch CUDA memory; every computation is one of the library's entry points.
"""
import torch

from . import (VDN_WS_BACKWARD, VDN_WS_LAYER, VDN_WS_LAYER_FP8, VDN_WS_SCAN, VDN_WS_SOFTMAX,
               vda_bidir_scan, vda_frame_stats, vda_readout, vdn_gated_merge, vdn_hybrid_backward,
               vdn_hybrid_forward, vdn_hybrid_forward_fp8, vdn_hybrid_forward_train,
               vdn_read_status, vdn_softmax_window, vdn_workspace_size)

_DT = {0: torch.float32, 1: torch.bfloat16}


def io_dtype(cfg):
    return _DT[cfg.dtype]


def _ws(cfg, kind, device):
    n = vdn_workspace_size(cfg, kind)
    if n == 0:
        raise ValueError("invalid configuration")
    return torch.empty(n, dtype=torch.uint8, device=device)


class HybridLayer:
    """Owns the workspace, the status word and the output of one layer shape."""

    def __init__(self, cfg, device="cuda", fp8=False):
        self.cfg = cfg
        self.fp8 = fp8
        self.device = torch.device(device)
        self.ws = _ws(cfg, VDN_WS_LAYER_FP8 if fp8 else VDN_WS_LAYER, self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        c = cfg
        shape = (c.B, c.L, c.H, c.d_out) if c.w_per_head else (c.B, c.L, c.d_out)
        self.Y = torch.empty(shape, dtype=io_dtype(c), device=self.device)

    def forward(self, q, k, v, gate_logits, W1, W2, stream=None):
        fwd = vdn_hybrid_forward_fp8 if self.fp8 else vdn_hybrid_forward
        fwd(self.cfg, q, k, v, gate_logits, W1, W2, self.Y, self.ws, self.status, stream)
        return self.Y

    def check_status(self, stream=None):
        return vdn_read_status(self.status, stream)


class HybridLayerTrain:
    """Forward that keeps what the backward needs (Z, lse), and the backward.

    bf16 only. forward() returns Y; backward(dY) returns the cotangents
    dq, dk, dv (bf16, like q), dgate_logits [H] and dW1, dW2 (fp32).
    """

    def __init__(self, cfg, device="cuda"):
        self.cfg = c = cfg
        self.device = dev = torch.device(device)
        self.ws = _ws(cfg, VDN_WS_LAYER, dev)
        self.bws = _ws(cfg, VDN_WS_BACKWARD, dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        bf = torch.bfloat16
        self.Y = torch.empty((c.B, c.L, c.d_out), dtype=bf, device=dev)
        self.Z = torch.empty((c.B, c.L, 2, c.H, c.dv), dtype=bf, device=dev)
        self.lse = torch.empty((c.B, c.H, c.L), dtype=torch.float32, device=dev)
        self.dq = torch.empty((c.B, c.H, c.L, c.d), dtype=bf, device=dev)
        self.dk = torch.empty_like(self.dq)
        self.dv = torch.empty((c.B, c.H, c.L, c.dv), dtype=bf, device=dev)
        self.dgate = torch.empty(c.H, dtype=torch.float32, device=dev)
        self.dW1 = torch.empty((c.H * c.dv, c.d_out), dtype=torch.float32, device=dev)
        self.dW2 = torch.empty_like(self.dW1)
        self._saved = None

    def forward(self, q, k, v, gate_logits, W1, W2, stream=None):
        vdn_hybrid_forward_train(self.cfg, q, k, v, gate_logits, W1, W2, self.Y, self.Z, self.lse,
                                 self.ws, self.status, stream)
        self._saved = (q, k, v, gate_logits, W1, W2)
        return self.Y

    def backward(self, dY, stream=None):
        if self._saved is None:
            raise RuntimeError("backward() needs a forward() first")
        q, k, v, g, W1, W2 = self._saved
        vdn_hybrid_backward(self.cfg, q, k, v, g, W1, W2, self.Z, self.lse, dY, self.dq, self.dk,
                            self.dv, self.dgate, self.dW1, self.dW2, self.bws, self.status, stream)
        return dict(dq=self.dq, dk=self.dk, dv=self.dv, dgate_logits=self.dgate, dW1=self.dW1,
                    dW2=self.dW2)

    def check_status(self, stream=None):
        return vdn_read_status(self.status, stream)


def run_stages(cfg, x, softmax=True, fused=True, readout=True, stream=None):
    """Run the entry points one by one; returns every intermediate.

    x: dict with q, k, v (CUDA tensors), gate_logits, and W1, W2 when merging.
    """
    c = cfg
    dev = x["k"].device
    out = {}
    BH = c.B * c.H
    G = torch.empty((c.B, c.H, c.T, c.d, c.d), dtype=torch.float32, device=dev)
    C = torch.empty((c.B, c.H, c.T, c.dv, c.d), dtype=torch.float32, device=dev)
    vda_frame_stats(c, x["k"], x["v"], G, C, stream)
    out["G"], out["C"] = G, C
    S_fwd = torch.empty((c.B, c.H, c.nb, c.dv, c.d), dtype=torch.float32, device=dev)
    S_bwd = torch.empty_like(S_fwd)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = _ws(c, VDN_WS_SCAN, dev)
    vda_bidir_scan(c, G, C, S_fwd, S_bwd, ws, status, stream)
    out["S_fwd"], out["S_bwd"] = S_fwd, S_bwd
    dt = io_dtype(c)
    if readout:
        o_lin = torch.empty((c.B, c.L, c.H, c.dv), dtype=dt, device=dev)
        vda_readout(c, x["q"], S_fwd, S_bwd, o_lin, stream)
        out["o_lin"] = o_lin
    if softmax:
        sws = _ws(c, VDN_WS_SOFTMAX, dev)
        o_sm = torch.empty((c.B, c.L, c.H, c.dv), dtype=dt, device=dev)
        vdn_softmax_window(c, x["q"], x["k"], x["v"], None, None, None, o_sm, sws, status, stream)
        out["o_sm"] = o_sm
        if fused:
            Z = torch.empty((c.B, c.L, 2, c.H, c.dv), dtype=dt, device=dev)
            vdn_softmax_window(c, x["q"], x["k"], x["v"], S_fwd, S_bwd, x["gate_logits"], Z, sws,
                               status, stream)
            out["Z"] = Z
            if c.d_out and "W1" in x:
                shape = (c.B, c.L, c.H, c.d_out) if c.w_per_head else (c.B, c.L, c.d_out)
                Y = torch.empty(shape, dtype=dt, device=dev)
                vdn_gated_merge(c, Z, x["W1"], x["W2"], Y, stream)
                out["Y"] = Y
    out["status"] = vdn_read_status(status, stream)
    del BH
    return out
