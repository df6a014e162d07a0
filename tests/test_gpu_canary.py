"""Guard regions around every output of every entry point (the stand-in for a
memory checker on this pool).

Each output buffer, the workspaces and the status word sit inside one
allocation between two 4 KiB guard regions of a known byte pattern (the
padding up to the next 256 bytes after the buffer belongs to the upper
guard). Outputs start as NaN (or as an e4m3 NaN code), so that a row the
kernels skip shows up as non-finite. After each call through the C ABI
every guard must be unchanged and every output finite. The shapes are the
odd ones: frames of 1, 65 and 129 tokens, a partial last block, context
tokens, two batch items.
"""
import numpy as np
import pytest
import torch

import softmax_attention_video_vdn_b200 as vdn
from softmax_attention_video_vdn_b200 import build as vbuild
from synthetic import get_workload, make_inputs
from tests.helpers import cfg_of

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _library():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    vbuild.build()
    vdn.load_library()


class Guarded:
    """A tensor of `shape` and `dtype` inside [guard | buffer | pad + guard]."""

    def __init__(self, name, shape, dtype, fill="nan"):
        self.name = name
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n = n
        inner = (n + 255) // 256 * 256
        self.raw = torch.full((GUARD + inner + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(shape)
        if fill == "nan":
            if dtype == torch.uint8:
                self.t.fill_(0x7F)          # an e4m3 NaN code
            else:
                self.t.fill_(float("nan"))
        elif fill is not None:
            self.t.fill_(fill)

    def guards_intact(self):
        lo = self.raw[:GUARD]
        hi = self.raw[GUARD + self.n:]
        return bool((lo == PATTERN).all()) and bool((hi == PATTERN).all())


def _finite(t):
    if t.dtype == torch.uint8:                 # e4m3 codes: no NaN code
        return bool(((t & 0x7F) != 0x7F).all())
    return bool(torch.isfinite(t.float()).all())


SHAPES = {
    # 65-token frames, partial last block (T = 11: block 2 = {10})
    "n65_partial_block": dict(B=1, H=2, T=11, N=65, d_out=136, seed=61),
    # one-token frames, context tokens, two batch items
    "n1_context": dict(B=2, H=1, T=7, N=1, d_out=128, n_ctx=33, seed=62),
    # 129-token frames, partial last block and context tokens
    "n129_context": dict(B=1, H=1, T=16, N=129, d_out=256, n_ctx=77, seed=63),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_outputs_stay_inside_their_buffers(name):
    wl = get_workload("small", **SHAPES[name])
    x = make_inputs(wl, device="cuda")
    cfg = cfg_of(wl)
    B, H, L, T, nb, d, dv = cfg.B, cfg.H, cfg.L, cfg.T, cfg.nb, cfg.d, cfg.dv
    bf, f32, u8 = torch.bfloat16, torch.float32, torch.uint8
    q, k, v, gate, W1, W2 = (x[n] for n in ("q", "k", "v", "gate_logits", "W1", "W2"))
    bufs = []

    def out(nm, shape, dtype, fill="nan"):
        g = Guarded(nm, shape, dtype, fill)
        bufs.append(g)
        return g.t

    def ws(nm, kind):
        return out(nm, (vdn.vdn_workspace_size(cfg, kind),), u8, fill=None)

    status = out("status", (1,), torch.int32, fill=0)

    def check(step, outputs):
        st = vdn.vdn_read_status(status)
        assert st == 0, f"{step}: {vdn.vdn_status_string(st)}"
        bad = [g.name for g in bufs if not g.guards_intact()]
        assert not bad, f"{step}: guard overwritten around {bad}"
        for nm, t in outputs:
            assert _finite(t), f"{step}: {nm} has unwritten or non-finite entries"

    # linear branch, stage by stage
    G = out("G", (B, H, T, d, d), f32)
    C = out("C", (B, H, T, dv, d), f32)
    vdn.vda_frame_stats(cfg, k, v, G, C)
    check("vda_frame_stats", [("G", G), ("C", C)])
    S_f = out("S_fwd", (B, H, nb, dv, d), f32)
    S_b = out("S_bwd", (B, H, nb, dv, d), f32)
    vdn.vda_bidir_scan(cfg, G, C, S_f, S_b, ws("scan ws", vdn.VDN_WS_SCAN), status)
    check("vda_bidir_scan", [("S_fwd", S_f), ("S_bwd", S_b)])
    S_f2 = out("S_fwd (no-alloc)", (B, H, nb, dv, d), f32)
    S_b2 = out("S_bwd (no-alloc)", (B, H, nb, dv, d), f32)
    vdn.vda_bidir_scan_noalloc(cfg, G, C, S_f2, S_b2, status)
    check("vda_bidir_scan_noalloc", [("S_fwd", S_f2), ("S_bwd", S_b2)])
    o_lin = out("o_lin", (B, L, H, dv), bf)
    vdn.vda_readout(cfg, q, S_f, S_b, o_lin)
    check("vda_readout", [("o_lin", o_lin)])

    # softmax branch and gated halves of Z
    sm_ws = ws("softmax ws", vdn.VDN_WS_SOFTMAX)
    o_sm = out("o_sm", (B, L, H, dv), bf)
    vdn.vdn_softmax_window(cfg, q, k, v, None, None, None, o_sm, sm_ws, status)
    check("vdn_softmax_window (o_sm)", [("o_sm", o_sm)])
    Z = out("Z", (B, L, 2, H, dv), bf)
    vdn.vdn_softmax_window(cfg, q, k, v, None, None, gate, Z, sm_ws, status)
    vdn.vda_readout_gated(cfg, q, S_f, S_b, gate, Z)
    check("vdn_softmax_window + vda_readout_gated", [("Z", Z)])
    Z2 = out("Z (with states)", (B, L, 2, H, dv), bf)
    vdn.vdn_softmax_window(cfg, q, k, v, S_f, S_b, gate, Z2, sm_ws, status)
    check("vdn_softmax_window (with states)", [("Z", Z2)])
    Y = out("Y", (B, L, wl.d_out), bf)
    vdn.vdn_gated_merge(cfg, Z2, W1, W2, Y)
    check("vdn_gated_merge", [("Y", Y)])
    Y2 = out("Y (layer)", (B, L, wl.d_out), bf)
    vdn.vdn_hybrid_forward(cfg, q, k, v, gate, W1, W2, Y2, ws("layer ws", vdn.VDN_WS_LAYER),
                           status)
    check("vdn_hybrid_forward", [("Y", Y2)])

    # e4m3 softmax branch
    qws = ws("quant ws", vdn.VDN_WS_QUANT)
    x8, sc = [], []
    for nm, t in (("q8", q), ("k8", k), ("v8", v)):
        x8.append(out(nm, tuple(t.shape), u8))
        sc.append(out(nm + " scale", (B * H,), f32))
        vdn.vdn_quantize_fp8(cfg, t, x8[-1], sc[-1], qws)
    check("vdn_quantize_fp8", list(zip(("q8", "k8", "v8"), x8)) + [("scales", s) for s in sc])
    Z8 = out("Z (e4m3)", (B, L, 2, H, dv), bf)
    vdn.vdn_softmax_window_fp8(cfg, x8[0], x8[1], x8[2], sc[0], sc[1], sc[2], gate, Z8, sm_ws,
                               status)
    vdn.vda_readout_gated(cfg, q, S_f, S_b, gate, Z8)
    check("vdn_softmax_window_fp8", [("Z", Z8)])
    Y8 = out("Y (e4m3 layer)", (B, L, wl.d_out), bf)
    vdn.vdn_hybrid_forward_fp8(cfg, q, k, v, gate, W1, W2, Y8,
                               ws("fp8 layer ws", vdn.VDN_WS_LAYER_FP8), status)
    check("vdn_hybrid_forward_fp8", [("Y", Y8)])

    # backward, part by part and whole
    lse = out("lse", (B, H, L), f32)
    o_sm2 = out("o_sm (lse)", (B, L, H, dv), bf)
    vdn.vdn_softmax_window_lse(cfg, q, k, v, o_sm2, lse, sm_ws, status)
    check("vdn_softmax_window_lse", [("o_sm", o_sm2), ("lse", lse)])
    gen = torch.Generator(device="cuda")
    gen.manual_seed(wl.seed)
    do = torch.randn((B, L, H, dv), generator=gen, device="cuda").to(bf)
    grads = [out(nm, (B, H, L, d), bf) for nm in ("dq", "dk", "dv")]
    vdn.vdn_softmax_window_bwd(cfg, q, k, v, o_sm2, lse, do, *grads,
                               ws("softmax bwd ws", vdn.VDN_WS_SOFTMAX_BWD), status)
    check("vdn_softmax_window_bwd", list(zip(("dq", "dk", "dv"), grads)))
    do_lin = torch.randn((B, H, L, dv), generator=gen, device="cuda").to(bf)
    lgrads = [out(nm, (B, H, L, d), bf) for nm in ("dq (lin)", "dk (lin)", "dv (lin)")]
    vdn.vda_linear_bwd(cfg, q, k, v, do_lin, *lgrads, ws("linear bwd ws", vdn.VDN_WS_LINEAR_BWD),
                       status)
    check("vda_linear_bwd", list(zip(("dq", "dk", "dv"), lgrads)))
    dY = torch.randn((B, L, wl.d_out), generator=gen, device="cuda").to(bf)
    dZ = out("dZ", (B, L, 2, H, dv), bf)
    dW = [out(nm, (H * dv, wl.d_out), f32) for nm in ("dW1", "dW2")]
    vdn.vdn_gated_merge_bwd(cfg, Z2, W1, W2, dY, dZ, *dW, status)
    check("vdn_gated_merge_bwd", [("dZ", dZ), ("dW1", dW[0]), ("dW2", dW[1])])
    Yt = out("Y (train)", (B, L, wl.d_out), bf)
    Zt = out("Z (train)", (B, L, 2, H, dv), bf)
    lt = out("lse (train)", (B, H, L), f32)
    vdn.vdn_hybrid_forward_train(cfg, q, k, v, gate, W1, W2, Yt, Zt, lt,
                                 ws("train ws", vdn.VDN_WS_LAYER), status)
    check("vdn_hybrid_forward_train", [("Y", Yt), ("Z", Zt), ("lse", lt)])
    hg = [out(nm, (B, H, L, d), bf) for nm in ("dq (layer)", "dk (layer)", "dv (layer)")]
    dgate = out("dgate_logits", (H,), f32)
    hW = [out(nm, (H * dv, wl.d_out), f32) for nm in ("dW1 (layer)", "dW2 (layer)")]
    vdn.vdn_hybrid_backward(cfg, q, k, v, gate, W1, W2, Zt, lt, dY, *hg, dgate, *hW,
                            ws("backward ws", vdn.VDN_WS_BACKWARD), status)
    check("vdn_hybrid_backward", list(zip(("dq", "dk", "dv"), hg)) + [("dgate", dgate),
                                                                      ("dW1", hW[0]),
                                                                      ("dW2", hW[1])])
