"""The layer backward through the C ABI, against the fp64 backward oracle.

Tolerances (max |err| / max |ref|): the kernels round P and dS to bf16 for
the tensor-core products, the saved o and the cotangents entering them are
bf16, and every gradient is stored as bf16. A rounding-level emulation of
those steps against the oracle gives 2e-3 to 5e-3 on the test shapes (also
with frames of fewer tokens than dimensions, where G_f is singular: the
linear branch's fp32 operands enter the tensor cores as a hi + lo pair of
bf16 matrices). The stated bound is TOL_BWD = 2e-2, as for the forward's bf16
outputs. The merge's weight gradients accumulate exact bf16 products in fp32:
TOL_DW = 1e-3 against the oracle on the same bf16 Z.
"""
import numpy as np
import pytest
import torch

import oracle as O
import softmax_attention_video_vdn_b200 as vdn
from softmax_attention_video_vdn_b200 import build as vbuild
from softmax_attention_video_vdn_b200.layer import HybridLayerTrain
from synthetic import get_workload, make_inputs, to_f64
from tests.helpers import cfg_of, rel_err

pytestmark = pytest.mark.gpu

TOL_BWD = 2e-2
TOL_DW = 1e-3
TOL_LSE = 2e-3     # absolute, log2 units (fp32 row sums)


@pytest.fixture(scope="module", autouse=True)
def _library():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    vbuild.build()
    vdn.load_library()


def _ws(cfg, kind):
    return torch.empty(vdn.vdn_workspace_size(cfg, kind), dtype=torch.uint8, device="cuda")


def _randn_bf16(shape, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).cuda()


MINI = {
    "ragged_tiles": dict(B=1, H=2, T=12, N=200, d_out=256, seed=31),
    "single_frame": dict(B=1, H=1, T=1, N=130, d_out=256, seed=32),
    "partial_last_block": dict(B=2, H=1, T=21, N=72, d_out=256, seed=33),
    "no_anchors": dict(B=1, H=1, T=16, N=128, anchors=0, d_out=256, seed=34),
    "context_tokens": dict(B=1, H=1, T=12, N=100, d_out=256, n_ctx=150, seed=35),
    # 4-frame blocks, a +-2 block window and a partial last block (T = 23:
    # block 5 = {20, 21, 22}): the scans' state cotangents enter at other
    # frames, and the backward's reuse of the forward's segments rests on the
    # mask's symmetry for this window too
    "wide_window": dict(B=1, H=1, T=23, N=100, block_frames=4, window_blocks=2, d_out=256,
                        seed=36),
    # more than one softmax backward launch (over 40 query segments)
    "many_segments": dict(B=1, H=1, T=241, N=12, d_out=256, seed=37),
}


@pytest.mark.parametrize("name", list(MINI))
def test_softmax_backward_against_oracle(name):
    wl = get_workload("small", **MINI[name])
    x = make_inputs(wl, device="cuda")
    cfg = cfg_of(wl)
    B, H, L = cfg.B, cfg.H, cfg.L
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = torch.empty((B, L, H, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, L), dtype=torch.float32, device="cuda")
    vdn.vdn_softmax_window_lse(cfg, x["q"], x["k"], x["v"], o, lse, _ws(cfg, vdn.VDN_WS_SOFTMAX),
                               status)
    do = _randn_bf16((B, L, H, 128), 100 + wl.seed)
    dq, dk, dv = (torch.empty((B, H, L, 128), dtype=torch.bfloat16, device="cuda")
                  for _ in range(3))
    vdn.vdn_softmax_window_bwd(cfg, x["q"], x["k"], x["v"], o, lse, do, dq, dk, dv,
                               _ws(cfg, vdn.VDN_WS_SOFTMAX_BWD), status)
    assert vdn.vdn_read_status(status) == 0
    q, k, v = (to_f64(x[n]) for n in ("q", "k", "v"))
    do64 = to_f64(do)
    mask = O.frame_mask(wl.T, wl.block_frames, wl.window_blocks, wl.anchors)
    scale = 1.0 / np.sqrt(wl.d)
    ref = [np.zeros((B, H, L, 128)) for _ in range(3)]
    lse_ref = np.zeros((B, H, L))
    for b in range(B):
        for h in range(H):
            r = O.softmax_window_bwd(q[b, h], k[b, h], v[b, h], do64[b, :, h], wl.T, wl.N,
                                     wl.n_ctx, mask, scale)
            for i in range(3):
                ref[i][b, h] = r[i]
            lse_ref[b, h] = O.softmax_row_lse2(q[b, h], k[b, h], wl.T, wl.N, wl.n_ctx, mask, scale)
    assert np.abs(to_f64(lse) - lse_ref).max() <= TOL_LSE
    for got, want, n in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
        assert rel_err(to_f64(got), want) <= TOL_BWD, n


@pytest.mark.parametrize("name", list(MINI))
def test_linear_backward_against_oracle(name):
    wl = get_workload("small", **dict(MINI[name], beta=0.7))
    x = make_inputs(wl, device="cuda")
    cfg = cfg_of(wl)
    B, H, L = cfg.B, cfg.H, cfg.L
    TN = wl.T * wl.N
    do = _randn_bf16((B, H, L, 128), 200 + wl.seed)
    dq, dk, dv = (torch.full((B, H, L, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
                  for _ in range(3))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    vdn.vda_linear_bwd(cfg, x["q"], x["k"], x["v"], do, dq, dk, dv,
                       _ws(cfg, vdn.VDN_WS_LINEAR_BWD), status)
    assert vdn.vdn_read_status(status) == 0
    q, k, v, do64 = (to_f64(t) for t in (x["q"], x["k"], x["v"], do))
    got = [to_f64(t) for t in (dq, dk, dv)]
    for g in got:
        assert np.isfinite(g).all()
        assert not g[:, :, TN:].any()          # context rows: no linear branch
    for b in range(B):
        for h in range(H):
            r = O.linear_branch_bwd(q[b, h, :TN], k[b, h, :TN], v[b, h, :TN], do64[b, h, :TN],
                                    wl.T, wl.N, wl.lam, wl.beta, wl.block_frames,
                                    wl.window_blocks, wl.anchors)
            for g, key in zip(got, ("dq", "dk", "dv")):
                assert rel_err(g[b, h, :TN], r[key]) <= TOL_BWD, (key, b, h)


def test_merge_backward_against_oracle():
    wl = get_workload("small", B=1, H=2, T=12, N=200, d_out=256, seed=41)
    x = make_inputs(wl, device="cuda")
    cfg = cfg_of(wl)
    B, H, L = cfg.B, cfg.H, cfg.L
    Z = _randn_bf16((B, L, 2, H, 128), 301)
    dY = _randn_bf16((B, L, wl.d_out), 302)
    dZ = torch.empty_like(Z)
    dW1 = torch.empty((H * 128, wl.d_out), dtype=torch.float32, device="cuda")
    dW2 = torch.empty_like(dW1)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    vdn.vdn_gated_merge_bwd(cfg, Z, x["W1"], x["W2"], dY, dZ, dW1, dW2, status)
    assert vdn.vdn_read_status(status) == 0
    # with the gate logits at 0 (g = 1/2) the oracle's o = 2 Z exactly
    Z64 = to_f64(Z)
    o_sm = 2.0 * Z64[:, :, 0].transpose(0, 2, 1, 3)
    o_lin = 2.0 * Z64[:, :, 1].transpose(0, 2, 1, 3)
    r = O.gated_merge_bwd(o_sm, o_lin, np.zeros(H), to_f64(x["W1"]), to_f64(x["W2"]),
                          to_f64(dY))
    dz_ref = np.stack([r["dz_sm"].transpose(0, 2, 1, 3), r["dz_lin"].transpose(0, 2, 1, 3)],
                      axis=2)
    assert rel_err(to_f64(dZ), dz_ref) <= 2.0 ** -8
    assert rel_err(dW1.cpu().numpy(), r["dW1"]) <= TOL_DW
    assert rel_err(dW2.cpu().numpy(), r["dW2"]) <= TOL_DW


LAYER = {
    "plain": dict(B=1, H=2, T=12, N=200, d_out=256, beta=0.5, seed=51),
    "context": dict(B=1, H=2, T=12, N=100, d_out=256, n_ctx=150, seed=52),
    "thin_frames": dict(B=2, H=1, T=21, N=72, d_out=256, beta=0.8, seed=53),
    "wide_window": dict(B=1, H=2, T=23, N=100, block_frames=4, window_blocks=2, d_out=256,
                        beta=0.6, seed=54),
}


@pytest.mark.parametrize("name", list(LAYER))
def test_layer_backward_against_oracle(name):
    wl = get_workload("small", **LAYER[name])
    x = make_inputs(wl, device="cuda")
    cfg = cfg_of(wl)
    layer = HybridLayerTrain(cfg)
    Y = layer.forward(x["q"], x["k"], x["v"], x["gate_logits"], x["W1"], x["W2"])
    dY = _randn_bf16(tuple(Y.shape), 400 + wl.seed)
    g = layer.backward(dY)
    assert layer.check_status() == 0
    x64 = {n: to_f64(x[n]) for n in ("q", "k", "v", "gate_logits", "W1", "W2")}
    ref = O.vdn_layer_bwd(x64, wl, to_f64(dY))
    assert rel_err(to_f64(Y), ref["fwd"]["Y"]) <= 2e-2
    for key in ("dq", "dk", "dv", "dgate_logits"):
        assert rel_err(to_f64(g[key]), ref[key]) <= TOL_BWD, key
    for key in ("dW1", "dW2"):
        assert rel_err(g[key].cpu().numpy(), ref[key]) <= TOL_BWD, key


def test_layer_backward_768p_sampled_rows():
    """The 768p workload in the benchmark's launch configuration: every
    gradient finite, and dq on sampled query rows of one head against the
    oracle computed row by row (softmax rows over their allowed keys, the
    linear branch's block states of that head, the merge for those tokens)."""
    wl = get_workload("768p")
    x = make_inputs(wl, device="cuda")
    cfg = cfg_of(wl)
    layer = HybridLayerTrain(cfg)
    layer.forward(x["q"], x["k"], x["v"], x["gate_logits"], x["W1"], x["W2"])
    dY = _randn_bf16((wl.B, wl.L, wl.d_out), 777)
    g = layer.backward(dY)
    assert layer.check_status() == 0
    for key, t in g.items():
        assert torch.isfinite(t).all(), key
    h = 5
    rng = np.random.default_rng(9)
    rows = np.sort(np.concatenate([rng.choice(wl.L, 24, replace=False),
                                   [0, wl.N - 1, 7 * wl.N + 3, wl.L - 1]]))
    q, k, v = (to_f64(x[n][0, h]) for n in ("q", "k", "v"))
    # the merge backward at the sampled tokens gives every head's do_sm and
    # do_lin there (o_sm and o_lin only enter the gate's and W's cotangents)
    R = len(rows)
    dYr = to_f64(dY[0, torch.as_tensor(rows)])[None]
    mb = O.gated_merge_bwd(np.zeros((1, wl.H, R, wl.dv)), np.zeros((1, wl.H, R, wl.dv)),
                           to_f64(x["gate_logits"]), to_f64(x["W1"]), to_f64(x["W2"]), dYr)
    mask = O.frame_mask(wl.T)
    ref = O.softmax_window_bwd_dq_rows(rows, q, k, v, mb["do_sm"][0, h], wl.N, mask,
                                       1.0 / np.sqrt(wl.d))
    # a row's linear dq depends only on its own cotangent: the oracle's linear
    # backward with do_lin zero outside the sampled rows gives it exactly
    do_lin = np.zeros((wl.L, wl.dv))
    do_lin[rows] = mb["do_lin"][0, h]
    lb = O.linear_branch_bwd(q, k, v, do_lin, wl.T, wl.N, wl.lam, wl.beta)
    ref = ref + lb["dq"][rows]
    got = to_f64(g["dq"][0, h, torch.as_tensor(rows)])
    assert rel_err(got, ref) <= TOL_BWD
