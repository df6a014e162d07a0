"""The head-sharded layer on one GPU (a process group of one rank over NCCL),
against the fp64 oracle and the single-GPU layer; and the head-group merge,
which reads Z in the layout the ranks of a head-sharded layer receive it in,
against the plain merge on one GPU.

With one rank the exchanges are pure layout changes, so Y must also equal the
single-GPU layer's bit for bit (the same kernels on the same values, the K
products of the merge in the same order)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle as O
import softmax_attention_video_vdn_b200 as vdn
from softmax_attention_video_vdn_b200 import build as vbuild
from softmax_attention_video_vdn_b200.layer import HybridLayer
from softmax_attention_video_vdn_b200.ulysses import UlyssesLayer
from synthetic import get_workload, make_inputs, to_f64
from tests.helpers import TOL, cfg_of, rel_err

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module", autouse=True)
def _library():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    vbuild.build()
    vdn.load_library()


@pytest.fixture(scope="module")
def one_rank_group():
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1)
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("kw", [
    dict(B=1, H=2, T=12, N=200, d_out=256, beta=0.5, seed=51),
    # context tokens are sharded with the video tokens; two batch items
    dict(B=2, H=2, T=7, N=65, d_out=256, n_ctx=77, seed=52),
])
def test_one_rank_head_sharded_layer(one_rank_group, kw):
    wl = get_workload("small", **kw)
    x = make_inputs(wl, device="cuda")
    cfg = cfg_of(wl)
    ref = HybridLayer(cfg).forward(x["q"], x["k"], x["v"], x["gate_logits"], x["W1"], x["W2"])
    seq = {n: x[n].permute(0, 2, 1, 3).contiguous() for n in ("q", "k", "v")}  # [B, L, H, d]
    layer = UlyssesLayer(cfg)
    Y = layer.forward(seq["q"], seq["k"], seq["v"], x["gate_logits"], x["W1"], x["W2"])
    torch.cuda.synchronize()
    assert vdn.vdn_read_status(layer.status) == 0
    assert torch.equal(Y, ref)
    x64 = {n: to_f64(x[n]) for n in ("q", "k", "v", "gate_logits", "W1", "W2")}
    want = O.vdn_layer(x64, wl)["Y"]
    e = rel_err(to_f64(Y), want)
    assert e <= TOL["bf16"], e


@pytest.mark.parametrize("groups,kw", [
    (2, dict(B=1, H=4, T=1, N=300, d_out=264, seed=71)),
    (3, dict(B=2, H=6, T=1, N=200, d_out=128, seed=72)),
    (4, dict(B=1, H=8, T=1, N=1000, d_out=512, seed=73)),
])
def test_head_group_merge_equals_plain_merge(groups, kw):
    wl = get_workload("small", **kw)
    x = make_inputs(wl, device="cuda")
    cfg = cfg_of(wl)
    B, L, H = cfg.B, cfg.L, cfg.H
    g = torch.Generator(device="cuda")
    g.manual_seed(wl.seed)
    Z = torch.randn((B, L, 2, H, 128), generator=g, device="cuda").to(torch.bfloat16)
    Y = torch.empty((B, L, wl.d_out), dtype=torch.bfloat16, device="cuda")
    vdn.vdn_gated_merge(cfg, Z, x["W1"], x["W2"], Y)
    # the received layout: [B, groups, L, 2, H/groups, dv]
    Zg = Z.view(B, L, 2, groups, H // groups, 128).permute(0, 3, 1, 2, 4, 5).contiguous()
    Yg = torch.full_like(Y, float("nan"))
    vdn.vdn_gated_merge_head_groups(cfg, groups, Zg, x["W1"], x["W2"], Yg)
    torch.cuda.synchronize()
    assert torch.equal(Yg, Y)
    # and against the oracle's merge (gate logits at 0: o = 2 Z)
    Z64 = to_f64(Z)
    o_sm = 2.0 * Z64[:, :, 0].transpose(0, 2, 1, 3)
    o_lin = 2.0 * Z64[:, :, 1].transpose(0, 2, 1, 3)
    want, _ = O.gated_merge(o_sm, o_lin, np.zeros(H), to_f64(x["W1"]), to_f64(x["W2"]))
    assert rel_err(to_f64(Yg), want) <= TOL["bf16"]


@pytest.mark.parametrize("groups,kw", [
    (1, dict(B=1, H=2, T=3, N=100, seed=81)),
    (4, dict(B=2, H=8, T=2, N=75, n_ctx=14, seed=82)),
    (8, dict(B=1, H=24, T=1, N=640, seed=83)),
])
def test_pack_head_groups_layout(groups, kw):
    wl = get_workload("small", **kw)
    cfg = cfg_of(wl)
    B, L, H = cfg.B, cfg.L, cfg.H
    g = torch.Generator(device="cuda")
    g.manual_seed(wl.seed)
    x = torch.randn((B, L, H, 128), generator=g, device="cuda").to(torch.bfloat16)
    out = torch.full((B, H // groups, groups, L, 128), float("nan"), dtype=torch.bfloat16,
                     device="cuda")
    vdn.vdn_pack_head_groups(cfg, groups, x, out)
    torch.cuda.synchronize()
    want = x.reshape(B, L, groups, H // groups, 128).permute(0, 3, 2, 1, 4)
    assert torch.equal(out, want)
