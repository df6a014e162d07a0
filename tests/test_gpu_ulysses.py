"""The head-sharded layer on one GPU (a process group of one rank over NCCL):
the re-sharding is then a pure layout change, and Y must equal the
single-GPU layer's bit for bit (the same kernels on the same values)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

import softmax_attention_video_vdn_b200 as vdn
from softmax_attention_video_vdn_b200 import build as vbuild
from softmax_attention_video_vdn_b200.layer import HybridLayer
from softmax_attention_video_vdn_b200.ulysses import UlyssesLayer
from synthetic import get_workload, make_inputs
from tests.helpers import cfg_of

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_head_sharded_layer_equals_layer():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    vbuild.build()
    vdn.load_library()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        wl = get_workload("small", B=1, H=2, T=12, N=200, d_out=256, beta=0.5, seed=51)
        x = make_inputs(wl, device="cuda")
        cfg = cfg_of(wl)
        ref = HybridLayer(cfg).forward(x["q"], x["k"], x["v"], x["gate_logits"], x["W1"], x["W2"])
        seq = {n: x[n].permute(0, 2, 1, 3).contiguous() for n in ("q", "k", "v")}  # [B, L, H, d]
        layer = UlyssesLayer(cfg)
        Y = layer.forward(seq["q"], seq["k"], seq["v"], x["gate_logits"], x["W1"], x["W2"])
        torch.cuda.synchronize()
        assert vdn.vdn_read_status(layer.status) == 0
        assert torch.equal(Y, ref)
    finally:
        dist.destroy_process_group()
