"""Failure detection on the GPU without a GPU fault.

A bounded wait that nothing satisfies must give up, report VDN_ERR_TIMEOUT
through the status word and leave the context usable; a frame whose
G_f + lambda I is not positive definite must report VDN_ERR_NUMERIC.
"""
import numpy as np
import pytest
import torch

import oracle as O
import softmax_attention_video_vdn_b200 as vdn
from softmax_attention_video_vdn_b200 import build as vbuild
from softmax_attention_video_vdn_b200.layer import HybridLayer, _ws
from synthetic import get_workload, make_inputs, to_f64
from tests.helpers import cfg_of, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    vbuild.build()
    vdn.load_library()


def test_bounded_wait_times_out_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    vdn.vdn_selftest_timeout(status, 50)
    assert vdn.vdn_read_status(status) == 5          # VDN_ERR_TIMEOUT
    assert vdn.vdn_read_status(status) == 0          # read clears the word
    # the context is still usable: a full layer runs and matches the oracle
    wl = get_workload("small", B=1, H=1, T=12, N=130, d_out=128, seed=31)
    x = make_inputs(wl)
    xg = {k: (t.cuda() if torch.is_tensor(t) else t) for k, t in x.items()}
    layer = HybridLayer(cfg_of(wl))
    Y = layer.forward(xg["q"], xg["k"], xg["v"], xg["gate_logits"], xg["W1"], xg["W2"])
    assert layer.check_status() == 0
    ref = O.vdn_layer({k: to_f64(t) for k, t in x.items()}, wl)
    assert rel_err(to_f64(Y), ref["Y"]) <= 2e-2


def test_non_positive_definite_frame_reports_numeric():
    wl = get_workload("small", B=1, H=1, T=12, N=64, seed=32)
    cfg = cfg_of(wl)
    G = -2.0 * torch.eye(wl.d, device="cuda").expand(1, 1, wl.T, wl.d, wl.d).contiguous()
    C = torch.zeros((1, 1, wl.T, wl.dv, wl.d), device="cuda")
    S_f = torch.empty((1, 1, cfg.nb, wl.dv, wl.d), device="cuda")
    S_b = torch.empty_like(S_f)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    vdn.vda_bidir_scan(cfg, G, C, S_f, S_b, _ws(cfg, vdn.VDN_WS_SCAN, "cuda"), status)
    assert vdn.vdn_read_status(status) == 6          # VDN_ERR_NUMERIC
