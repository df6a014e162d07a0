"""vda_bidir_scan_noalloc: the scan for callers that cannot allocate device
memory at call time (code inside another framework's allocator or plugin
hook, real-time loops that forbid allocation). It must give the same states
as vda_bidir_scan with a caller workspace, on consecutive calls that share
the library's scratch array.

This file is collected last so that a failure here leaves every other test
already run; it passes alone in a fresh process and after the other tests.
"""
import ctypes

import pytest
import torch

import softmax_attention_video_vdn_b200 as vdn
from softmax_attention_video_vdn_b200 import build as vbuild
from softmax_attention_video_vdn_b200.layer import _ws
from synthetic import get_workload, make_inputs
from tests.helpers import cfg_of, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    vbuild.build()
    vdn.load_library()


def _stats(cfg, x):
    G = torch.empty((cfg.B, cfg.H, cfg.T, cfg.d, cfg.d), dtype=torch.float32, device="cuda")
    C = torch.empty((cfg.B, cfg.H, cfg.T, cfg.dv, cfg.d), dtype=torch.float32, device="cuda")
    vdn.vda_frame_stats(cfg, x["k"], x["v"], G, C)
    return G, C


@pytest.mark.parametrize("name,over", [
    ("small", dict(B=1, H=2, T=40, N=300, seed=21)),     # 80 frames of 128-dim maps
    ("tiny", dict()),                                    # fp32, d = dv = 64
])
def test_noalloc_scan_matches_workspace_scan(name, over):
    wl = get_workload(name, **over)
    cfg = cfg_of(wl)
    x = {k: (t.cuda() if torch.is_tensor(t) else t) for k, t in make_inputs(wl).items()}
    G, C = _stats(cfg, x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref_f = torch.empty((cfg.B, cfg.H, cfg.nb, cfg.dv, cfg.d), dtype=torch.float32, device="cuda")
    ref_b = torch.empty_like(ref_f)
    vdn.vda_bidir_scan(cfg, G, C, ref_f, ref_b, _ws(cfg, vdn.VDN_WS_SCAN, "cuda"), status)
    for call in range(2):   # two calls in a row share the scratch array
        S_f = torch.full_like(ref_f, float("nan"))
        S_b = torch.full_like(ref_b, float("nan"))
        vdn.vda_bidir_scan_noalloc(cfg, G, C, S_f, S_b, status)
        assert vdn.vdn_read_status(status) == 0
        assert rel_err(S_f.double().cpu(), ref_f.double().cpu()) <= 1e-3, call
        assert rel_err(S_b.double().cpu(), ref_b.double().cpu()) <= 1e-3, call


def test_noalloc_scan_rejects_shapes_beyond_its_scratch():
    lib = vdn.load_library()
    cfg = cfg_of(get_workload("small"))          # 8 x 40 = 320 frames of 128-dim maps
    fake = ctypes.c_void_p(0x1000)               # rejected before any device access
    st = lib.vda_bidir_scan_noalloc(ctypes.byref(cfg), fake, fake, fake, fake, None, None)
    assert st == 4
    assert "holds" in vdn.vdn_last_error()
