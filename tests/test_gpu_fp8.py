"""FP8 (e4m3) softmax branch through the C ABI, against the oracle.

* vdn_quantize_fp8 is compared bit for bit with the oracle's quantiser
  (codes and per-(b, h) scales): both take the rounding decision on the same
  fp32 quotient.
* vdn_softmax_window_fp8 is compared with the fp64 oracle run on the
  dequantised inputs (code * scale). What remains is the rounding of P to
  e4m3 before the P V product: each weight moves by at most 2^-4 of itself
  (3 mantissa bits) or 2^-10 below 2^-6, so |err| <= (2^-4 + 2^-9) max|v|
  whenever the row's weights sum to at least half the row length (true for
  these inputs, whose logits stay within a few units). That bound is
  checked, and so is the stated tolerance max|err| / max|ref| <= 6.25e-2
  (2^-4, tight enough to catch a wrong scale or layout; measured 3.4e-2).
* Against the oracle on the original inputs the quantisation of q, k and v
  adds its own 2^-4 per element: the stated tolerance there is 1.25e-1
  (2^-3; measured 5.8e-2 on o_sm).
"""
import numpy as np
import pytest
import torch

import oracle as O
from oracle.fp8 import dequantize_e4m3, quantize_e4m3
import softmax_attention_video_vdn_b200 as vdn
from softmax_attention_video_vdn_b200 import build as vbuild
from softmax_attention_video_vdn_b200.layer import HybridLayer
from synthetic import get_workload, make_inputs, to_f64
from tests.helpers import cfg_of, rel_err

pytestmark = pytest.mark.gpu

TOL_FP8 = 2.0 ** -4          # against the oracle on the dequantised inputs
TOL_FP8_INPUTS = 2.0 ** -3   # against the oracle on the original inputs
P_BOUND = 2.0 ** -4 + 2.0 ** -9


@pytest.fixture(scope="module", autouse=True)
def _library():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    vbuild.build()
    vdn.load_library()


def _quantize_gpu(cfg, x):
    x8 = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
    sc = torch.empty(cfg.B * cfg.H, dtype=torch.float32, device="cuda")
    ws = torch.empty(vdn.vdn_workspace_size(cfg, vdn.VDN_WS_QUANT), dtype=torch.uint8,
                     device="cuda")
    vdn.vdn_quantize_fp8(cfg, x, x8, sc, ws)
    torch.cuda.synchronize()
    return x8, sc


def test_quantize_matches_oracle_bit_for_bit():
    wl = get_workload("small", B=2, H=2, T=5, N=100, seed=21)
    x = make_inputs(wl, device="cuda")
    cfg = cfg_of(wl)
    x["q"][1, 1] = 0                      # a head of zeros: scale 1, codes 0
    x["v"][0, 1, :50] *= 1000             # wide range: subnormal codes elsewhere
    for name in ("q", "k", "v"):
        codes, sc = _quantize_gpu(cfg, x[name])
        ref_codes, ref_sc = quantize_e4m3(x[name].float().cpu().numpy())
        assert np.array_equal(sc.cpu().numpy(), ref_sc.reshape(-1)), name
        assert np.array_equal(codes.cpu().numpy(), ref_codes), name


MINI = {
    "ragged_tiles": dict(B=1, H=2, T=12, N=200, d_out=256, seed=31),
    "single_frame": dict(B=1, H=1, T=1, N=130, d_out=256, seed=32),
    "partial_last_block": dict(B=2, H=1, T=21, N=72, d_out=256, seed=33),
    "no_anchors": dict(B=1, H=1, T=16, N=128, anchors=0, d_out=256, seed=34),
    "context_tokens": dict(B=1, H=1, T=12, N=100, d_out=256, n_ctx=150, seed=35),
    "many_segments": dict(B=1, H=1, T=241, N=12, d_out=256, seed=36),
}


@pytest.mark.parametrize("name", list(MINI))
def test_fp8_softmax_against_dequantized_oracle(name):
    wl = get_workload("small", **MINI[name])
    x = make_inputs(wl, device="cuda")
    cfg = cfg_of(wl)
    q8, sq = _quantize_gpu(cfg, x["q"])
    k8, sk = _quantize_gpu(cfg, x["k"])
    v8, sv = _quantize_gpu(cfg, x["v"])
    o = torch.empty((cfg.B, cfg.L, cfg.H, cfg.dv), dtype=torch.bfloat16, device="cuda")
    sws = torch.empty(vdn.vdn_workspace_size(cfg, vdn.VDN_WS_SOFTMAX), dtype=torch.uint8,
                      device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    vdn.vdn_softmax_window_fp8(cfg, q8, k8, v8, sq, sk, sv, None, o, sws, status)
    assert vdn.vdn_read_status(status) == 0
    # the oracle on code * scale, codes from the oracle's own quantiser
    deq = {}
    for n in ("q", "k", "v"):
        c, s = quantize_e4m3(x[n].float().cpu().numpy())
        deq[n] = dequantize_e4m3(c, s)
    mask = O.frame_mask(wl.T, wl.block_frames, wl.window_blocks, wl.anchors)
    ref = np.zeros((cfg.B, cfg.H, cfg.L, cfg.dv))
    for b in range(cfg.B):
        for h in range(cfg.H):
            ref[b, h] = O.softmax_joint(deq["q"][b, h], deq["k"][b, h], deq["v"][b, h], wl.T,
                                        wl.N, wl.n_ctx, mask, 1.0 / np.sqrt(wl.d))
    got = to_f64(o).transpose(0, 2, 1, 3)
    err = np.abs(got - ref).max()
    assert err <= P_BOUND * np.abs(deq["v"]).max() + 2.0 ** -8 * np.abs(ref).max()
    assert rel_err(got, ref) <= TOL_FP8


def test_fp8_layer_against_oracle():
    wl = get_workload("small", B=1, H=2, T=12, N=200, d_out=256, beta=0.5, seed=41)
    x = make_inputs(wl, device="cuda")
    cfg = cfg_of(wl)
    layer = HybridLayer(cfg, fp8=True)
    Y = layer.forward(x["q"], x["k"], x["v"], x["gate_logits"], x["W1"], x["W2"])
    assert layer.check_status() == 0
    x64 = {n: to_f64(t) for n, t in x.items() if n in ("q", "k", "v", "gate_logits", "W1", "W2")}
    ref = O.vdn_layer(x64, wl)
    assert rel_err(to_f64(Y), ref["Y"]) <= TOL_FP8_INPUTS
    # the bf16 layer on the same inputs stays within the same distance
    Yb = HybridLayer(cfg).forward(x["q"], x["k"], x["v"], x["gate_logits"], x["W1"], x["W2"])
    assert rel_err(to_f64(Y), to_f64(Yb)) <= TOL_FP8_INPUTS
