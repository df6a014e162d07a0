"""The C-ABI library on the host: load, exports, window plan, validation.

No compute call reaches the GPU here: every call either is host-only
(vdn_window_plan, vdn_workspace_size, vdn_status_string) or is rejected by
argument validation before anything is launched.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
import softmax_attention_video_vdn_b200 as vdn
from softmax_attention_video_vdn_b200 import build as vbuild
from synthetic import WORKLOADS
from tests.helpers import cfg_of

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    vbuild.build()
    return vdn.load_library()


def _header_functions():
    src = open(os.path.join(ROOT, "include", "vdn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(v\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol(lib):
    names = _header_functions()
    assert set(names) == set(vdn.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(7):
        assert vdn.vdn_status_string(code)
    assert vdn.vdn_status_string(99) == "unknown status"


@pytest.mark.parametrize("T", [1, 2, 5, 6, 10, 11, 15, 16, 20, 40, 60, 61, 100, 101, 240])
@pytest.mark.parametrize("bf,W,anc", [(5, 1, 1), (5, 1, 0), (3, 2, 1), (4, 0, 1), (1, 1, 1)])
def test_window_plan_is_bit_exact(lib, T, bf, W, anc):
    cfg = vdn.make_config(B=1, H=1, T=T, N=1, d=128, dv=128, block_frames=bf, window_blocks=W,
                          anchors=anc)
    mask, plan = vdn.vdn_window_plan(cfg)
    m_ref, segs = O.window_plan(T, bf, W, anc)
    np.testing.assert_array_equal(mask, m_ref)
    np.testing.assert_array_equal(plan, O.serialize_plan(segs))


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_window_plan_of_each_workload(lib, name):
    wl = WORKLOADS[name]
    mask, plan = vdn.vdn_window_plan(cfg_of(wl))
    m_ref, segs = O.window_plan(wl.T, wl.block_frames, wl.window_blocks, wl.anchors)
    np.testing.assert_array_equal(mask, m_ref)
    np.testing.assert_array_equal(plan, O.serialize_plan(segs))


def test_window_plan_short_buffer(lib):
    cfg = vdn.make_config(B=1, H=1, T=60, N=1, d=128, dv=128)
    n = ctypes.c_size_t(3)
    buf = (ctypes.c_int32 * 3)()
    st = lib.vdn_window_plan(ctypes.byref(cfg), None, ctypes.cast(buf, ctypes.c_void_p),
                             ctypes.byref(n))
    assert st == 1 and n.value > 3


def _bad_cfgs():
    base = dict(B=1, H=2, T=20, N=64, d=128, dv=128, dtype="bf16", lam=1e-2, beta=0.5)
    yield "B0", dict(base, B=0), 1
    yield "T0", dict(base, T=0), 1
    yield "N0", dict(base, N=0), 1
    yield "d200", dict(base, d=200), 1
    yield "d12", dict(base, d=12, dtype="f32"), 1
    yield "lam0", dict(base, lam=0.0), 1
    yield "lam_neg", dict(base, lam=-1.0), 1
    yield "beta0", dict(base, beta=0.0), 1
    yield "beta2", dict(base, beta=1.5), 1
    yield "anchors2", dict(base, anchors=2), 1
    yield "bf0", dict(base, block_frames=0), 1
    yield "W-1", dict(base, window_blocks=-1), 1
    yield "bf16_d64", dict(base, d=64, dv=64), 2
    yield "f32_d24", dict(base, d=24, dv=24, dtype="f32"), 2
    yield "huge_L", dict(base, T=70000, N=40000), 2


@pytest.mark.parametrize("name,kw,code", list(_bad_cfgs()))
def test_validation_rejects_before_launch(lib, name, kw, code):
    cfg = vdn.make_config(**kw)
    fake = ctypes.c_void_p(0x1000)   # never dereferenced: validation fails first
    assert lib.vda_frame_stats(ctypes.byref(cfg), fake, fake, fake, fake, None) == code
    assert lib.vda_readout(ctypes.byref(cfg), fake, fake, fake, fake, None) == code
    assert lib.vda_readout_gated(ctypes.byref(cfg), fake, fake, fake, fake, fake, None) == code
    assert lib.vdn_workspace_size(ctypes.byref(cfg), vdn.VDN_WS_LAYER) == 0


def test_null_and_misaligned_pointers(lib):
    cfg = vdn.make_config(B=1, H=2, T=20, N=64, d=128, dv=128, dtype="bf16", d_out=256)
    ok = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1004)
    assert lib.vda_frame_stats(ctypes.byref(cfg), None, ok, ok, ok, None) == 1
    assert lib.vda_frame_stats(ctypes.byref(cfg), odd, ok, ok, ok, None) == 1
    assert lib.vda_bidir_scan(ctypes.byref(cfg), ok, ok, ok, ok, None, 0, None, None) == 4
    assert lib.vda_bidir_scan(ctypes.byref(cfg), ok, ok, ok, ok, ok, 16, None, None) == 4
    # S_fwd given without S_bwd / gate
    assert lib.vdn_softmax_window(ctypes.byref(cfg), ok, ok, ok, ok, None, None, ok, ok, 256,
                                  None, None) == 1
    assert lib.vdn_softmax_window(ctypes.byref(cfg), ok, ok, ok, ok, ok, None, ok, ok, 256,
                                  None, None) == 1
    # the gated readout needs the gate and all pointers aligned
    assert lib.vda_readout_gated(ctypes.byref(cfg), ok, ok, ok, None, ok, None) == 1
    assert lib.vda_readout_gated(ctypes.byref(cfg), ok, ok, ok, ok, odd, None) == 1
    assert lib.vdn_softmax_window(ctypes.byref(cfg), ok, ok, ok, None, None, None, ok, None, 0,
                                  None, None) == 4
    assert lib.vdn_gated_merge(ctypes.byref(cfg), ok, ok, None, ok, None) == 1
    assert lib.vdn_hybrid_forward(ctypes.byref(cfg), ok, ok, ok, ok, ok, ok, ok, ok, 16, None,
                                  None) == 4
    assert lib.vdn_read_status(None, None) == 1


def test_workspace_sizes(lib):
    wl = WORKLOADS["768p"]
    cfg = cfg_of(wl)
    frames = wl.B * wl.H * wl.T
    scan = vdn.vdn_workspace_size(cfg, vdn.VDN_WS_SCAN)
    assert scan >= frames * (wl.d * wl.d + wl.dv * wl.d) * 4
    layer = vdn.vdn_workspace_size(cfg, vdn.VDN_WS_LAYER)
    z = wl.B * wl.L * 2 * wl.H * wl.dv * 2
    assert layer >= scan + z + 2 * frames * wl.d * wl.d * 4
    assert vdn.vdn_workspace_size(cfg, 99) == 0


def test_fp8_entry_validation(lib):
    ok = ctypes.c_void_p(0x1000)
    cfg32 = vdn.make_config(B=1, H=2, T=20, N=64, d=128, dv=128, dtype="f32", d_out=256)
    assert lib.vdn_quantize_fp8(ctypes.byref(cfg32), ok, ok, ok, ok, 4096, None) == 2
    assert lib.vdn_softmax_window_fp8(ctypes.byref(cfg32), ok, ok, ok, ok, ok, ok, None, ok, ok,
                                      256, None, None) == 2
    assert lib.vdn_workspace_size(ctypes.byref(cfg32), vdn.VDN_WS_LAYER_FP8) == 0
    cfg = vdn.make_config(B=1, H=2, T=20, N=64, d=128, dv=128, dtype="bf16", d_out=256)
    assert lib.vdn_quantize_fp8(ctypes.byref(cfg), None, ok, ok, ok, 4096, None) == 1
    assert lib.vdn_quantize_fp8(ctypes.byref(cfg), ok, ok, ok, ok, 4, None) == 4
    assert lib.vdn_softmax_window_fp8(ctypes.byref(cfg), ok, ok, ok, None, ok, ok, None, ok, ok,
                                      256, None, None) == 1
    assert lib.vdn_softmax_window_fp8(ctypes.byref(cfg), ok, ok, ok, ok, ok, ok, None, ok, None,
                                      0, None, None) == 4
    # the FP8 layer needs room for the e4m3 copies of q, k, v on top of the layer's
    fp8 = lib.vdn_workspace_size(ctypes.byref(cfg), vdn.VDN_WS_LAYER_FP8)
    plain = lib.vdn_workspace_size(ctypes.byref(cfg), vdn.VDN_WS_LAYER)
    assert fp8 >= plain + 3 * 2 * 20 * 64 * 128
    assert lib.vdn_hybrid_forward_fp8(ctypes.byref(cfg), ok, ok, ok, ok, ok, ok, ok, ok, plain,
                                      None, None) == 4


def test_context_tokens_validation(lib):
    ok = ctypes.c_void_p(0x1000)
    bad = vdn.make_config(B=1, H=2, T=20, N=64, d=128, dv=128, dtype="bf16", n_ctx=-1)
    assert lib.vda_readout(ctypes.byref(bad), ok, ok, ok, ok, None) == 1
    f32 = vdn.make_config(B=1, H=2, T=20, N=64, d=64, dv=64, dtype="f32", n_ctx=8)
    assert lib.vda_readout(ctypes.byref(f32), ok, ok, ok, ok, None) == 2
    cfg = vdn.make_config(B=1, H=2, T=20, N=64, d=128, dv=128, dtype="bf16", d_out=256, n_ctx=100)
    assert cfg.L == 20 * 64 + 100
    plain = vdn.make_config(B=1, H=2, T=20, N=64, d=128, dv=128, dtype="bf16", d_out=256)
    # Z grows by the context rows: 2 * H * dv bf16 values each
    grow = (lib.vdn_workspace_size(ctypes.byref(cfg), vdn.VDN_WS_LAYER)
            - lib.vdn_workspace_size(ctypes.byref(plain), vdn.VDN_WS_LAYER))
    assert grow >= 100 * 2 * 2 * 128 * 2


def test_backward_entry_validation(lib):
    ok = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1004)
    f32 = vdn.make_config(B=1, H=2, T=20, N=64, d=64, dv=64, dtype="f32", d_out=256)
    cfg = vdn.make_config(B=1, H=2, T=20, N=64, d=128, dv=128, dtype="bf16", d_out=256)
    c32, c16 = ctypes.byref(f32), ctypes.byref(cfg)
    # the backward is built for the bf16 tensor-core configuration only
    for kind in (vdn.VDN_WS_SOFTMAX_BWD, vdn.VDN_WS_LINEAR_BWD, vdn.VDN_WS_BACKWARD):
        assert lib.vdn_workspace_size(c32, kind) == 0
        assert lib.vdn_workspace_size(c16, kind) > 0
    assert lib.vdn_softmax_window_lse(c32, ok, ok, ok, ok, ok, ok, 256, None, None) == 2
    assert lib.vdn_softmax_window_bwd(c32, *([ok] * 9), ok, 1 << 30, None, None) == 2
    assert lib.vda_linear_bwd(c32, *([ok] * 7), ok, 1 << 30, None, None) == 2
    assert lib.vdn_gated_merge_bwd(c32, *([ok] * 7), None, None) == 2
    assert lib.vdn_hybrid_forward_train(c32, *([ok] * 9), ok, 1 << 30, None, None) == 2
    assert lib.vdn_hybrid_backward(c32, *([ok] * 15), ok, 1 << 30, None, None) == 2
    # null, misaligned and short-workspace arguments are rejected before a launch
    assert lib.vdn_softmax_window_lse(c16, ok, ok, ok, ok, None, ok, 256, None, None) == 1
    assert lib.vdn_softmax_window_bwd(c16, *([ok] * 8), odd, ok, 1 << 30, None, None) == 1
    assert lib.vdn_softmax_window_bwd(c16, *([ok] * 9), ok, 8, None, None) == 4
    assert lib.vda_linear_bwd(c16, *([ok] * 6), None, ok, 1 << 30, None, None) == 1
    assert lib.vda_linear_bwd(c16, *([ok] * 7), ok, 64, None, None) == 4
    assert lib.vdn_gated_merge_bwd(c16, *([ok] * 6), None, None, None) == 1
    assert lib.vdn_hybrid_forward_train(c16, *([ok] * 8), None, ok, 1 << 30, None, None) == 1
    assert lib.vdn_hybrid_backward(c16, *([ok] * 15), ok, 64, None, None) == 4
    shared = vdn.make_config(B=1, H=2, T=20, N=64, d=128, dv=128, dtype="bf16", d_out=256,
                             w_per_head=1)
    assert lib.vdn_gated_merge_bwd(ctypes.byref(shared), *([ok] * 7), None, None) == 2


def test_backward_workspace_covers_its_buffers(lib):
    wl = WORKLOADS["768p"]
    cfg = cfg_of(wl)
    mat = 128 * 128 * 4
    frames = wl.B * wl.H * wl.T
    lin = vdn.vdn_workspace_size(cfg, vdn.VDN_WS_LINEAR_BWD)
    # nine per-frame matrices and the per-frame states and cotangents of both scans
    assert lin >= (9 + 4) * frames * mat
    rows = wl.B * wl.H * wl.L
    full = vdn.vdn_workspace_size(cfg, vdn.VDN_WS_BACKWARD)
    assert full >= lin + rows * (2 * 128 * 2 + 2 * 128 * 2 + 8)
    assert vdn.vdn_workspace_size(cfg, vdn.VDN_WS_SOFTMAX_BWD) >= rows * 8


@pytest.mark.parametrize("bf,W,anc", [(5, 1, 1), (5, 1, 0), (3, 2, 1), (4, 0, 1), (1, 1, 1),
                                      (2, 3, 0)])
def test_plan_mask_is_symmetric(lib, bf, W, anc):
    # The backward kernels use one plan for both directions: the key ranges of
    # a segment are also the ranges of the queries that see its keys. That
    # holds exactly when the library's frame mask is symmetric.
    for T in (1, 2, 7, 11, 16, 40, 61):
        cfg = vdn.make_config(B=1, H=1, T=T, N=1, d=128, dv=128, block_frames=bf,
                              window_blocks=W, anchors=anc)
        mask, plan = vdn.vdn_window_plan(cfg)
        np.testing.assert_array_equal(mask, mask.T)
        # every frame of a segment has that segment's row (segments are the
        # units the backward's key-outer kernel iterates over)
        i = 0
        while i < len(plan):
            q0, q1, nr = plan[i:i + 3]
            row = np.zeros(T, dtype=np.uint8)
            for r in range(nr):
                k0, k1 = plan[i + 3 + 2 * r:i + 5 + 2 * r]
                row[k0:k1] = 1
            for f in range(q0, q1):
                np.testing.assert_array_equal(mask[f], row)
                np.testing.assert_array_equal(mask[:, f], row)
            i += 3 + 2 * nr
