"""Python binding of the VDN hybrid attention layer's C ABI (libvdn.so).

Argument marshalling only: every function passes raw device pointers of
torch CUDA tensors, sizes and the current CUDA stream to the entry point of
the same name in ``include/vdn.h``; all arithmetic runs in the library's
sm_100a kernels. There is no fallback: if the shared library cannot be
loaded, every call raises.

Layouts (row-major): q, k [B,H,L,d]; v [B,H,L,dv]; G [B,H,T,d,d];
C [B,H,T,dv,d]; S_fwd, S_bwd [B,H,nb,dv,d]; o_lin, o_sm [B,L,H,dv];
Z [B,L,2,H,dv]; W1, W2 [H*dv, d_out] (or [dv, d_out] shared by heads);
Y [B,L,d_out] (or [B,L,H,d_out]). L = T*N, nb = ceil(T / block_frames).
"""
import ctypes
import math
import os

import numpy as np

__all__ = [
    "VdnConfig", "VDNError", "make_config", "load_library", "library_path",
    "vdn_window_plan", "vdn_workspace_size", "vda_frame_stats", "vda_bidir_scan",
    "vda_bidir_scan_noalloc", "vda_readout", "vda_readout_gated", "vdn_softmax_window",
    "vdn_gated_merge", "vdn_gated_merge_head_groups", "vdn_pack_head_groups",
    "vdn_hybrid_forward", "vdn_read_status", "vdn_quantize_fp8",
    "vdn_softmax_window_fp8", "vdn_hybrid_forward_fp8", "VDN_WS_QUANT", "VDN_WS_LAYER_FP8",
    "vdn_status_string", "vdn_last_error", "vdn_selftest_timeout", "EXPORTS",
    "VDN_F32", "VDN_BF16", "VDN_WS_SCAN", "VDN_WS_SOFTMAX", "VDN_WS_LAYER",
    "VDN_WS_SOFTMAX_BWD", "VDN_WS_LINEAR_BWD", "VDN_WS_BACKWARD", "vdn_softmax_window_lse",
    "vdn_softmax_window_bwd", "vda_linear_bwd", "vdn_gated_merge_bwd", "vdn_hybrid_forward_train",
    "vdn_hybrid_backward",
]

VDN_F32, VDN_BF16 = 0, 1
VDN_WS_SCAN, VDN_WS_SOFTMAX, VDN_WS_LAYER, VDN_WS_QUANT, VDN_WS_LAYER_FP8 = 1, 2, 3, 4, 5
VDN_WS_SOFTMAX_BWD, VDN_WS_LINEAR_BWD, VDN_WS_BACKWARD = 6, 7, 8
STATUS_NAMES = {0: "VDN_OK", 1: "VDN_ERR_INVALID_ARG", 2: "VDN_ERR_UNSUPPORTED",
                3: "VDN_ERR_CUDA", 4: "VDN_ERR_WORKSPACE", 5: "VDN_ERR_TIMEOUT",
                6: "VDN_ERR_NUMERIC"}

# Every symbol declared in include/vdn.h.
EXPORTS = ("vdn_window_plan", "vdn_workspace_size", "vda_frame_stats", "vda_bidir_scan",
           "vda_bidir_scan_noalloc", "vda_readout", "vda_readout_gated", "vdn_softmax_window",
           "vdn_gated_merge", "vdn_gated_merge_head_groups", "vdn_pack_head_groups",
           "vdn_hybrid_forward",
           "vdn_read_status", "vdn_status_string",
           "vdn_last_error", "vdn_selftest_timeout", "vdn_quantize_fp8",
           "vdn_softmax_window_fp8", "vdn_hybrid_forward_fp8", "vdn_softmax_window_lse",
           "vdn_softmax_window_bwd", "vda_linear_bwd", "vdn_gated_merge_bwd",
           "vdn_hybrid_forward_train", "vdn_hybrid_backward")

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path():
    return os.environ.get("VDN_LIBRARY", os.path.join(_HERE, "libvdn.so"))


class VdnConfig(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("T", ctypes.c_int32),
                ("N", ctypes.c_int32), ("d", ctypes.c_int32), ("dv", ctypes.c_int32),
                ("block_frames", ctypes.c_int32), ("window_blocks", ctypes.c_int32),
                ("anchors", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("lambda_", ctypes.c_float), ("beta", ctypes.c_float),
                ("softmax_scale", ctypes.c_float), ("d_out", ctypes.c_int32),
                ("w_per_head", ctypes.c_int32), ("n_ctx", ctypes.c_int32)]

    @property
    def L(self):
        """Tokens per (b, h): the T*N video tokens, then the context tokens."""
        return self.T * self.N + self.n_ctx

    @property
    def nb(self):
        return -(-self.T // self.block_frames)


def make_config(B, H, T, N, d, dv, dtype="bf16", lam=1e-2, beta=1.0, block_frames=5,
                window_blocks=1, anchors=1, softmax_scale=0.0, d_out=0, w_per_head=0, n_ctx=0):
    c = VdnConfig()
    c.B, c.H, c.T, c.N, c.d, c.dv = B, H, T, N, d, dv
    c.block_frames, c.window_blocks, c.anchors = block_frames, window_blocks, int(anchors)
    c.dtype = {"f32": VDN_F32, "bf16": VDN_BF16}[dtype] if isinstance(dtype, str) else int(dtype)
    c.lambda_, c.beta, c.softmax_scale = lam, beta, softmax_scale
    c.d_out, c.w_per_head, c.n_ctx = d_out, w_per_head, n_ctx
    return c


class VDNError(RuntimeError):
    def __init__(self, name, status):
        self.status = status
        detail = vdn_status_string(status) if _LIB else "library not loaded"
        if status == 3 and _LIB:
            detail += "; " + vdn_last_error()
        super().__init__(f"{name}: {STATUS_NAMES.get(status, status)} ({detail})")


_LIB = None


def load_library(path=None):
    """Load libvdn.so (raises OSError if it is missing)."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    lib = ctypes.CDLL(path or library_path())
    P, Z, I32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    cfgp = ctypes.POINTER(VdnConfig)
    sig = {
        "vdn_window_plan": (I32, [cfgp, P, P, ctypes.POINTER(ctypes.c_size_t)]),
        "vdn_workspace_size": (Z, [cfgp, I32]),
        "vda_frame_stats": (I32, [cfgp, P, P, P, P, P]),
        "vda_bidir_scan": (I32, [cfgp, P, P, P, P, P, Z, P, P]),
        "vda_bidir_scan_noalloc": (I32, [cfgp, P, P, P, P, P, P]),
        "vda_readout": (I32, [cfgp, P, P, P, P, P]),
        "vda_readout_gated": (I32, [cfgp, P, P, P, P, P, P]),
        "vdn_quantize_fp8": (I32, [cfgp, P, P, P, P, Z, P]),
        "vdn_softmax_window_fp8": (I32, [cfgp, P, P, P, P, P, P, P, P, P, Z, P, P]),
        "vdn_hybrid_forward_fp8": (I32, [cfgp, P, P, P, P, P, P, P, P, Z, P, P]),
        "vdn_softmax_window": (I32, [cfgp, P, P, P, P, P, P, P, P, Z, P, P]),
        "vdn_gated_merge": (I32, [cfgp, P, P, P, P, P]),
        "vdn_gated_merge_head_groups": (I32, [cfgp, I32, P, P, P, P, P]),
        "vdn_pack_head_groups": (I32, [cfgp, I32, P, P, P]),
        "vdn_hybrid_forward": (I32, [cfgp, P, P, P, P, P, P, P, P, Z, P, P]),
        "vdn_softmax_window_lse": (I32, [cfgp, P, P, P, P, P, P, Z, P, P]),
        "vdn_softmax_window_bwd": (I32, [cfgp] + [P] * 9 + [P, Z, P, P]),
        "vda_linear_bwd": (I32, [cfgp] + [P] * 7 + [P, Z, P, P]),
        "vdn_gated_merge_bwd": (I32, [cfgp] + [P] * 7 + [P, P]),
        "vdn_hybrid_forward_train": (I32, [cfgp] + [P] * 9 + [P, Z, P, P]),
        "vdn_hybrid_backward": (I32, [cfgp] + [P] * 15 + [P, Z, P, P]),
        "vdn_read_status": (I32, [P, P]),
        "vdn_selftest_timeout": (I32, [P, I32, P]),
        "vdn_status_string": (ctypes.c_char_p, [I32]),
        "vdn_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    if path is None:
        _LIB = lib
    return lib


def _lib():
    return _LIB if _LIB is not None else load_library()


def vdn_status_string(status):
    return _lib().vdn_status_string(int(status)).decode()


def vdn_last_error():
    return _lib().vdn_last_error().decode()


def _ptr(t):
    """Device pointer of a contiguous CUDA tensor, or NULL for None."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _call(name, *args):
    status = getattr(_lib(), name)(*args)
    if status != 0:
        raise VDNError(name, status)


# ---------------------------------------------------------------- host calls
def vdn_window_plan(cfg):
    """(mask uint8 [T, T], plan int32 [n]) computed by the library (host)."""
    n = ctypes.c_size_t(0)
    _call("vdn_window_plan", ctypes.byref(cfg), None, None, ctypes.byref(n))
    mask = np.zeros((cfg.T, cfg.T), dtype=np.uint8)
    plan = np.zeros(n.value, dtype=np.int32)
    _call("vdn_window_plan", ctypes.byref(cfg), mask.ctypes.data_as(ctypes.c_void_p),
          plan.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n))
    return mask, plan[:n.value]


def vdn_workspace_size(cfg, kind):
    return int(_lib().vdn_workspace_size(ctypes.byref(cfg), int(kind)))


# -------------------------------------------------------------- device calls
def vda_frame_stats(cfg, k, v, G, C, stream=None):
    _call("vda_frame_stats", ctypes.byref(cfg), _ptr(k), _ptr(v), _ptr(G), _ptr(C), _stream(stream))


def vda_bidir_scan(cfg, G, C, S_fwd, S_bwd, ws, dev_status, stream=None):
    _call("vda_bidir_scan", ctypes.byref(cfg), _ptr(G), _ptr(C), _ptr(S_fwd), _ptr(S_bwd),
          _ptr(ws), ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream))


def vda_bidir_scan_noalloc(cfg, G, C, S_fwd, S_bwd, dev_status, stream=None):
    """vda_bidir_scan with the library's own fixed scratch (no workspace)."""
    _call("vda_bidir_scan_noalloc", ctypes.byref(cfg), _ptr(G), _ptr(C), _ptr(S_fwd),
          _ptr(S_bwd), _ptr(dev_status), _stream(stream))


def vda_readout(cfg, q, S_fwd, S_bwd, o_lin, stream=None):
    _call("vda_readout", ctypes.byref(cfg), _ptr(q), _ptr(S_fwd), _ptr(S_bwd), _ptr(o_lin),
          _stream(stream))


def vda_readout_gated(cfg, q, S_fwd, S_bwd, gate_logits, Z, stream=None):
    _call("vda_readout_gated", ctypes.byref(cfg), _ptr(q), _ptr(S_fwd), _ptr(S_bwd),
          _ptr(gate_logits), _ptr(Z), _stream(stream))


def vdn_softmax_window(cfg, q, k, v, S_fwd, S_bwd, gate_logits, out, ws, dev_status, stream=None):
    _call("vdn_softmax_window", ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(S_fwd),
          _ptr(S_bwd), _ptr(gate_logits), _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
          _ptr(dev_status), _stream(stream))


def vdn_quantize_fp8(cfg, x, x8, scale, ws, stream=None):
    _call("vdn_quantize_fp8", ctypes.byref(cfg), _ptr(x), _ptr(x8), _ptr(scale), _ptr(ws),
          ws.numel() * ws.element_size(), _stream(stream))


def vdn_softmax_window_fp8(cfg, q8, k8, v8, q_scale, k_scale, v_scale, gate_logits, out, ws,
                           dev_status, stream=None):
    _call("vdn_softmax_window_fp8", ctypes.byref(cfg), _ptr(q8), _ptr(k8), _ptr(v8),
          _ptr(q_scale), _ptr(k_scale), _ptr(v_scale), _ptr(gate_logits), _ptr(out), _ptr(ws),
          ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream))


def vdn_hybrid_forward_fp8(cfg, q, k, v, gate_logits, W1, W2, Y, ws, dev_status, stream=None):
    _call("vdn_hybrid_forward_fp8", ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v),
          _ptr(gate_logits), _ptr(W1), _ptr(W2), _ptr(Y), _ptr(ws),
          ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream))


def vdn_gated_merge(cfg, Z, W1, W2, Y, stream=None):
    _call("vdn_gated_merge", ctypes.byref(cfg), _ptr(Z), _ptr(W1), _ptr(W2), _ptr(Y),
          _stream(stream))


def vdn_gated_merge_head_groups(cfg, n_groups, Z, W1, W2, Y, stream=None):
    """Merge for Z [B, n_groups, Ls, 2, H/n_groups, dv] (head groups received
    from the ranks of a head-sharded layer); Y [B, Ls, d_out]."""
    _call("vdn_gated_merge_head_groups", ctypes.byref(cfg), int(n_groups), _ptr(Z), _ptr(W1),
          _ptr(W2), _ptr(Y), _stream(stream))


def vdn_pack_head_groups(cfg, n_groups, x, out, stream=None):
    """x [B, Ls, H, 128] -> out [B, H/n_groups, n_groups, Ls, 128] (bf16)."""
    _call("vdn_pack_head_groups", ctypes.byref(cfg), int(n_groups), _ptr(x), _ptr(out),
          _stream(stream))


def vdn_hybrid_forward(cfg, q, k, v, gate_logits, W1, W2, Y, ws, dev_status, stream=None):
    _call("vdn_hybrid_forward", ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(gate_logits),
          _ptr(W1), _ptr(W2), _ptr(Y), _ptr(ws), ws.numel() * ws.element_size(),
          _ptr(dev_status), _stream(stream))


def _nbytes(t):
    return t.numel() * t.element_size()


# ----------------------------------------------------------------- backward
def vdn_softmax_window_lse(cfg, q, k, v, o_sm, lse, ws, dev_status, stream=None):
    _call("vdn_softmax_window_lse", ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(o_sm),
          _ptr(lse), _ptr(ws), _nbytes(ws), _ptr(dev_status), _stream(stream))


def vdn_softmax_window_bwd(cfg, q, k, v, o_sm, lse, do_sm, dq, dk, dv, ws, dev_status,
                           stream=None):
    _call("vdn_softmax_window_bwd", ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(o_sm),
          _ptr(lse), _ptr(do_sm), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), _nbytes(ws),
          _ptr(dev_status), _stream(stream))


def vda_linear_bwd(cfg, q, k, v, do_lin, dq, dk, dv, ws, dev_status, stream=None):
    _call("vda_linear_bwd", ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(do_lin), _ptr(dq),
          _ptr(dk), _ptr(dv), _ptr(ws), _nbytes(ws), _ptr(dev_status), _stream(stream))


def vdn_gated_merge_bwd(cfg, Z, W1, W2, dY, dZ, dW1, dW2, dev_status, stream=None):
    _call("vdn_gated_merge_bwd", ctypes.byref(cfg), _ptr(Z), _ptr(W1), _ptr(W2), _ptr(dY),
          _ptr(dZ), _ptr(dW1), _ptr(dW2), _ptr(dev_status), _stream(stream))


def vdn_hybrid_forward_train(cfg, q, k, v, gate_logits, W1, W2, Y, Z, lse, ws, dev_status,
                             stream=None):
    _call("vdn_hybrid_forward_train", ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v),
          _ptr(gate_logits), _ptr(W1), _ptr(W2), _ptr(Y), _ptr(Z), _ptr(lse), _ptr(ws),
          _nbytes(ws), _ptr(dev_status), _stream(stream))


def vdn_hybrid_backward(cfg, q, k, v, gate_logits, W1, W2, Z, lse, dY, dq, dk, dv, dgate_logits,
                        dW1, dW2, ws, dev_status, stream=None):
    _call("vdn_hybrid_backward", ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(gate_logits),
          _ptr(W1), _ptr(W2), _ptr(Z), _ptr(lse), _ptr(dY), _ptr(dq), _ptr(dk), _ptr(dv),
          _ptr(dgate_logits), _ptr(dW1), _ptr(dW2), _ptr(ws), _nbytes(ws), _ptr(dev_status),
          _stream(stream))


def vdn_selftest_timeout(dev_status, limit_ms, stream=None):
    """Launch the bounded-wait self-test (its wait never completes)."""
    _call("vdn_selftest_timeout", _ptr(dev_status), int(limit_ms), _stream(stream))


def vdn_read_status(dev_status, stream=None):
    """Synchronise, read and clear the device status word; returns the code."""
    return int(_lib().vdn_read_status(_ptr(dev_status), _stream(stream)))


def default_scale(cfg):
    return cfg.softmax_scale if cfg.softmax_scale > 0 else 1.0 / math.sqrt(cfg.d)
