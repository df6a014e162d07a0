"""Shared test helpers: workload -> C config, error metric, input copies."""
import numpy as np

import softmax_attention_video_vdn_b200 as vdn

TOL = {"f32": 1e-4, "bf16": 2e-2}   # max |err| / max |ref|


def cfg_of(wl, **over):
    kw = dict(B=wl.B, H=wl.H, T=wl.T, N=wl.N, d=wl.d, dv=wl.dv, dtype=wl.dtype, lam=wl.lam,
              beta=wl.beta, block_frames=wl.block_frames, window_blocks=wl.window_blocks,
              anchors=wl.anchors, d_out=wl.d_out, w_per_head=wl.w_per_head,
              n_ctx=getattr(wl, "n_ctx", 0))
    kw.update(over)
    return vdn.make_config(**kw)


def rel_err(got, ref):
    """max |got - ref| / max |ref| (0 when both are zero)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    den = np.abs(ref).max()
    num = np.abs(got - ref).max()
    if den == 0:
        return float(num)
    return float(num / den)
