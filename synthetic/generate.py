"""Seeded input generator.

Draw order (fixed, so a seed names one input set): q, k, v, gate_logits, W1,
W2, then the structure draws of the key distribution. Every draw is N(0, 1)
unless stated. Layout of q, k, v is [B, H, T*N, d] row-major (token index
f*N + n, n the row-major position in the spatial grid).

Keys are L2-normalised per token in fp32 and then rounded to the workload's
dtype (bf16 round-to-nearest-even), so both the oracle and the CUDA path see
exactly the same stored values. W1, W2 ~ N(0, 1/fan_in) with fan_in = the
rows of W (dv when shared by heads, H*dv otherwise).

Key distributions:
  gauss          k ~ N(0, 1)
  student_t      k ~ Student-t(nu) elementwise, drawn as z / sqrt(chi2_nu / nu)
                 with chi2_nu a sum of nu squared normals (integer nu)
  rank_deficient a seeded choice of floor(frac*T) frames (shared by every
                 (b, h)); for each (b, h, f) of them a random orthonormal
                 d x r basis U (QR of a Gaussian) and k = z U^T, z ~ N(0, I_r)

Generation runs on any torch device with a torch.Generator seeded by the
workload's seed; values drawn on CPU and on CUDA differ, so every comparison
uses one input set copied to wherever it is needed.
"""
import numpy as np
import torch

_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _randn(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def make_inputs(wl, device="cpu"):
    """Return a dict of torch tensors on `device` for workload `wl`.

    Keys: q, k, v ([B,H,L,d] / [B,H,L,dv], dtype of the workload), gate_logits
    ([H] fp32), W1, W2 (dtype of the workload; absent when wl.d_out == 0),
    and for rank-deficient keys the sorted frame indices (deficient_frames).
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    H = wl.H
    B, T, N, d, dv = wl.B, wl.T, wl.N, wl.d, wl.dv
    L = wl.L      # T * N video tokens, then wl.n_ctx context tokens
    dt = _DT[wl.dtype]

    q = _randn((B, H, L, d), gen, dev)
    if wl.keys == "student_t":
        nu = int(wl.extra.get("nu", 3))
        z = _randn((B, H, L, d), gen, dev)
        chi2 = torch.zeros_like(z)
        for _ in range(nu):
            chi2.add_(_randn((B, H, L, d), gen, dev).square_())
        k = z / torch.sqrt(chi2 / nu)
        del z, chi2
    else:
        k = _randn((B, H, L, d), gen, dev)
    v = _randn((B, H, L, dv), gen, dev)
    gate = _randn((H,), gen, dev)
    out = {}
    if wl.d_out:
        fan_in = dv if wl.w_per_head else H * dv
        rows = dv if wl.w_per_head else H * dv
        W1 = _randn((rows, wl.d_out), gen, dev) / np.sqrt(fan_in)
        W2 = _randn((rows, wl.d_out), gen, dev) / np.sqrt(fan_in)
        out["W1"] = W1.to(dt)
        out["W2"] = W2.to(dt)

    if wl.keys == "rank_deficient":
        if wl.n_ctx:
            raise ValueError("rank-deficient frames are drawn for video-only sequences")
        frac = float(wl.extra.get("deficient_frac", 0.1))
        r = int(wl.extra.get("rank", 16))
        n_def = int(np.floor(frac * T))
        frames = torch.randperm(T, generator=gen, device=dev)[:n_def].sort().values
        kv = k.view(B, H, T, N, d)
        for f in frames.tolist():
            U, _ = torch.linalg.qr(_randn((B, H, d, r), gen, dev))
            zz = _randn((B, H, N, r), gen, dev)
            kv[:, :, f] = zz @ U.transpose(-1, -2)
        out["deficient_frames"] = frames.cpu()

    k = k / torch.linalg.vector_norm(k, dim=-1, keepdim=True)
    out.update(q=q.to(dt), k=k.to(dt), v=v.to(dt), gate_logits=gate)
    return out


def to_f64(t):
    """Exact fp64 numpy copy of a (CPU or CUDA) tensor's stored values."""
    return t.detach().to("cpu", torch.float64).numpy()
