"""Backward pass of the VDN hybrid layer: a plain, slow, fp64 NumPy reference.

TEST INFRASTRUCTURE ONLY: tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` may use it; the product path may not.

The pages train this layer (mlsanity abstract and the flyP critical read:
stage-1 layer-wise alignment fits the hybrid layer to the softmax layer it
replaces) but print no gradient formula. Every function here is therefore the
derivative of the forward pass in ``vdn_oracle`` taken literally, step by step
in reverse order (reverse-mode differentiation by hand), with no algebraic
shortcut that the forward does not state:

* merge: Y = sum_h g_h o_sm,h W1_h + (1 - g_h) o_lin,h W2_h, g_h = sigmoid(logit_h);
* softmax: P = softmax(scale q k^T over the allowed keys), o_sm = P v;
* linear branch: G_f = K_f^T K_f, C_f = V_f^T K_f, M_f = (G_f + lambda I)^-1,
  A_f = I - beta G_f M_f, B_f = beta C_f M_f, the forward and backward scans
  S <- S A_f + B_f, o_lin = (S_fwd(b) + S_bwd(b)) q.

The loss is L = <dY, Y> for a given output cotangent dY; every function
returns the cotangents of its inputs. Pins: finite differences of the
forward oracle in fp64 and, for the softmax part, PyTorch's autograd of its
own attention routine (tests/test_oracle_backward.py).
"""
import numpy as np
import scipy.linalg

from .vdn_oracle import _is_anchor, frame_stats, sigmoid, vdn_layer, window_bounds, window_plan

__all__ = ["softmax_window_bwd", "softmax_window_bwd_dq_rows", "linear_branch_bwd", "gated_merge_bwd", "vdn_layer_bwd",
           "ridge_inverse", "softmax_row_lse2"]


# ------------------------------------------------------------ softmax branch
def _softmax_rows_bwd(qr, k, v, dor, cols, scale, dq, dk, dv, rows):
    """Backward of softmax(scale qr k[cols]^T) v[cols] for one set of query rows
    that share the key set `cols`; accumulates into dq[rows], dk[cols], dv[cols]."""
    s = (qr @ k[cols].T) * scale
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    dp = dor @ v[cols].T                               # dL/dP
    ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))  # softmax Jacobian, row by row
    dq[rows] += scale * (ds @ k[cols])
    dk[cols] += scale * (ds.T @ qr)
    dv[cols] += p.T @ dor


def softmax_window_bwd(q, k, v, do, T, N, n_ctx, mask, scale):
    """Cotangents of q, k, v for the softmax branch of one (b, h).

    Same key sets as the forward (``softmax_window`` / ``softmax_joint``): the
    queries of video frame f attend the key frames of mask row f and the
    context tokens; context queries attend every token. q, k, do: [L, d|dv],
    L = T*N + n_ctx. Returns dq, dk, dv.
    """
    L = q.shape[0]
    TN = T * N
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    ctx = np.arange(TN, TN + n_ctx)
    for f in range(T):
        cols = np.concatenate([np.arange(j * N, (j + 1) * N) for j in np.nonzero(mask[f])[0]]
                              + [ctx])
        rows = np.arange(f * N, (f + 1) * N)
        _softmax_rows_bwd(q[rows], k, v, do[rows], cols, scale, dq, dk, dv, rows)
    if n_ctx:
        _softmax_rows_bwd(q[TN:], k, v, do[TN:], np.arange(L), scale, dq, dk, dv,
                          np.arange(TN, L))
    return dq, dk, dv


def softmax_window_bwd_dq_rows(rows, q, k, v, do_rows, N, mask, scale):
    """dq of the softmax branch at selected video query rows only (sampled
    rows of a large case; no context tokens). A row's dq depends only on its
    own cotangent and its own key set, so rows of one query frame are done
    together, exactly as ``softmax_window_bwd`` does them. do_rows: [len(rows),
    dv] cotangents of o_sm at those rows. Returns [len(rows), d]."""
    rows = np.asarray(rows)
    out = np.zeros((len(rows), q.shape[1]))
    dk, dv = np.zeros_like(k), np.zeros_like(v)      # not needed here
    frames = rows // N
    for f in np.unique(frames):
        sel = np.nonzero(frames == f)[0]
        cols = np.concatenate([np.arange(j * N, (j + 1) * N) for j in np.nonzero(mask[f])[0]])
        _softmax_rows_bwd(q[rows[sel]], k, v, do_rows[sel], cols, scale, out, dk, dv, sel)
    return out


def softmax_row_lse2(q, k, T, N, n_ctx, mask, scale):
    """log2 of sum_j exp(scale q_i . k_j) over each row's allowed keys (the
    softmax normaliser in base 2, as the backward's saved row statistic)."""
    L = q.shape[0]
    TN = T * N
    out = np.zeros(L)
    ctx = np.arange(TN, TN + n_ctx)
    for f in range(T):
        cols = np.concatenate([np.arange(j * N, (j + 1) * N) for j in np.nonzero(mask[f])[0]]
                              + [ctx])
        s = (q[f * N:(f + 1) * N] @ k[cols].T) * scale
        m = s.max(axis=1)
        out[f * N:(f + 1) * N] = (m + np.log(np.exp(s - m[:, None]).sum(axis=1))) / np.log(2.0)
    if n_ctx:
        s = (q[TN:] @ k.T) * scale
        m = s.max(axis=1)
        out[TN:] = (m + np.log(np.exp(s - m[:, None]).sum(axis=1))) / np.log(2.0)
    return out


# ------------------------------------------------------------- linear branch
def ridge_inverse(Gf, lam):
    """M_f = (G_f + lambda I)^-1 from a Cholesky factor, as the forward solve."""
    d = Gf.shape[0]
    eye = np.eye(d)
    Lc = np.linalg.cholesky(Gf + lam * eye)
    Linv = scipy.linalg.solve_triangular(Lc, eye, lower=True)
    return Linv.T @ Linv


def linear_branch_bwd(q, k, v, do_lin, T, N, lam, beta, block_frames=5, window_blocks=1,
                      anchors=1):
    """Cotangents of q, k, v for the linear branch of one (b, h) (video tokens).

    Steps, reverse of the forward:
      readout   o_t = (S_fwd(b) + S_bwd(b)) q_t:  dq_t = (S_fwd + S_bwd)^T do_t,
                dS_fwd(b) = dS_bwd(b) = sum_t do_t q_t^T over the block's
                non-anchor tokens;
      scans     X' = X A_f + B_f:  dA_f += X^T dX', dB_f += dX', dX = dX' A_f^T,
                with each block state's cotangent added where the forward
                read it;
      solve     A_f = I - beta G_f M_f, B_f = beta C_f M_f, M_f = (G_f + lam I)^-1:
                dM = -beta G^T dA + beta C^T dB, dG = -beta dA M^T - M^T dM M^T,
                dC = beta dB M^T;
      stats     dK_f = K_f (dG + dG^T) + V_f dC, dV_f = K_f dC^T.
    q, k: [T*N, d], v, do_lin: [T*N, dv]. Returns dq, dk, dv and the
    per-frame cotangents (dG, dC) for inspection.
    """
    d, dv_ = k.shape[1], v.shape[1]
    G, C = frame_stats(k, v, T, N)
    eye = np.eye(d)
    M = np.zeros((T, d, d))
    A = np.zeros((T, d, d))
    Bm = np.zeros((T, dv_, d))
    for f in range(T):
        if _is_anchor(f, T, anchors):
            continue
        M[f] = ridge_inverse(G[f], lam)
        A[f] = eye - beta * (G[f] @ M[f])
        Bm[f] = beta * (C[f] @ M[f])
    # forward states, kept per frame (the forward oracle's scans)
    fwd_after = np.zeros((T, dv_, d))
    S = np.zeros((dv_, d))
    for f in range(T):
        if not _is_anchor(f, T, anchors):
            S = S @ A[f] + Bm[f]
        fwd_after[f] = S
    bwd_after = np.zeros((T, dv_, d))
    S = np.zeros((dv_, d))
    for f in range(T - 1, -1, -1):
        if not _is_anchor(f, T, anchors):
            S = S @ A[f] + Bm[f]
        bwd_after[f] = S
    nb = -(-T // block_frames)
    S_fwd = np.zeros((nb, dv_, d))
    S_bwd = np.zeros((nb, dv_, d))
    inj_f = np.zeros((T, dv_, d))    # cotangent entering fwd_after[f]
    inj_b = np.zeros((T, dv_, d))    # cotangent entering bwd_after[f]
    win = [window_bounds(b, T, block_frames, window_blocks) for b in range(nb)]
    for b, (ws, we) in enumerate(win):
        if ws >= 1:
            S_fwd[b] = fwd_after[ws - 1]
        if we <= T - 1:
            S_bwd[b] = bwd_after[we]

    # readout
    dq = np.zeros_like(q)
    dS = np.zeros((nb, dv_, d))      # cotangent of S_fwd(b) (= that of S_bwd(b))
    for f in range(T):
        if _is_anchor(f, T, anchors):
            continue
        b = f // block_frames
        rows = slice(f * N, (f + 1) * N)
        dq[rows] += do_lin[rows] @ (S_fwd[b] + S_bwd[b])
        dS[b] += do_lin[rows].T @ q[rows]
    for b, (ws, we) in enumerate(win):
        if ws >= 1:
            inj_f[ws - 1] += dS[b]
        if we <= T - 1:
            inj_b[we] += dS[b]

    # scans in reverse
    dA = np.zeros((T, d, d))
    dB = np.zeros((T, dv_, d))
    g = np.zeros((dv_, d))
    for f in range(T - 1, -1, -1):
        g = g + inj_f[f]                       # dL / d fwd_after[f]
        if not _is_anchor(f, T, anchors):
            prev = fwd_after[f - 1] if f >= 1 else np.zeros((dv_, d))
            dA[f] += prev.T @ g
            dB[f] += g
            g = g @ A[f].T
    h = np.zeros((dv_, d))
    for f in range(T):
        h = h + inj_b[f]                       # dL / d bwd_after[f]
        if not _is_anchor(f, T, anchors):
            nxt = bwd_after[f + 1] if f + 1 <= T - 1 else np.zeros((dv_, d))
            dA[f] += nxt.T @ h
            dB[f] += h
            h = h @ A[f].T

    # solve and stats
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dG_all = np.zeros((T, d, d))
    dC_all = np.zeros((T, dv_, d))
    for f in range(T):
        if _is_anchor(f, T, anchors):
            continue
        dM = -beta * (G[f].T @ dA[f]) + beta * (C[f].T @ dB[f])
        dG = -beta * (dA[f] @ M[f].T) - M[f].T @ dM @ M[f].T
        dC = beta * (dB[f] @ M[f].T)
        rows = slice(f * N, (f + 1) * N)
        Kf, Vf = k[rows], v[rows]
        dk[rows] += Kf @ (dG + dG.T) + Vf @ dC
        dv[rows] += Kf @ dC.T
        dG_all[f], dC_all[f] = dG, dC
    return dict(dq=dq, dk=dk, dv=dv, dG=dG_all, dC=dC_all, dS=dS, dA=dA, dB=dB)


# ---------------------------------------------------------------------- merge
def gated_merge_bwd(o_sm, o_lin, gate_logits, W1, W2, dY, w_per_head=0):
    """Cotangents of o_sm, o_lin, the gate logits and W1, W2 for
    ``vdn_oracle.gated_merge``. o_sm, o_lin: [B, H, L, dv]; dY as Y."""
    B, H, L, dv = o_sm.shape
    g = sigmoid(gate_logits)
    gb = g.reshape(1, H, 1, 1)
    z_sm = gb * o_sm
    z_lin = (1.0 - gb) * o_lin
    if w_per_head:
        dz_sm = np.einsum("blhe,de->bhld", dY, W1)
        dz_lin = np.einsum("blhe,de->bhld", dY, W2)
        dW1 = np.einsum("bhld,blhe->de", z_sm, dY)
        dW2 = np.einsum("bhld,blhe->de", z_lin, dY)
    else:
        dz_sm = np.zeros_like(o_sm)
        dz_lin = np.zeros_like(o_lin)
        dW1 = np.zeros_like(W1)
        dW2 = np.zeros_like(W2)
        for h in range(H):
            rows = slice(h * dv, (h + 1) * dv)
            dz_sm[:, h] = dY @ W1[rows].T
            dz_lin[:, h] = dY @ W2[rows].T
            dW1[rows] = np.einsum("bld,ble->de", z_sm[:, h], dY)
            dW2[rows] = np.einsum("bld,ble->de", z_lin[:, h], dY)
    do_sm = gb * dz_sm
    do_lin = (1.0 - gb) * dz_lin
    dg = (dz_sm * o_sm).sum(axis=(0, 2, 3)) - (dz_lin * o_lin).sum(axis=(0, 2, 3))
    dlogit = dg * g * (1.0 - g)
    return dict(do_sm=do_sm, do_lin=do_lin, dgate_logits=dlogit, dW1=dW1, dW2=dW2,
                dz_sm=dz_sm, dz_lin=dz_lin)


# ---------------------------------------------------------------------- layer
def vdn_layer_bwd(x, wl, dY):
    """Cotangents of every input of ``vdn_oracle.vdn_layer`` for L = <dY, Y>.

    x: q, k, v, gate_logits, W1, W2 (fp64); wl: the workload description.
    Returns dq, dk, dv, dgate_logits, dW1, dW2 and the intermediate
    cotangents (do_sm, do_lin) and forward values (the forward dict).
    """
    fwd = vdn_layer(x, wl)
    q, k, v = x["q"], x["k"], x["v"]
    B, H, L, d = q.shape
    T, N = wl.T, wl.N
    n_ctx = getattr(wl, "n_ctx", 0)
    TN = T * N
    bf, W, anc = wl.block_frames, wl.window_blocks, wl.anchors
    scale = 1.0 / np.sqrt(d)
    mask, _ = window_plan(T, bf, W, anc)
    mb = gated_merge_bwd(fwd["o_sm"], fwd["o_lin"], x["gate_logits"], x["W1"], x["W2"], dY,
                         wl.w_per_head)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            sq, sk, sv = softmax_window_bwd(q[b, h], k[b, h], v[b, h], mb["do_sm"][b, h], T, N,
                                            n_ctx, mask, scale)
            lb = linear_branch_bwd(q[b, h, :TN], k[b, h, :TN], v[b, h, :TN],
                                   mb["do_lin"][b, h, :TN], T, N, wl.lam, wl.beta, bf, W, anc)
            dq[b, h] = sq
            dk[b, h] = sk
            dv[b, h] = sv
            dq[b, h, :TN] += lb["dq"]
            dk[b, h, :TN] += lb["dk"]
            dv[b, h, :TN] += lb["dv"]
    return dict(dq=dq, dk=dk, dv=dv, dgate_logits=mb["dgate_logits"], dW1=mb["dW1"],
                dW2=mb["dW2"], do_sm=mb["do_sm"], do_lin=mb["do_lin"], fwd=fwd)

