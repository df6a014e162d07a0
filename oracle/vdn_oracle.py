"""Video DeltaNet (VDN) hybrid attention layer, video-to-video forward pass:
a plain, slow, fp64 NumPy reference.

TEST INFRASTRUCTURE ONLY: tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` may use it; the product path may not.

Sources (web pages about "Video DeltaNet: A Video-Native Hybrid Attention for
Livestream Video Generation"):

* mlsanity index page, "Abstract (arXiv)": local softmax attention plus
  bidirectional linear memory; the linear branch (Video Delta Attention, VDA)
  updates memory once per frame using all of the frame's spatial tokens;
  separate output projections and learnable gates combine the two branches.
* besthub.dev article, "Video Delta Attention (VDA)": all spatial tokens of a
  frame jointly solve one state update; the update is non-expansive.
  "Hybrid Attention Architecture": the branch outputs are merged by a gate.
* sd114.wiki article, "双向滑动窗口Softmax分支" (bidirectional sliding-window
  softmax branch): 5 consecutive latent frames form a block; a block attends
  to itself, the previous and the next block; every frame also attends to all
  tokens of the first and last frames, which attend to every frame.
* same article, "双向线性注意力分支" (bidirectional linear branch): for frame
  i a forward state summarises the frames before the window and a backward
  state the frames after it; the two ranges are disjoint and exclude what the
  window and the anchors already cover; the query reads both and the results
  are summed.
* flyP critical read, "一、方法拆解" (method breakdown): each frame matches 15
  neighbouring frames token-to-token (the 3-block window), plus the first and
  last frames as boundary anchors.

The pages never write VDA as an equation. This library fixes one closed form
and uses it everywhere:

    G_f = K_f^T K_f,  C_f = V_f^T K_f,  M_f = (G_f + lambda I)^-1,
    S <- S (I - beta G_f M_f) + beta C_f M_f ,   output (S_fwd + S_bwd) q.

For beta = 1 this is the ridge regression argmin_S' ||S' K_f^T - V_f^T||^2 +
lambda ||S' - S||^2; for beta < 1 it moves a fraction beta of the way there.

Conventions: per (b, h), K_f, Q_f are the N x d rows of frame f, V_f the
N x dv rows; token index t = f*N + n. States S are dv x d. Block of frame f is
f // block_frames. Everything is float64; inputs are the exact stored values
(bf16 or fp32) upcast to float64.
"""
import numpy as np
import scipy.linalg

__all__ = [
    "frame_mask", "window_plan", "serialize_plan", "window_bounds",
    "frame_stats", "frame_solve", "bidir_states", "readout",
    "softmax_window", "softmax_window_rows", "softmax_joint", "gated_merge", "vdn_layer",
    "linear_branch", "sigmoid",
]


# ---------------------------------------------------------------- window plan
def frame_mask(T, block_frames=5, window_blocks=1, anchors=1):
    """Frame-level attention mask m[i, j] (uint8), built by explicit loops.

    sd114.wiki, bidirectional sliding-window softmax branch: i attends j when
    their blocks differ by at most `window_blocks`; with anchors, every frame
    attends frames 0 and T-1, and frames 0 and T-1 attend every frame.
    """
    m = np.zeros((T, T), dtype=np.uint8)
    for i in range(T):
        for j in range(T):
            in_window = abs(i // block_frames - j // block_frames) <= window_blocks
            anchor = bool(anchors) and (j == 0 or j == T - 1 or i == 0 or i == T - 1)
            m[i, j] = 1 if (in_window or anchor) else 0
    return m


def _runs(row):
    """Maximal runs of ones of a 0/1 row as [start, end) pairs."""
    out, j, T = [], 0, len(row)
    while j < T:
        if row[j]:
            s = j
            while j < T and row[j]:
                j += 1
            out.append((s, j))
        else:
            j += 1
    return out


def window_plan(T, block_frames=5, window_blocks=1, anchors=1):
    """Query segments and their key-frame ranges, derived from the mask.

    A segment is a maximal run of consecutive query frames in one block whose
    mask rows are identical; its key ranges are the maximal runs of ones of
    that row. Returns (mask, [(q_f0, q_f1, [(k_f0, k_f1), ...]), ...]).
    """
    m = frame_mask(T, block_frames, window_blocks, anchors)
    segs, i = [], 0
    while i < T:
        j = i + 1
        while (j < T and j // block_frames == i // block_frames
               and np.array_equal(m[j], m[i])):
            j += 1
        segs.append((i, j, _runs(m[i])))
        i = j
    return m, segs


def serialize_plan(segs):
    """Flat int32 form: per segment q_f0, q_f1, n_ranges, then k_f0, k_f1 pairs."""
    out = []
    for q0, q1, rr in segs:
        out += [q0, q1, len(rr)]
        for k0, k1 in rr:
            out += [k0, k1]
    return np.asarray(out, dtype=np.int32)


def window_bounds(b, T, block_frames=5, window_blocks=1):
    """First frame of block b's window and one past its last frame."""
    ws = max(0, (b - window_blocks) * block_frames)
    we = min(T, (b + window_blocks + 1) * block_frames)
    return ws, we


def _is_anchor(f, T, anchors):
    return bool(anchors) and (f == 0 or f == T - 1)


# ------------------------------------------------------------- linear branch
def frame_stats(k, v, T, N):
    """Per-frame G_f = K_f^T K_f (d x d) and C_f = V_f^T K_f (dv x d).

    besthub.dev, VDA: the frame's spatial tokens enter one joint update; these
    two Gram-type sums are all of the frame that the closed form needs.
    k: [T*N, d], v: [T*N, dv] (one (b, h)). Returns G [T,d,d], C [T,dv,d].
    """
    d, dv = k.shape[1], v.shape[1]
    G = np.empty((T, d, d))
    C = np.empty((T, dv, d))
    for f in range(T):
        Kf = k[f * N:(f + 1) * N]
        Vf = v[f * N:(f + 1) * N]
        G[f] = Kf.T @ Kf
        C[f] = Vf.T @ Kf
    return G, C


def frame_solve(Gf, Cf, lam, beta):
    """One frame's affine map S -> S A_f + B_f of the closed-form VDA update.

    M_f = (G_f + lambda I)^-1 from a Cholesky factor and two triangular
    solves; A_f = I - beta G_f M_f; B_f = beta C_f M_f.
    """
    d = Gf.shape[0]
    eye = np.eye(d)
    Lc = np.linalg.cholesky(Gf + lam * eye)
    Linv = scipy.linalg.solve_triangular(Lc, eye, lower=True)
    M = Linv.T @ Linv
    A = eye - beta * (Gf @ M)
    Bm = beta * (Cf @ M)
    return A, Bm


def bidir_states(A, Bm, T, block_frames=5, window_blocks=1, anchors=1):
    """Forward and backward states per block, by a plain sequential scan.

    sd114.wiki, bidirectional linear branch: for a query in block b the forward
    state covers the frames before b's window and the backward state the
    frames after it; anchor frames (covered by softmax) take no part. The
    forward scan applies frames in increasing order from S = 0; the backward
    scan applies them in decreasing order from S = 0, so the frame nearest to
    the window is applied last in both.

    A, Bm: [T, d, d], [T, dv, d] per-frame maps. Returns S_fwd, S_bwd of shape
    [nb, dv, d].
    """
    dv, d = Bm.shape[1], Bm.shape[2]
    nb = -(-T // block_frames)
    fwd_after = np.zeros((T, dv, d))   # state after frames 0..f were processed
    S = np.zeros((dv, d))
    for f in range(T):
        if not _is_anchor(f, T, anchors):
            S = S @ A[f] + Bm[f]
        fwd_after[f] = S
    bwd_after = np.zeros((T, dv, d))   # state after frames T-1 .. f were processed
    S = np.zeros((dv, d))
    for f in range(T - 1, -1, -1):
        if not _is_anchor(f, T, anchors):
            S = S @ A[f] + Bm[f]
        bwd_after[f] = S
    S_fwd = np.zeros((nb, dv, d))
    S_bwd = np.zeros((nb, dv, d))
    for b in range(nb):
        ws, we = window_bounds(b, T, block_frames, window_blocks)
        if ws >= 1:
            S_fwd[b] = fwd_after[ws - 1]
        if we <= T - 1:
            S_bwd[b] = bwd_after[we]
    return S_fwd, S_bwd


def readout(q, S_fwd, S_bwd, T, N, block_frames=5, anchors=1):
    """o_lin[t] = (S_fwd(b) + S_bwd(b)) q_t for tokens of non-anchor frames.

    sd114.wiki, bidirectional linear branch: the query reads both states and
    the results are summed. Anchor frames already see every frame through
    softmax, so their linear output is 0. q: [T*N, d]; returns [T*N, dv].
    """
    dv = S_fwd.shape[1]
    out = np.zeros((T * N, dv))
    for f in range(T):
        if _is_anchor(f, T, anchors):
            continue
        b = f // block_frames
        S = S_fwd[b] + S_bwd[b]
        out[f * N:(f + 1) * N] = q[f * N:(f + 1) * N] @ S.T
    return out


def linear_branch(q, k, v, T, N, lam, beta, block_frames=5, window_blocks=1,
                  anchors=1):
    """Stats, per-frame solve, bidirectional scan and readout for one (b, h)."""
    G, C = frame_stats(k, v, T, N)
    d, dv = k.shape[1], v.shape[1]
    A = np.zeros((T, d, d))
    Bm = np.zeros((T, dv, d))
    for f in range(T):
        if _is_anchor(f, T, anchors):
            A[f] = np.eye(d)      # never applied; kept finite for inspection
            continue
        A[f], Bm[f] = frame_solve(G[f], C[f], lam, beta)
    S_fwd, S_bwd = bidir_states(A, Bm, T, block_frames, window_blocks, anchors)
    o_lin = None if q is None else readout(q, S_fwd, S_bwd, T, N, block_frames, anchors)
    return dict(G=G, C=C, A=A, Bm=Bm, S_fwd=S_fwd, S_bwd=S_bwd, o_lin=o_lin)


# ------------------------------------------------------------ softmax branch
def _softmax_frame(qf, k, v, mask_row, N, scale):
    cols = np.concatenate([np.arange(j * N, (j + 1) * N)
                           for j in np.nonzero(mask_row)[0]])
    s = (qf @ k[cols].T) * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ v[cols]


def softmax_window(q, k, v, T, N, mask, scale):
    """Masked softmax attention, one query frame at a time.

    Every query of frame i attends the key tokens of the frames j with
    m[i, j] = 1 (window and anchors, union: a frame is attended once), with
    scores q.k * scale and an exact (not online) softmax. q, k: [T*N, d],
    v: [T*N, dv]; returns [T*N, dv].
    """
    out = np.zeros((T * N, v.shape[1]))
    for f in range(T):
        out[f * N:(f + 1) * N] = _softmax_frame(
            q[f * N:(f + 1) * N], k, v, mask[f], N, scale)
    return out


def softmax_window_rows(rows, q, k, v, N, mask, scale):
    """The same output for selected query token indices only (sampled rows).

    Rows of one query frame share that frame's key set, so they are computed
    together from one gather of the allowed keys.
    """
    rows = np.asarray(rows)
    out = np.zeros((len(rows), v.shape[1]))
    frames = rows // N
    for f in np.unique(frames):
        sel = np.nonzero(frames == f)[0]
        out[sel] = _softmax_frame(q[rows[sel]], k, v, mask[f], N, scale)
    return out


def softmax_joint(q, k, v, T, N, n_ctx, mask, scale):
    """Softmax branch of a sequence of T*N video tokens followed by n_ctx
    context (text or audio) tokens.

    mlsanity abstract: the hybrid replaces only video-to-video interactions;
    interactions involving text or audio keep softmax. flyP critical read,
    "具体作用范围": softmax stays for cross-modal interactions that text or
    audio take part in; the VDN hybrid covers only video-to-video ones.
    Reading: a query of video frame i attends the key frames of its mask row
    and every context token, in one softmax; a context query attends every
    token. q, k: [T*N + n_ctx, d], v: [T*N + n_ctx, dv]; returns the same
    rows of output.
    """
    TN = T * N
    ctx = np.arange(TN, TN + n_ctx)
    out = np.zeros((TN + n_ctx, v.shape[1]))
    for f in range(T):
        cols = np.concatenate([np.arange(j * N, (j + 1) * N) for j in np.nonzero(mask[f])[0]]
                              + [ctx])
        s = (q[f * N:(f + 1) * N] @ k[cols].T) * scale
        p = np.exp(s - s.max(axis=1, keepdims=True))
        out[f * N:(f + 1) * N] = (p / p.sum(axis=1, keepdims=True)) @ v[cols]
    if n_ctx:
        s = (q[TN:] @ k.T) * scale
        p = np.exp(s - s.max(axis=1, keepdims=True))
        out[TN:] = (p / p.sum(axis=1, keepdims=True)) @ v
    return out


# ---------------------------------------------------------------------- merge
def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, dtype=np.float64)))


def gated_merge(o_sm, o_lin, gate_logits, W1, W2, w_per_head=0):
    """Separate output projections merged by a per-head learned gate.

    mlsanity abstract / besthub.dev "Hybrid Attention Architecture": each
    branch has its own projection and a learnable gate balances them. The gate
    of head h is g_h = sigmoid(logit_h) and is convex:
        w_per_head = 0: Y[b,t,:]   = sum_h g_h o_sm[b,h,t] W1[h rows] + (1-g_h) o_lin[b,h,t] W2[h rows]
        w_per_head = 1: Y[b,t,h,:] = g_h o_sm[b,h,t] W1 + (1-g_h) o_lin[b,h,t] W2
    o_sm, o_lin: [B,H,L,dv]. Returns Y ([B,L,d_out] or [B,L,H,d_out]) and the
    gated branch outputs Z [B,L,2,H,dv].
    """
    B, H, L, dv = o_sm.shape
    g = sigmoid(gate_logits).reshape(1, H, 1, 1)
    z_sm = g * o_sm
    z_lin = (1.0 - g) * o_lin
    Z = np.stack([z_sm.transpose(0, 2, 1, 3), z_lin.transpose(0, 2, 1, 3)], axis=2)
    if w_per_head:
        Y = np.einsum("bhld,de->blhe", z_sm, W1) + np.einsum("bhld,de->blhe", z_lin, W2)
    else:
        Y = np.zeros((B, L, W1.shape[1]))
        for h in range(H):
            Y += z_sm[:, h] @ W1[h * dv:(h + 1) * dv] + z_lin[:, h] @ W2[h * dv:(h + 1) * dv]
    return Y, Z


# ---------------------------------------------------------------------- layer
def vdn_layer(x, wl, softmax=True, merge=True):
    """The whole hybrid layer for fp64 inputs x (dict of numpy arrays).

    x: q [B,H,L,d], k [B,H,L,d], v [B,H,L,dv], gate_logits [H], W1, W2.
    wl: a workload description with T, N, lam, beta, block_frames,
    window_blocks, anchors, w_per_head and optionally n_ctx (context tokens
    after the T*N video tokens of each head: softmax only, o_lin = 0).
    Returns every intermediate.
    """
    q, k, v = x["q"], x["k"], x["v"]
    B, H, L, d = q.shape
    dv = v.shape[-1]
    T, N = wl.T, wl.N
    n_ctx = getattr(wl, "n_ctx", 0)
    TN = T * N
    bf, W, anc = wl.block_frames, wl.window_blocks, wl.anchors
    scale = 1.0 / np.sqrt(d)
    mask, segs = window_plan(T, bf, W, anc)
    nb = -(-T // bf)
    out = dict(mask=mask, segments=segs,
               G=np.zeros((B, H, T, d, d)), C=np.zeros((B, H, T, dv, d)),
               S_fwd=np.zeros((B, H, nb, dv, d)), S_bwd=np.zeros((B, H, nb, dv, d)),
               o_lin=np.zeros((B, H, L, dv)))
    if softmax:
        out["o_sm"] = np.zeros((B, H, L, dv))
    for b in range(B):
        for h in range(H):
            lb = linear_branch(q[b, h, :TN], k[b, h, :TN], v[b, h, :TN], T, N, wl.lam, wl.beta,
                               bf, W, anc)
            for key in ("G", "C", "S_fwd", "S_bwd"):
                out[key][b, h] = lb[key]
            out["o_lin"][b, h, :TN] = lb["o_lin"]
            if softmax and n_ctx:
                out["o_sm"][b, h] = softmax_joint(q[b, h], k[b, h], v[b, h], T, N, n_ctx, mask,
                                                  scale)
            elif softmax:
                out["o_sm"][b, h] = softmax_window(q[b, h], k[b, h], v[b, h], T, N, mask, scale)
    if softmax and merge and "W1" in x:
        out["Y"], out["Z"] = gated_merge(out["o_sm"], out["o_lin"], x["gate_logits"],
                                         x["W1"], x["W2"], wl.w_per_head)
    return out
