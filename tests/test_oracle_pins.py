"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test checks the oracle against what the pages or the mathematics fix:
hand-written masks from the pages' window rules, a library attention routine,
least squares, spectral bounds, reversal symmetry and closed-form limits of
the gate. A dropped term, a wrong sign or index, or a transposed operand in
the oracle fails at least one of them.
"""
import numpy as np
import pytest
import torch

import oracle as O
from synthetic import get_workload, make_inputs, to_f64


def _rand_keys(rng, n, d):
    k = rng.standard_normal((n, d))
    return k / np.linalg.norm(k, axis=1, keepdims=True)


# ------------------------------------------------------------------ the mask
@pytest.mark.parametrize("name,T", [("mask_T12_bf5_w1_anchors.txt", 12),
                                    ("mask_T16_bf5_w1_anchors.txt", 16)])
def test_mask_matches_hand_written_fixture(fixture_rows, name, T):
    rows = fixture_rows(name)
    want = np.array([[int(c) for c in r] for r in rows], dtype=np.uint8)
    assert want.shape == (T, T)
    np.testing.assert_array_equal(O.frame_mask(T, 5, 1, 1), want)


def test_mask_window_counts_match_pages():
    # flyP critical read, method breakdown: an interior frame matches 15
    # neighbouring frames token-to-token, plus the first and last frames.
    T = 60
    m = O.frame_mask(T)
    for i in range(10, 50):
        assert m[i].sum() == 15 + 2
        blk = i // 5
        win = [j for j in range(T) if abs(j // 5 - blk) <= 1]
        assert len(win) == 15 and all(m[i, j] for j in win)
    # edge blocks see one neighbouring block only: 10 window frames + 1 anchor
    for i in list(range(1, 5)) + list(range(55, 59)):
        assert m[i].sum() == 10 + 1
    assert m[0].all() and m[T - 1].all() and m[:, 0].all() and m[:, T - 1].all()
    np.testing.assert_array_equal(m, m.T)


@pytest.mark.parametrize("T", range(1, 11))
def test_short_videos_are_fully_attended(T):
    assert O.frame_mask(T).all()


def test_anchor_density_figure(fixture_rows):
    # The pages give +3.57% density for the anchors but not the frame count;
    # at T=100 the block window + anchors rule gives +3.580 percentage points.
    page = float(fixture_rows("anchor_density.txt")[0])
    T = 100
    inc = 100.0 * (O.frame_mask(T, anchors=1).sum() - O.frame_mask(T, anchors=0).sum()) / T**2
    assert abs(inc - 3.58) < 5e-4
    assert abs(inc - page) < 0.011


@pytest.mark.parametrize("T,bf,W,anc", [(60, 5, 1, 1), (61, 5, 1, 1), (240, 5, 1, 1),
                                        (20, 5, 1, 1), (11, 5, 1, 1), (23, 4, 2, 1),
                                        (30, 5, 1, 0), (7, 3, 0, 1)])
def test_plan_segments_rebuild_the_mask(T, bf, W, anc):
    m, segs = O.window_plan(T, bf, W, anc)
    rebuilt = np.zeros_like(m)
    covered = []
    for q0, q1, rr in segs:
        assert q0 < q1 and (q1 - 1) // bf == q0 // bf   # inside one block
        covered += list(range(q0, q1))
        for k0, k1 in rr:
            rebuilt[q0:q1, k0:k1] = 1
    assert covered == list(range(T))
    np.testing.assert_array_equal(rebuilt, m)
    flat = O.serialize_plan(segs)
    assert flat.dtype == np.int32 and flat[0] == 0


# ---------------------------------------------------- coverage of the frames
@pytest.mark.parametrize("T", [12, 20, 31, 60, 61])
def test_linear_ranges_partition_the_frames(T):
    # sd114.wiki, bidirectional linear branch: window, anchors, forward range
    # and backward range are disjoint and together cover every frame.
    m = O.frame_mask(T)
    for i in range(T):
        soft = set(np.nonzero(m[i])[0])
        before = {j for j in range(T) if not m[i, j] and j < i}
        after = {j for j in range(T) if not m[i, j] and j > i}
        assert soft | before | after == set(range(T))
        assert not (soft & before) and not (soft & after) and not (before & after)
        b = i // 5
        ws, we = O.window_bounds(b, T)
        if i not in (0, T - 1):
            assert before == set(range(1, ws)) and after == set(range(we, T - 1))


def _scan_by_sets(A, Bm, frames):
    S = np.zeros_like(Bm[0])
    for f in frames:
        S = S @ A[f] + Bm[f]
    return S


@pytest.mark.parametrize("T,anc", [(23, 1), (31, 1), (26, 0)])
def test_states_equal_scan_over_mask_complement(T, anc):
    rng = np.random.default_rng(7)
    d = dv = 6
    N = 9
    k = _rand_keys(rng, T * N, d)
    v = rng.standard_normal((T * N, dv))
    lb = O.linear_branch(None, k, v, T, N, 1e-2, 0.7, anchors=anc)
    m = O.frame_mask(T, anchors=anc)
    for i in range(T):
        if anc and i in (0, T - 1):
            continue
        b = i // 5
        before = [j for j in range(T) if not m[i, j] and j < i]
        after = [j for j in range(T - 1, -1, -1) if not m[i, j] and j > i]
        np.testing.assert_allclose(lb["S_fwd"][b], _scan_by_sets(lb["A"], lb["Bm"], before),
                                   rtol=0, atol=1e-12)
        np.testing.assert_allclose(lb["S_bwd"][b], _scan_by_sets(lb["A"], lb["Bm"], after),
                                   rtol=0, atol=1e-12)


# --------------------------------------------------------- softmax branch
def test_softmax_equals_dense_masked_attention():
    rng = np.random.default_rng(3)
    T, N, d, dv = 13, 4, 8, 5
    q = rng.standard_normal((T * N, d))
    k = _rand_keys(rng, T * N, d)
    v = rng.standard_normal((T * N, dv))
    m = O.frame_mask(T)
    scale = 1 / np.sqrt(d)
    tok = np.kron(m, np.ones((N, N), dtype=np.uint8)).astype(bool)
    s = (q @ k.T) * scale
    s = np.where(tok, s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    want = p @ v
    got = O.softmax_window(q, k, v, T, N, m, scale)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)
    rows = [0, 5, 17, T * N - 1]
    np.testing.assert_allclose(O.softmax_window_rows(rows, q, k, v, N, m, scale), want[rows],
                               rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("T", [1, 4, 10])
def test_short_video_softmax_is_full_attention(T):
    rng = np.random.default_rng(T)
    N, d, dv = 6, 16, 16
    q = rng.standard_normal((T * N, d))
    k = _rand_keys(rng, T * N, d)
    v = rng.standard_normal((T * N, dv))
    got = O.softmax_window(q, k, v, T, N, O.frame_mask(T), 1 / np.sqrt(d))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0]
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------- linear branch
@pytest.mark.parametrize("T", [1, 2, 5, 10])
def test_linear_branch_is_zero_when_the_window_covers_all(T):
    rng = np.random.default_rng(11)
    N, d = 5, 4
    q = rng.standard_normal((T * N, d))
    k = _rand_keys(rng, T * N, d)
    v = rng.standard_normal((T * N, d))
    lb = O.linear_branch(q, k, v, T, N, 1e-2, 0.5)
    assert not lb["S_fwd"].any() and not lb["S_bwd"].any() and not lb["o_lin"].any()


def test_update_is_least_squares_map_as_lambda_vanishes():
    rng = np.random.default_rng(5)
    N, d, dv = 40, 8, 6
    K = _rand_keys(rng, N, d)
    V = rng.standard_normal((N, dv))
    A, Bm = O.frame_solve(K.T @ K, V.T @ K, 1e-12, 1.0)
    X, *_ = np.linalg.lstsq(K, V, rcond=None)        # K X ~= V
    np.testing.assert_allclose(Bm, X.T, rtol=1e-8, atol=1e-9)
    assert np.abs(A).max() < 1e-9


@pytest.mark.parametrize("lam,beta", [(1e-2, 1.0), (0.3, 1.0), (1e-2, 0.5), (2.0, 0.25)])
def test_update_is_ridge_step(lam, beta):
    # S' = argmin ||S' K^T - V^T||^2 + lam ||S' - S||^2 solved as the stacked
    # least-squares system [K; sqrt(lam) I] X = [V; sqrt(lam) S^T] (QR/SVD,
    # independent of the Cholesky path), then moved a fraction beta from S.
    rng = np.random.default_rng(int(lam * 100 + beta * 10))
    N, d, dv = 12, 7, 5
    K = _rand_keys(rng, N, d)
    V = rng.standard_normal((N, dv))
    S = rng.standard_normal((dv, d))
    A, Bm = O.frame_solve(K.T @ K, V.T @ K, lam, beta)
    lhs = np.vstack([K, np.sqrt(lam) * np.eye(d)])
    rhs = np.vstack([V, np.sqrt(lam) * S.T])
    X, *_ = np.linalg.lstsq(lhs, rhs, rcond=None)
    want = (1 - beta) * S + beta * X.T
    np.testing.assert_allclose(S @ A + Bm, want, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("keys", ["gauss", "rank_deficient", "student_t"])
def test_update_is_non_expansive(keys):
    # besthub.dev, VDA: the update is non-expansive. A_f = I - beta G M is
    # symmetric with eigenvalues 1 - beta s/(s+lam) in [1-beta, 1].
    wl = get_workload("vda_only", B=1, H=1, T=12, N=96, d=32, dv=32, keys=keys,
                      extra={"deficient_frac": 0.5, "rank": 4, "nu": 3})
    x = make_inputs(wl)
    k, v = to_f64(x["k"])[0, 0], to_f64(x["v"])[0, 0]
    G, C = O.frame_stats(k, v, wl.T, wl.N)
    for beta in (1.0, 0.5):
        for f in range(wl.T):
            A, _ = O.frame_solve(G[f], C[f], wl.lam, beta)
            np.testing.assert_allclose(A, A.T, atol=1e-9)
            assert np.linalg.norm(A, 2) <= 1 + 1e-9
            ev = np.linalg.eigvalsh((A + A.T) / 2)
            assert ev.min() >= 1 - beta - 1e-9 and ev.max() <= 1 + 1e-9


def test_gram_trace_is_token_count():
    # keys are unit vectors, so trace(K_f^T K_f) = N for every frame
    wl = get_workload("tiny")
    x = make_inputs(wl)
    k, v = to_f64(x["k"])[0, 1], to_f64(x["v"])[0, 1]
    G, C = O.frame_stats(k, v, wl.T, wl.N)
    np.testing.assert_allclose(np.trace(G, axis1=1, axis2=2), wl.N, rtol=1e-6)
    assert C.shape == (wl.T, wl.dv, wl.d)


@pytest.mark.parametrize("T", [20, 40])
def test_reversal_swaps_forward_and_backward(T):
    rng = np.random.default_rng(T)
    N, d = 7, 5
    q = rng.standard_normal((T * N, d))
    k = _rand_keys(rng, T * N, d)
    v = rng.standard_normal((T * N, d))
    rev = lambda x: x.reshape(T, N, -1)[::-1].reshape(T * N, -1)  # noqa: E731
    a = O.linear_branch(q, k, v, T, N, 1e-2, 0.8)
    b = O.linear_branch(rev(q), rev(k), rev(v), T, N, 1e-2, 0.8)
    nb = T // 5
    for blk in range(nb):
        np.testing.assert_allclose(b["S_fwd"][blk], a["S_bwd"][nb - 1 - blk], rtol=1e-9, atol=1e-10)
        np.testing.assert_allclose(b["S_bwd"][blk], a["S_fwd"][nb - 1 - blk], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(b["o_lin"], rev(a["o_lin"]), rtol=1e-9, atol=1e-10)


# -------------------------------------------------------------------- merge
@pytest.mark.parametrize("w_per_head", [0, 1])
def test_gate_limits(w_per_head):
    rng = np.random.default_rng(2)
    B, H, L, dv, do = 2, 3, 5, 4, 6
    o_sm = rng.standard_normal((B, H, L, dv))
    o_lin = rng.standard_normal((B, H, L, dv))
    rows = dv if w_per_head else H * dv
    W1 = rng.standard_normal((rows, do))
    W2 = rng.standard_normal((rows, do))
    for logit, which in ((60.0, "sm"), (-60.0, "lin")):
        Y, Z = O.gated_merge(o_sm, o_lin, np.full(H, logit), W1, W2, w_per_head)
        src, W = (o_sm, W1) if which == "sm" else (o_lin, W2)
        if w_per_head:
            want = np.stack([src[:, h] @ W for h in range(H)], axis=2)
        else:
            want = src.transpose(0, 2, 1, 3).reshape(B, L, H * dv) @ W
        np.testing.assert_allclose(Y, want, rtol=1e-12, atol=1e-12)
    Y, Z = O.gated_merge(o_sm, o_lin, np.zeros(H), W1, W2, w_per_head)
    np.testing.assert_allclose(Z[:, :, 0], 0.5 * o_sm.transpose(0, 2, 1, 3))
    np.testing.assert_allclose(Z[:, :, 1], 0.5 * o_lin.transpose(0, 2, 1, 3))


def test_tiny_layer_runs_and_is_finite():
    wl = get_workload("tiny")
    x = {k: (to_f64(t) if hasattr(t, "detach") else t) for k, t in make_inputs(wl).items()}
    out = O.vdn_layer(x, wl)
    for key in ("o_sm", "o_lin", "Y", "Z", "S_fwd", "S_bwd"):
        assert np.isfinite(out[key]).all()
    assert out["Y"].shape == (1, wl.L, wl.H, wl.d_out)
    assert np.abs(out["o_lin"]).max() > 0


def _ridge_step(S, K, V, lam, beta):
    """One update solved as a stacked least-squares problem (no Cholesky)."""
    d = K.shape[1]
    lhs = np.vstack([K, np.sqrt(lam) * np.eye(d)])
    rhs = np.vstack([V, np.sqrt(lam) * S.T])
    X, *_ = np.linalg.lstsq(lhs, rhs, rcond=None)
    return (1 - beta) * S + beta * X.T


@pytest.mark.parametrize("beta", [1.0, 0.6])
def test_block_states_are_chained_ridge_steps(beta):
    # T=12: frames 10 and 11 form block 2; its window starts at frame 5, so its
    # forward state has seen frames 1..4 in order (frame 0 is an anchor). Block
    # 0's window ends at frame 10, so its backward state has seen frame 10 only
    # (frame 11 is an anchor).
    T, N, d, dv, lam = 12, 6, 4, 3, 0.1
    rng = np.random.default_rng(19)
    k = _rand_keys(rng, T * N, d)
    v = rng.standard_normal((T * N, dv))
    lb = O.linear_branch(None, k, v, T, N, lam, beta)
    fr = lambda x, f: x[f * N:(f + 1) * N]  # noqa: E731
    S = np.zeros((dv, d))
    for f in (1, 2, 3, 4):
        S = _ridge_step(S, fr(k, f), fr(v, f), lam, beta)
    np.testing.assert_allclose(lb["S_fwd"][2], S, rtol=1e-9, atol=1e-11)
    S = _ridge_step(np.zeros((dv, d)), fr(k, 10), fr(v, 10), lam, beta)
    np.testing.assert_allclose(lb["S_bwd"][0], S, rtol=1e-9, atol=1e-11)
    assert not lb["S_fwd"][0].any() and not lb["S_bwd"][2].any()


def test_readout_recalls_values_of_the_last_memorised_frame():
    # With beta=1, lambda->0 and N=d, the state after frame 4 maps each key of
    # frame 4 exactly to its value. Queries of frame 10 set to those keys must
    # read back frame 4's values: this fixes S q (not S^T q) and the index of
    # the forward state.
    T, d = 12, 6
    N = d
    rng = np.random.default_rng(23)
    k = _rand_keys(rng, T * N, d)
    v = rng.standard_normal((T * N, d))
    q = rng.standard_normal((T * N, d))
    q[10 * N:11 * N] = k[4 * N:5 * N]
    lb = O.linear_branch(q, k, v, T, N, 1e-13, 1.0)
    np.testing.assert_allclose(lb["o_lin"][10 * N:11 * N], v[4 * N:5 * N], rtol=1e-6, atol=1e-7)
    assert not lb["o_lin"][:N].any() and not lb["o_lin"][11 * N:].any()   # anchors


# ------------------------------------------------- joint multimodal attention
def _sdpa(q, k, v, scale, mask=None):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]  # noqa: E731
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=m, scale=scale)[0, 0].numpy()


def _joint_inputs(T, N, n_ctx, seed):
    rng = np.random.default_rng(seed)
    L = T * N + n_ctx
    return rng.standard_normal((L, 16)), _rand_keys(rng, L, 16), rng.standard_normal((L, 8))


def test_joint_without_context_is_the_window_softmax():
    T, N = 13, 6
    q, k, v = _joint_inputs(T, N, 0, 3)
    m = O.frame_mask(T)
    np.testing.assert_allclose(O.softmax_joint(q, k, v, T, N, 0, m, 0.25),
                               O.softmax_window(q, k, v, T, N, m, 0.25), rtol=0, atol=1e-13)


def test_joint_context_rows_are_full_attention():
    # mlsanity abstract: interactions involving text or audio keep softmax;
    # a context query sees every token
    T, N, n_ctx = 14, 5, 9
    q, k, v = _joint_inputs(T, N, n_ctx, 4)
    out = O.softmax_joint(q, k, v, T, N, n_ctx, O.frame_mask(T), 0.3)
    np.testing.assert_allclose(out[T * N:], _sdpa(q[T * N:], k, v, 0.3), rtol=0, atol=1e-12)


def test_joint_matches_dense_token_mask():
    # video rows: the frame mask expanded to tokens, plus every context key
    T, N, n_ctx = 16, 4, 7
    q, k, v = _joint_inputs(T, N, n_ctx, 5)
    m = O.frame_mask(T)
    L = T * N + n_ctx
    allow = np.ones((L, L), dtype=bool)
    allow[:T * N, :T * N] = np.kron(m, np.ones((N, N))).astype(bool)
    np.testing.assert_allclose(O.softmax_joint(q, k, v, T, N, n_ctx, m, 0.2),
                               _sdpa(q, k, v, 0.2, allow), rtol=0, atol=1e-12)


def test_joint_short_video_is_full_attention():
    # T <= 10: every frame pair is inside a window or an anchor
    T, N, n_ctx = 8, 5, 6
    q, k, v = _joint_inputs(T, N, n_ctx, 6)
    np.testing.assert_allclose(O.softmax_joint(q, k, v, T, N, n_ctx, O.frame_mask(T), 0.25),
                               _sdpa(q, k, v, 0.25), rtol=0, atol=1e-12)


def test_layer_with_context_has_no_linear_output_on_context_rows():
    wl = get_workload("small", B=1, H=1, T=12, N=6, d=16, dv=8, d_out=8, n_ctx=5, seed=9)
    x = {n: to_f64(t) for n, t in make_inputs(wl).items() if n != "deficient_frames"}
    ref = O.vdn_layer(x, wl)
    assert ref["o_lin"].shape[2] == wl.L
    assert not ref["o_lin"][:, :, wl.T * wl.N:].any()
    # the video part of the linear branch is the video-only layer's
    vid = {n: (a[:, :, :wl.T * wl.N] if n in ("q", "k", "v") else a) for n, a in x.items()}
    ref0 = O.vdn_layer(vid, wl.with_(n_ctx=0))
    np.testing.assert_array_equal(ref["o_lin"][:, :, :wl.T * wl.N], ref0["o_lin"])


# -------------------------------------------------------------- whole layer
def _layer_independent(x, wl):
    """Y and Z of the hybrid layer built without the oracle's layer code.

    Only the hand-pinned frame mask comes from the oracle. The softmax branch
    is PyTorch's fp64 scaled-dot-product attention at its own default scale
    under the frame mask expanded to tokens (context tokens see and are seen
    by every token). Each video query frame's linear state is a chain of ridge
    steps, each solved as a stacked least-squares problem, over the frames its
    mask row excludes: those before it in increasing order and those after it
    in decreasing order (sd114.wiki, bidirectional linear branch), then read
    as (S_fwd + S_bwd) q. The gate is the logistic function of scipy, and the
    projections are one matrix product of the concatenated heads.
    """
    from scipy.special import expit
    q, k, v = x["q"], x["k"], x["v"]
    B, H, L, d = q.shape
    dv = v.shape[-1]
    T, N = wl.T, wl.N
    TN = T * N
    m = O.frame_mask(T, wl.block_frames, wl.window_blocks, wl.anchors)
    allow = np.ones((L, L), dtype=bool)
    allow[:TN, :TN] = np.kron(m, np.ones((N, N))).astype(bool)
    o_sm = np.zeros((B, H, L, dv))
    o_lin = np.zeros((B, H, L, dv))
    for b in range(B):
        for h in range(H):
            o_sm[b, h] = _sdpa(q[b, h], k[b, h], v[b, h], None, allow)
            fr = lambda a, f: a[b, h, f * N:(f + 1) * N]  # noqa: E731
            for i in range(T):
                S = np.zeros((dv, d))
                for order in ([j for j in range(T) if j < i and not m[i, j]],
                              [j for j in range(T - 1, -1, -1) if j > i and not m[i, j]]):
                    Sd = np.zeros((dv, d))
                    for j in order:
                        Sd = _ridge_step(Sd, fr(k, j), fr(v, j), wl.lam, wl.beta)
                    S = S + Sd
                o_lin[b, h, i * N:(i + 1) * N] = fr(q, i) @ S.T
    g = expit(x["gate_logits"])[None, None, :, None]
    z_sm = g * o_sm.transpose(0, 2, 1, 3)            # [B, L, H, dv]
    z_lin = (1.0 - g) * o_lin.transpose(0, 2, 1, 3)
    Z = np.stack([z_sm, z_lin], axis=2)
    if wl.w_per_head:
        Y = z_sm @ x["W1"] + z_lin @ x["W2"]          # [B, L, H, d_out]
    else:
        Y = z_sm.reshape(B, L, H * dv) @ x["W1"] + z_lin.reshape(B, L, H * dv) @ x["W2"]
    return Y, Z


@pytest.mark.parametrize("case", [
    dict(T=23, N=6, anchors=1),                                   # ragged last block
    dict(T=21, N=5, anchors=0),                                   # anchors off, 1-frame block
    dict(T=17, N=4, anchors=1, n_ctx=7),                          # context tokens
    dict(T=22, N=5, anchors=1, block_frames=4, window_blocks=2),  # wider window
    dict(T=16, N=6, anchors=1, w_per_head=1),                     # head-shared projections
])
def test_layer_equals_independent_build(case):
    # mlsanity abstract (local softmax + bidirectional linear memory, separate
    # projections, learnable gates); sd114.wiki, both branch sections. The
    # gate logits are spread out so that a swapped gate shows; lambda and beta
    # differ so that swapping them shows; d = 8 makes 1/d and 1/sqrt(d) differ.
    n_ctx = case.pop("n_ctx", 0)
    wph = case.pop("w_per_head", 0)
    wl = get_workload("small", B=2, H=3, d=8, dv=6, d_out=5, lam=0.05, beta=0.7, seed=31,
                      n_ctx=n_ctx, w_per_head=wph, **case)
    x = {n: to_f64(t) for n, t in make_inputs(wl).items() if n != "deficient_frames"}
    x["gate_logits"] = np.array([-1.5, 0.4, 2.0])
    Y, Z = _layer_independent(x, wl)
    ref = O.vdn_layer(x, wl)
    assert np.abs(Y).max() > 0 and np.abs(Z[:, :, 1]).max() > 0
    np.testing.assert_allclose(ref["Z"], Z, rtol=0, atol=1e-10 * np.abs(Z).max())
    np.testing.assert_allclose(ref["Y"], Y, rtol=0, atol=1e-10 * np.abs(Y).max())
