"""Pins of the fp64 backward oracle to facts outside itself (CPU only).

* Central finite differences of the forward oracle (itself pinned by
  test_oracle_pins.py): for L = <dY, Y>, (L(x + e u) - L(x - e u)) / 2e must
  equal <dL/dx, u> for random directions u of every input, and entry by entry
  for every key of one head (the key reaches the output through the softmax,
  the frame statistics, the ridge inverse, both scans and the readout).
* PyTorch's own attention routine under autograd for the softmax branch.
* Closed forms: a single key (softmax weight 1), a video shorter than two
  frames with anchors (no linear branch), and a gate at its limits.
A dropped term, a sign or a transposed operand in any step of the backward
fails one of them.
"""
import numpy as np
import pytest
import torch

import oracle as O
from synthetic import get_workload, make_inputs, to_f64

NAMES = ("q", "k", "v", "gate_logits", "W1", "W2")


def _tiny(**over):
    base = dict(B=1, H=2, T=7, N=3, d=4, dv=4, d_out=5, block_frames=2, window_blocks=1,
                anchors=1, lam=0.5, beta=0.7, seed=11)
    base.update(over)
    return get_workload("tiny", **base)


def _inputs(wl):
    x = make_inputs(wl)
    return {n: to_f64(x[n]) for n in NAMES}


def _loss(x, wl, dY):
    return float((O.vdn_layer(x, wl)["Y"] * dY).sum())


def _dY(wl, seed=5):
    rng = np.random.default_rng(seed)
    shape = (wl.B, wl.L, wl.H, wl.d_out) if wl.w_per_head else (wl.B, wl.L, wl.d_out)
    return rng.standard_normal(shape)


CASES = {
    "anchors": {},
    "no_anchors": dict(anchors=0),
    "ragged_last_block": dict(T=8, block_frames=3),
    "context_tokens": dict(n_ctx=4),
    "shared_projection": dict(w_per_head=1),
    "wide_window": dict(T=9, window_blocks=2, beta=1.0),
}


@pytest.mark.parametrize("case", list(CASES))
def test_directional_derivatives_match_finite_differences(case):
    wl = _tiny(**CASES[case])
    x = _inputs(wl)
    dY = _dY(wl)
    grads = O.vdn_layer_bwd(x, wl, dY)
    key = {"q": "dq", "k": "dk", "v": "dv", "gate_logits": "dgate_logits", "W1": "dW1",
           "W2": "dW2"}
    rng = np.random.default_rng(7)
    eps = 1e-6
    for name in NAMES:
        for _ in range(2):
            u = rng.standard_normal(x[name].shape)
            xp = dict(x)
            xm = dict(x)
            xp[name] = x[name] + eps * u
            xm[name] = x[name] - eps * u
            fd = (_loss(xp, wl, dY) - _loss(xm, wl, dY)) / (2 * eps)
            an = float((grads[key[name]] * u).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_key_gradient_entry_by_entry():
    wl = _tiny()
    x = _inputs(wl)
    dY = _dY(wl)
    dk = O.vdn_layer_bwd(x, wl, dY)["dk"]
    eps = 1e-6
    b, h = 0, 1
    for t in range(wl.L):
        for c in range(wl.d):
            xp = dict(x)
            xm = dict(x)
            xp["k"] = x["k"].copy()
            xm["k"] = x["k"].copy()
            xp["k"][b, h, t, c] += eps
            xm["k"][b, h, t, c] -= eps
            fd = (_loss(xp, wl, dY) - _loss(xm, wl, dY)) / (2 * eps)
            assert abs(fd - dk[b, h, t, c]) <= 1e-6 * max(1.0, abs(fd)), (t, c)


def test_linear_branch_alone_matches_finite_differences():
    # the linear branch of one (b, h) with a loss on o_lin only
    wl = _tiny(T=11, N=4, block_frames=2, beta=0.9, lam=0.3)
    x = _inputs(wl)
    q, k, v = x["q"][0, 0], x["k"][0, 0], x["v"][0, 0]
    rng = np.random.default_rng(3)
    do = rng.standard_normal(v.shape)
    args = (wl.T, wl.N, wl.lam, wl.beta, wl.block_frames, wl.window_blocks, wl.anchors)
    g = O.linear_branch_bwd(q, k, v, do, *args)

    def loss(qq, kk, vv):
        return float((O.linear_branch(qq, kk, vv, *args)["o_lin"] * do).sum())

    eps = 1e-6
    for which, grad in (("q", g["dq"]), ("k", g["dk"]), ("v", g["dv"])):
        u = rng.standard_normal(q.shape)
        p = dict(q=q, k=k, v=v)
        m = dict(q=q, k=k, v=v)
        p[which] = p[which] + eps * u
        m[which] = m[which] - eps * u
        fd = (loss(p["q"], p["k"], p["v"]) - loss(m["q"], m["k"], m["v"])) / (2 * eps)
        an = float((grad * u).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), which


@pytest.mark.parametrize("n_ctx", [0, 5])
def test_softmax_backward_matches_torch_autograd(n_ctx):
    T, N, d, bf = 9, 4, 8, 2
    mask = O.frame_mask(T, bf, 1, 1)
    rng = np.random.default_rng(13)
    L = T * N + n_ctx
    q, k, v, do = (rng.standard_normal((L, d)) for _ in range(4))
    scale = 1.0 / np.sqrt(d)
    dq, dk, dv = O.softmax_window_bwd(q, k, v, do, T, N, n_ctx, mask, scale)
    allowed = np.ones((L, L), dtype=bool)
    tok_frame = np.arange(T * N) // N
    allowed[:T * N, :T * N] = mask[tok_frame][:, tok_frame].astype(bool)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(
        tq[None, None], tk[None, None], tv[None, None], attn_mask=torch.tensor(allowed)[None, None],
        scale=scale)[0, 0]
    out.backward(torch.tensor(do))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_sampled_row_dq_matches_torch_autograd():
    # the row-wise dq used on large cases: torch's autograd of its own
    # attention routine, read at the sampled rows
    T, N, d = 13, 5, 8
    mask = O.frame_mask(T)
    rng = np.random.default_rng(17)
    L = T * N
    q, k, v, do = (rng.standard_normal((L, d)) for _ in range(4))
    scale = 1.0 / np.sqrt(d)
    rows = np.array([0, 3, 4, 5, 22, 23, 40, L - 2, L - 1])
    got = O.softmax_window_bwd_dq_rows(rows, q, k, v, do[rows], N, mask, scale)
    tok_frame = np.arange(L) // N
    allowed = mask[tok_frame][:, tok_frame].astype(bool)
    tq = torch.tensor(q, requires_grad=True)
    out = torch.nn.functional.scaled_dot_product_attention(
        tq[None, None], torch.tensor(k)[None, None], torch.tensor(v)[None, None],
        attn_mask=torch.tensor(allowed)[None, None], scale=scale)[0, 0]
    out.backward(torch.tensor(do))
    # cotangents of the other rows do not reach these rows' dq
    np.testing.assert_allclose(got, tq.grad.numpy()[rows], rtol=1e-10, atol=1e-12)


def test_single_key_closed_form():
    # one frame of one token: the softmax weight is 1, so o_sm = v and
    # dv = do while q and k get nothing; the frame is an anchor, so the
    # linear branch is absent too
    mask = O.frame_mask(1)
    rng = np.random.default_rng(2)
    q, k, v, do = (rng.standard_normal((1, 6)) for _ in range(4))
    dq, dk, dv = O.softmax_window_bwd(q, k, v, do, 1, 1, 0, mask, 0.4)
    assert np.all(dq == 0) and np.all(dk == 0)
    np.testing.assert_allclose(dv, do, rtol=1e-15)
    g = O.linear_branch_bwd(q, k, v, do, 1, 1, 0.1, 0.5)
    assert not g["dq"].any() and not g["dk"].any() and not g["dv"].any()


def test_gate_gradient_limits():
    # with the logit at 0 (g = 1/2) the gate cotangent is (dz_sm.o_sm - dz_lin.o_lin)/4,
    # and it vanishes as the gate saturates
    rng = np.random.default_rng(4)
    B, H, L, dv, n = 1, 2, 6, 3, 4
    o_sm, o_lin = rng.standard_normal((2, B, H, L, dv))
    W1, W2 = rng.standard_normal((2, H * dv, n))
    dY = rng.standard_normal((B, L, n))
    r = O.gated_merge_bwd(o_sm, o_lin, np.zeros(H), W1, W2, dY)
    want = ((r["dz_sm"] * o_sm).sum(axis=(0, 2, 3)) - (r["dz_lin"] * o_lin).sum(axis=(0, 2, 3)))
    np.testing.assert_allclose(r["dgate_logits"], want / 4, rtol=1e-13)
    r = O.gated_merge_bwd(o_sm, o_lin, np.array([60.0, -60.0]), W1, W2, dY)
    assert np.all(np.abs(r["dgate_logits"]) < 1e-20)
