"""The block form of the symmetric sweep that the d = 128 per-frame solve uses
(besthub.dev, "Video Delta Attention (VDA)": M_f = (G_f + lambda I)^-1 of an
SPD matrix), checked on the CPU against numpy's inverse.

Sweeping a panel P of eight pivots in one step equals its eight single
sweeps: the panel column is swept alone (one panel row at a time, the pivot
row and 1 / pivot broadcast), which leaves X = [A_iP A_PP^-1; -A_PP^-1]; every
other tile takes A_ij - X_i Y_j^T with Y the panel column before the sweep,
except the pivot rows' tiles, which start from zero (A_PP^-1 A_Pj =
-X_PP Y_j^T). After every panel the matrix holds -(G + lambda I)^-1. This
test restates that algebra with numpy products, so a wrong sign, a missing
zeroing of the pivot rows or the wrong Y would fail it."""
import numpy as np
import pytest


def _single_sweeps(col, kb):
    """The eight single sweeps of panel kb on its column (d x 8)."""
    x = col.copy()
    for kr in range(8):
        k = 8 * kb + kr
        p = x[k, kr]
        assert p > 0.0
        inv = 1.0 / p
        rowk = x[k].copy()
        fr = x[:, kr] * inv
        mask = np.ones(8, bool)
        mask[kr] = False
        x[:, mask] -= np.outer(fr, rowk[mask])
        x[:, kr] = fr
        x[k] = rowk * inv
        x[k, kr] = -inv
    return x


def blocked_sweep(a):
    a = a.copy()
    d = a.shape[0]
    for kb in range(d // 8):
        P = slice(8 * kb, 8 * kb + 8)
        Y = a[:, P].copy()
        X = _single_sweeps(Y, kb)
        new = a - X @ Y.T
        new[P, :] = -X[P] @ Y.T          # pivot rows start from zero
        new[:, P] = X                    # the panel's column takes X
        a = new
    return -a


@pytest.mark.parametrize("d", [8, 32, 128])
def test_blocked_sweep_is_the_inverse(d):
    rng = np.random.default_rng(d)
    K = rng.standard_normal((3 * d, d))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    for lam in (1e-2, 1e-3):
        R = K.T @ K + lam * np.eye(d)
        M = blocked_sweep(R)
        ref = np.linalg.inv(R)
        assert np.abs(M - ref).max() <= 1e-9 * np.abs(ref).max()
        assert np.abs(M - M.T).max() <= 1e-9 * np.abs(ref).max()


def test_blocked_sweep_rank_deficient_frame():
    # 16 distinct key directions among 128 dimensions (the long-scan
    # workload's deficient frames): only lambda keeps R invertible
    rng = np.random.default_rng(7)
    basis = rng.standard_normal((16, 128))
    K = rng.standard_normal((300, 16)) @ basis
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    R = K.T @ K + 1e-3 * np.eye(128)
    M = blocked_sweep(R)
    ref = np.linalg.inv(R)
    assert np.abs(M - ref).max() <= 1e-7 * np.abs(ref).max()
