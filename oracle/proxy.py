"""fp64 oracle of the offline LTP proxy derivation (test infrastructure only).

Fig. 2(b) of "Probe and Skip: Self-Predictive Token Skipping for Efficient
Long-Context LLM Inference" scores tokens with a low-rank proxy of the FFN's
transformation, y = (x A^T) B^T, which the method derives offline; Table A
sets its rank r and the number D_low of output channels it predicts.  The
pages do not print the fitting procedure, and the calibration data of their
Tables G/H is not available here.  Reading taken (the plainest one the pages
support): given calibration inputs X [n, D] (FFN inputs) and the FFN's outputs
Y = FFN(X),

1. keep the D_low output channels with the largest energy sum_i Y_ij^2
   (ties to the lower channel index), in ascending channel order;
2. fit the best rank-r linear map from X to those channels in least squares
   -- reduced-rank regression: the full least-squares map W (with a ridge
   term lambda * I, lambda = ridge * trace(X^T X) / D, to keep it well posed),
   then the rank-r map that is closest on the calibration set, W V_r V_r^T,
   where V_r holds the leading r right singular vectors of the fitted values
   X W;
3. A = (W V_r)^T [r, D], B = V_r [D_low, r].

The calibration inputs are an input here (the random draw lives with the
caller), so this file holds only the arithmetic of the fit.  Every function
is pinned in tests/test_oracle_proxy.py.
"""

from __future__ import annotations

import numpy as np

__all__ = ["ffn_outputs", "select_channels", "reduced_rank_regression", "fit_proxy"]


def ffn_outputs(X, w_gate, w_up, w_down):
    """SwiGLU FFN outputs W_down (silu(W_gate x) * W_up x) for every row of X (fp64)."""
    X = np.asarray(X, dtype=np.float64)
    g = X @ np.asarray(w_gate, dtype=np.float64).T
    u = X @ np.asarray(w_up, dtype=np.float64).T
    return (g / (1.0 + np.exp(-g)) * u) @ np.asarray(w_down, dtype=np.float64).T


def select_channels(Y, d_low):
    """Indices of the d_low columns of Y with the largest sum of squares
    (equal energies: the lower index first), ascending; all columns when
    d_low is None or not below the column count."""
    Y = np.asarray(Y, dtype=np.float64)
    n_out = Y.shape[1]
    if d_low is None or d_low >= n_out:
        return np.arange(n_out)
    energy = np.sum(Y * Y, axis=0)
    order = np.argsort(-energy, kind="stable")
    return np.sort(order[:d_low])


def reduced_rank_regression(X, Y, r, ridge=0.0):
    """The rank-r map closest to Y on X in least squares.

    Returns (A [r, D], B [Dy, r], explained): Y ~ (X A^T) B^T, and the share
    of Y's energy the rank-r fit reproduces, 1 - ||X A^T B^T - Y||^2 / ||Y||^2.
    """
    X = np.asarray(X, dtype=np.float64)
    Y = np.asarray(Y, dtype=np.float64)
    D = X.shape[1]
    G = X.T @ X
    lam = ridge * np.trace(G) / D
    W = np.linalg.solve(G + lam * np.eye(D), X.T @ Y)        # full least-squares map [D, Dy]
    _, _, Vt = np.linalg.svd(X @ W, full_matrices=False)   # fitted values: leading right singular vectors
    V_r = Vt[:r].T                                          # [Dy, r]
    A = (W @ V_r).T
    B = V_r
    resid = X @ A.T @ B.T - Y
    explained = 1.0 - float(np.sum(resid * resid) / np.sum(Y * Y))
    return A, B, explained


def fit_proxy(X, w_gate, w_up, w_down, r, d_low=None, ridge=1e-4):
    """The LTP proxy of one FFN from calibration inputs X: (A, B, channels, explained)."""
    Y = ffn_outputs(X, w_gate, w_up, w_down)
    ch = select_channels(Y, d_low)
    A, B, explained = reduced_rank_regression(X, Y[:, ch], r, ridge)
    return A, B, ch, explained
