"""Pins of the proxy-derivation oracle (oracle/proxy.py), and the product's
offline derivation (token_skipping_sparse_b200/proxy.py) against it.

Pins, each fixed by something other than the oracle itself:
  * an exact rank-r map is recovered exactly (closed form);
  * a lower rank keeps the leading singular directions: its explained share
    is the Eckart-Young ratio of Y's singular values (numpy's SVD);
  * full rank without ridge is ordinary least squares (numpy's lstsq);
  * full rank with ridge is ridge regression (scikit-learn's Ridge);
  * with X = I the fit is the truncated SVD of Y (textbook special case);
  * no random rank-r perturbation of the fitted map lowers the residual;
  * noise orthogonal to X's columns leaves the fit unchanged (Eckart-Young
    on the fitted values, numpy's QR and lstsq);
  * the channel choice is brute-force top energy with ties to the lower index;
  * the FFN outputs are torch's F.linear / F.silu composition.
Each of a set of planted mistakes (run on the CPU) makes at least one pin fail.
"""

import numpy as np
import pytest
import torch

import oracle.proxy as OP

_ORIG = {n: getattr(OP, n) for n in ("ffn_outputs", "select_channels", "reduced_rank_regression")}


def _rng(seed=0):
    return np.random.default_rng(seed)


def _low_rank_case(n=300, D=24, Dy=18, rank=5, seed=0):
    g = _rng(seed)
    X = g.standard_normal((n, D))
    M = g.standard_normal((D, rank)) @ g.standard_normal((rank, Dy))
    return X, M


# ---------------------------------------------------------------- pins
def pin_exact_low_rank_map_recovered():
    X, M = _low_rank_case()
    A, B, explained = OP.reduced_rank_regression(X, X @ M, 5)
    assert A.shape == (5, 24) and B.shape == (18, 5)
    assert explained > 1 - 1e-12
    np.testing.assert_allclose(A.T @ B.T, M, rtol=0, atol=1e-9)


def pin_lower_rank_is_eckart_young():
    X, M = _low_rank_case(seed=1)
    Y = X @ M
    s = np.linalg.svd(Y, compute_uv=False)
    for r in (1, 2, 3, 4):
        _, _, e = OP.reduced_rank_regression(X, Y, r)
        assert abs(e - float(np.sum(s[:r] ** 2) / np.sum(s ** 2))) < 1e-10


def pin_full_rank_is_least_squares():
    g = _rng(2)
    X, Y = g.standard_normal((200, 12)), g.standard_normal((200, 7))
    A, B, _ = OP.reduced_rank_regression(X, Y, 7)
    W, *_ = np.linalg.lstsq(X, Y, rcond=None)
    np.testing.assert_allclose(A.T @ B.T, W, rtol=0, atol=1e-10)


def pin_full_rank_with_ridge_is_ridge_regression():
    from sklearn.linear_model import Ridge
    g = _rng(3)
    X, Y = g.standard_normal((150, 10)), g.standard_normal((150, 6))
    ridge = 0.05
    A, B, _ = OP.reduced_rank_regression(X, Y, 6, ridge=ridge)
    alpha = ridge * np.trace(X.T @ X) / X.shape[1]
    W = Ridge(alpha=alpha, fit_intercept=False, solver="svd").fit(X, Y).coef_.T
    np.testing.assert_allclose(A.T @ B.T, W, rtol=0, atol=1e-10)


def pin_identity_design_is_truncated_svd():
    g = _rng(4)
    Y = g.standard_normal((16, 11))
    U, s, Vt = np.linalg.svd(Y, full_matrices=False)
    for r in (1, 3, 6):
        A, B, _ = OP.reduced_rank_regression(np.eye(16), Y, r)
        np.testing.assert_allclose(A.T @ B.T, (U[:, :r] * s[:r]) @ Vt[:r], rtol=0, atol=1e-10)


def pin_no_rank_r_perturbation_does_better():
    g = _rng(5)
    X, Y = g.standard_normal((120, 9)), g.standard_normal((120, 8))
    r = 3
    A, B, _ = OP.reduced_rank_regression(X, Y, r)
    best = np.sum((X @ A.T @ B.T - Y) ** 2)
    for step in (0.05, 1e-4):      # small steps see a gradient, large ones a curvature
        for _ in range(100):
            A2 = A + step * g.standard_normal(A.shape)
            B2 = B + step * g.standard_normal(B.shape)
            assert np.sum((X @ A2.T @ B2.T - Y) ** 2) >= best - 1e-9


def pin_noise_outside_the_column_space_does_not_move_the_fit():
    """Y = X M + E with E orthogonal to X's columns: the fit is the rank-r
    truncated SVD of X M (Eckart-Young), whatever E is."""
    X, M = _low_rank_case(n=200, D=10, Dy=8, rank=8, seed=8)
    Q, _ = np.linalg.qr(X)
    N = 3.0 * _rng(9).standard_normal((200, 8))
    E = N - Q @ (Q.T @ N)
    U, s, Vt = np.linalg.svd(X @ M, full_matrices=False)
    for r in (2, 5):
        A, B, _ = OP.reduced_rank_regression(X, X @ M + E, r)
        want, *_ = np.linalg.lstsq(X, (U[:, :r] * s[:r]) @ Vt[:r], rcond=None)
        np.testing.assert_allclose(A.T @ B.T, want, rtol=0, atol=1e-9)


def pin_channel_choice_is_top_energy():
    g = _rng(6)
    for trial in range(30):
        Y = g.integers(-2, 3, size=(5, 9)).astype(np.float64)      # many equal energies
        d_low = int(g.integers(1, 9))
        energy = (Y * Y).sum(axis=0)
        want = sorted(sorted(range(9), key=lambda j: (-energy[j], j))[:d_low])
        assert OP.select_channels(Y, d_low).tolist() == want
    assert OP.select_channels(Y, None).tolist() == list(range(9))
    assert OP.select_channels(Y, 9).tolist() == list(range(9))


def pin_ffn_outputs_are_the_swiglu_ffn():
    g = torch.Generator().manual_seed(7)
    x = torch.randn(20, 16, generator=g, dtype=torch.float64)
    wg, wu = (torch.randn(24, 16, generator=g, dtype=torch.float64) for _ in range(2))
    wd = torch.randn(16, 24, generator=g, dtype=torch.float64)
    F = torch.nn.functional
    want = F.linear(F.silu(F.linear(x, wg)) * F.linear(x, wu), wd).numpy()
    np.testing.assert_allclose(OP.ffn_outputs(x.numpy(), wg.numpy(), wu.numpy(), wd.numpy()), want, rtol=1e-12,
                               atol=1e-12)


PINS = [pin_exact_low_rank_map_recovered, pin_lower_rank_is_eckart_young, pin_full_rank_is_least_squares,
        pin_full_rank_with_ridge_is_ridge_regression, pin_identity_design_is_truncated_svd,
        pin_no_rank_r_perturbation_does_better, pin_noise_outside_the_column_space_does_not_move_the_fit,
        pin_channel_choice_is_top_energy,
        pin_ffn_outputs_are_the_swiglu_ffn]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin()


# ---------------------------------------------------------------- planted mistakes
def _rrr(X, Y, r, ridge=0.0, no_truncation=False, from_y=False, transposed_b=False):
    X, Y = np.asarray(X, dtype=np.float64), np.asarray(Y, dtype=np.float64)
    D = X.shape[1]
    G = X.T @ X
    W = np.linalg.solve(G + ridge * np.trace(G) / D * np.eye(D), X.T @ Y)
    _, _, Vt = np.linalg.svd(Y if from_y else X @ W, full_matrices=False)
    V = Vt.T if no_truncation else Vt[:r].T
    A, B = (W @ V).T, V
    if transposed_b:
        B = B[::-1]
    res = X @ A.T @ B.T - Y
    return A, B, 1.0 - float(np.sum(res * res) / np.sum(Y * Y))


MUTANTS = {
    "rrr_svd_of_y_not_fitted_values": ("reduced_rank_regression", lambda X, Y, r, ridge=0.0: _rrr(X, Y, r, ridge, from_y=True)),
    "rrr_no_truncation": ("reduced_rank_regression", lambda X, Y, r, ridge=0.0: _rrr(X, Y, r, ridge, no_truncation=True)),
    "rrr_output_rows_reversed": ("reduced_rank_regression", lambda X, Y, r, ridge=0.0: _rrr(X, Y, r, ridge, transposed_b=True)),
    "rrr_ridge_unscaled": ("reduced_rank_regression",
                           lambda X, Y, r, ridge=0.0: _rrr(X, Y, r, ridge * X.shape[1] / max(np.trace(np.asarray(X).T @ np.asarray(X)), 1e-300))),
    "rrr_trailing_directions": ("reduced_rank_regression",
                                lambda X, Y, r, ridge=0.0: (lambda A, B: (A, B, 0.0))(*_trailing(X, Y, r, ridge))),
    "channels_lowest_energy": ("select_channels",
                               lambda Y, d_low: (np.arange(np.asarray(Y).shape[1]) if d_low is None or d_low >= np.asarray(Y).shape[1]
                                                 else np.sort(np.argsort((np.asarray(Y) ** 2).sum(0), kind="stable")[:d_low]))),
    "channels_ties_high": ("select_channels",
                           lambda Y, d_low: (np.arange(np.asarray(Y).shape[1]) if d_low is None or d_low >= np.asarray(Y).shape[1]
                                             else np.sort((np.asarray(Y).shape[1] - 1 - np.argsort(-((np.asarray(Y) ** 2).sum(0))[::-1], kind="stable"))[:d_low]))),
    "channels_by_abs_sum": ("select_channels",
                            lambda Y, d_low: (np.arange(np.asarray(Y).shape[1]) if d_low is None or d_low >= np.asarray(Y).shape[1]
                                              else np.sort(np.argsort(-np.abs(np.asarray(Y)).sum(0), kind="stable")[:d_low]))),
    "ffn_gate_and_up_swapped": ("ffn_outputs", lambda X, wg, wu, wd: _ORIG["ffn_outputs"](X, wu, wg, wd)),
    "ffn_relu": ("ffn_outputs", lambda X, wg, wu, wd: (np.maximum(np.asarray(X) @ np.asarray(wg).T, 0) * (np.asarray(X) @ np.asarray(wu).T)) @ np.asarray(wd).T),
}


def _trailing(X, Y, r, ridge):
    X, Y = np.asarray(X, dtype=np.float64), np.asarray(Y, dtype=np.float64)
    D = X.shape[1]
    G = X.T @ X
    W = np.linalg.solve(G + ridge * np.trace(G) / D * np.eye(D), X.T @ Y)
    _, _, Vt = np.linalg.svd(X @ W, full_matrices=False)
    V = Vt[-r:].T
    return (W @ V).T, V


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    fn_name, mutant = MUTANTS[name]
    monkeypatch.setattr(OP, fn_name, mutant)
    caught = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, np.linalg.LinAlgError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the mutant {name}"


# ---------------------------------------------------------------- the product against the oracle
def test_product_derivation_matches_the_oracle():
    """token_skipping_sparse_b200.proxy on the same calibration inputs: the
    same channels, the same rank-r map and the same explained share."""
    from token_skipping_sparse_b200 import proxy as PP
    g = torch.Generator().manual_seed(11)
    D, F = 64, 160
    wg, wu = ((0.2 * torch.randn(F, D, generator=g)).to(torch.bfloat16) for _ in range(2))
    wd = (0.2 * torch.randn(D, F, generator=g)).to(torch.bfloat16)
    X = PP.calibration_inputs(D, 3000, seed=4)
    for r, d_low in ((8, 32), (16, None)):
        A, B, ch, e = PP.derive_ltp_proxy(wg, wu, wd, r, d_low, X=X, exact=True)
        oA, oB, och, oe = OP.fit_proxy(X.double().numpy(), wg.double().numpy(), wu.double().numpy(),
                                       wd.double().numpy(), r, d_low, ridge=1e-4)
        assert np.array_equal(ch.numpy(), och)
        M, oM = (A.T @ B.T).numpy(), oA.T @ oB.T
        # the product evaluates the FFN in fp32, the oracle in fp64
        assert np.abs(M - oM).max() <= 1e-4 * np.abs(oM).max()
        assert abs(e - oe) < 1e-5
