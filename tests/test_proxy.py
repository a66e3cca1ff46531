"""Offline LTP proxy derivation (reduced-rank regression on synthetic inputs)."""

import numpy as np
import torch

from token_skipping_sparse_b200 import proxy


def test_reduced_rank_fit_recovers_an_exact_low_rank_map():
    g = torch.Generator().manual_seed(0)
    X = torch.randn(400, 32, generator=g, dtype=torch.float64)
    M = torch.randn(32, 5, generator=g, dtype=torch.float64) @ torch.randn(5, 24, generator=g, dtype=torch.float64)
    Y = X @ M
    A, B, explained = proxy.reduced_rank_fit(X, Y, 5, ridge=0.0)
    assert explained > 1 - 1e-12
    torch.testing.assert_close((X @ A.T) @ B.T, Y, rtol=1e-9, atol=1e-9)
    # a lower rank keeps the leading singular directions of the fitted values
    _, _, e3 = proxy.reduced_rank_fit(X, Y, 3, ridge=0.0)
    s = torch.linalg.svdvals(Y)
    assert abs(e3 - float((s[:3] ** 2).sum() / (s ** 2).sum())) < 1e-9


def _ffn(D=64, F=128, seed=1):
    g = torch.Generator().manual_seed(seed)
    return [(0.2 * torch.randn(o, i, generator=g)).to(torch.bfloat16) for o, i in ((F, D), (F, D), (D, F))]


def test_derived_proxy_ranks_tokens_by_ffn_change():
    wg, wu, wd = _ffn()
    A, B, ch, explained = proxy.derive_ltp_proxy(wg, wu, wd, r=16, d_low=32, n_samples=4096, seed=3)
    assert A.shape == (16, 64) and B.shape == (32, 16) and len(ch) == 32
    assert 0.0 < explained < 1.0
    # more rank explains more
    _, _, _, e_hi = proxy.derive_ltp_proxy(wg, wu, wd, r=32, d_low=32, n_samples=4096, seed=3)
    assert e_hi >= explained - 1e-9
    # on fresh inputs from the same distribution, the proxy's score orders
    # tokens by the size of their FFN change far better than a random proxy
    g = torch.Generator().manual_seed(9)
    mean = torch.randn(1, 64, generator=torch.Generator().manual_seed(3))  # the fit's offset (seed 3)
    X = mean + torch.randn(2000, 64, generator=g)
    X = X / X.pow(2).mean(dim=1, keepdim=True).sqrt()
    true = proxy.ffn_outputs(X, wg, wu, wd)[:, ch].norm(dim=1).numpy()
    est = ((X @ A.float().T) @ B.float().T).norm(dim=1).numpy()
    Ar = torch.randn(16, 64, generator=g)
    Br = torch.randn(32, 16, generator=g)
    rnd = ((X @ Ar.T) @ Br.T).norm(dim=1).numpy()

    def spearman(a, b):
        ra, rb = np.argsort(np.argsort(a)), np.argsort(np.argsort(b))
        return float(np.corrcoef(ra, rb)[0, 1])
    assert spearman(est, true) > spearman(rnd, true) + 0.2
