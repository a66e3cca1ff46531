"""Offline derivation of the LTP low-rank proxy (the step before the hot path).

LTP scores a token by a low-rank proxy of the FFN's transformation, y =
(x A^T) B^T with A [r, D] and B [D_low, r] ("Probe and Skip: Self-Predictive
Token Skipping for Efficient Long-Context LLM Inference", Fig. 2(b); the
proxy is derived offline and D_low, r are Table A's).  The pages fit it on
calibration data; without a dataset this module fits it by reduced-rank
regression on synthetic FFN inputs:

1. draw inputs X [n, D] around a fixed offset direction (unit-RMS rows: the
   FFN input after RMSNorm with weight 1) and compute the FFN output
   Y = W_down (silu(W_gate x) * W_up x) for every row.  Hidden states of a
   trained model are not centred; around a zero mean a SwiGLU has no linear
   part at all (silu(g) u is even to first order), so the offset is what a
   linear proxy can capture (reading; ``offset`` = 0 gives centred inputs);
2. keep the D_low output channels with the largest energy sum_i Y_ij^2
   (Table A's channel-reduced proxy; all D channels when d_low is None);
3. least squares W = argmin ||X W - Y_sel|| (a small ridge keeps it well
   posed), then the best rank-r approximation of the fitted values X W by a
   truncated SVD: X W ~ U_r S_r V_r^T gives W_r = W V_r V_r^T, so
   A = (W V_r)^T [r, D] and B = V_r [D_low, r].

The result is returned in bf16 as the layer consumes it, with the chosen
channel indices.  Plain PyTorch linear algebra on the given device: this runs
once per model, not per token.
"""

from __future__ import annotations

import torch

__all__ = ["ffn_outputs", "reduced_rank_fit", "calibration_inputs", "derive_ltp_proxy"]


def ffn_outputs(x, w_gate, w_up, w_down):
    """SwiGLU FFN outputs for rows x (fp32 math on the given tensors)."""
    x = x.float()
    g = x @ w_gate.float().T
    u = x @ w_up.float().T
    return (torch.nn.functional.silu(g) * u) @ w_down.float().T


def reduced_rank_fit(X, Y, r, ridge=1e-4):
    """Best rank-r linear map X -> Y in least squares (fp64): returns
    (A [r, D], B [Dy, r], explained) with Y ~ (X A^T) B^T."""
    Xd, Yd = X.double(), Y.double()
    D = Xd.shape[1]
    G = Xd.T @ Xd
    G += ridge * torch.trace(G) / D * torch.eye(D, device=Xd.device, dtype=torch.float64)
    W = torch.linalg.solve(G, Xd.T @ Yd)                   # [D, Dy]
    _, _, Vh = torch.linalg.svd(Xd @ W, full_matrices=False)
    B = Vh[:r].T                                            # [Dy, r], orthonormal columns
    A = (W @ B).T                                           # [r, D]
    approx = (Xd @ A.T) @ B.T
    explained = 1.0 - float((approx - Yd).pow(2).sum() / Yd.pow(2).sum())
    return A, B, explained


def calibration_inputs(D, n_samples=8192, seed=0, offset=1.0, device="cpu"):
    """Synthetic FFN inputs [n_samples, D]: a fixed random offset direction
    (scaled by ``offset``) plus N(0, 1) noise, each row scaled to unit RMS."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    mean = torch.randn(1, D, generator=g, device=device, dtype=torch.float32) * offset
    X = mean + torch.randn(n_samples, D, generator=g, device=device, dtype=torch.float32)
    return X / X.pow(2).mean(dim=1, keepdim=True).sqrt()      # unit RMS rows, as after RMSNorm


def derive_ltp_proxy(w_gate, w_up, w_down, r, d_low=None, n_samples=8192, seed=0, ridge=1e-4, offset=1.0,
                     chunk=2048, X=None, exact=False):
    """Fit the LTP proxy of one FFN.

    Returns (A [r, D] bf16, B [d_low, r] bf16, channels [d_low] int64,
    explained) where ``explained`` is the share of the selected channels'
    output energy that the rank-r proxy reproduces on the samples.  ``X``
    replaces the drawn calibration inputs; ``exact`` returns A and B in fp64.
    """
    dev = w_gate.device
    if X is None:
        X = calibration_inputs(w_gate.shape[1], n_samples, seed, offset, dev)
    n = X.shape[0]
    Y = torch.cat([ffn_outputs(X[i:i + chunk], w_gate, w_up, w_down) for i in range(0, n, chunk)])
    if d_low is None or d_low >= Y.shape[1]:
        channels = torch.arange(Y.shape[1], device=dev)
    else:  # the d_low channels of largest output energy, equal energies to the lower channel
        channels = torch.argsort(-Y.double().pow(2).sum(dim=0), stable=True)[:d_low].sort().values
    A, B, explained = reduced_rank_fit(X, Y[:, channels], r, ridge)
    if exact:
        return A, B, channels, explained
    return A.to(torch.bfloat16), B.to(torch.bfloat16), channels, explained
