"""Shared helpers of the GPU parity tests (not collected as tests)."""

import numpy as np
import torch

import oracle as O


def np64(t):
    """torch tensor (any float dtype, any device) -> float64 numpy."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def dev(t):
    return t.cuda()


def bf16(x):
    """fp64 numpy -> torch bf16 (exact when x is already bf16-representable)."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def assert_close(got, want, atol, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    err = np.abs(got - want)
    i = int(np.argmax(err)) if err.size else 0
    assert err.size == 0 or err.max() <= atol, \
        f"{what}: max |err| {err.max():.3e} > {atol:.1e} at flat {i} (got {got.flat[i]!r}, want {want.flat[i]!r})"


def assert_bf16_close(got, want, atol, what="", ulps=1):
    """bf16 outputs: within atol, or within `ulps` bf16 ulps of the oracle
    value (a rounding flip between the fp32 kernel and the fp64 oracle at
    each of the `ulps` bf16 roundings the value went through)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    ulp = np.where(want != 0, 2.0 ** (np.floor(np.log2(np.abs(want) + 1e-300)) - 7), 2.0 ** -133)
    err = np.abs(got - want)
    bad = err > np.maximum(atol, ulps * ulp * 1.0001)
    if bad.any():
        i = int(np.argmax(bad))
        raise AssertionError(f"{what}: {int(bad.sum())} elements off; first flat {i}: got {got.flat[i]!r} "
                             f"want {want.flat[i]!r}")


def band_check(gpu_idx, ora_idx, f_oracle, tau, rel=1e-3):
    """Selected index sets agree except for candidates whose oracle score is
    within rel*tau of the oracle threshold tau."""
    g = set(np.asarray(gpu_idx).tolist())
    o = set(np.asarray(ora_idx).tolist())
    diff = g ^ o
    f = np.asarray(f_oracle, dtype=np.float64)
    out_of_band = [j for j in diff if abs(f[j] - tau) > rel * abs(tau)]
    assert not out_of_band, f"{len(out_of_band)} selections differ outside the band, e.g. {out_of_band[:5]}"
    return len(diff)
