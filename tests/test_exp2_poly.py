"""The FMA-pipe exp2 of the reduced-attention softmax (exp2_poly2 in csrc/sm100.cuh).

CPU: the four constants compiled into the kernel are the fp32 roundings of
the minimax fit that token_skipping_sparse_b200/exp2_poly_fit.py derives, and
that fit's error bound holds.  GPU: the device function against exp2 in
float64 over [-126, 0] within the bound, exact 0 for -inf and below -127,
exact 1 at 0, and tiny non-negative values in between."""

import os
import re
import importlib.util

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUND = 1.02e-4


def _fit_module():
    spec = importlib.util.spec_from_file_location(
        "exp2_poly_fit", os.path.join(ROOT, "token_skipping_sparse_b200", "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_kernel_constants_are_the_fit():
    m = _fit_module()
    c, t = m.fit()
    assert t < BOUND
    src = open(os.path.join(ROOT, "token_skipping_sparse_b200", "csrc", "sm100.cuh")).read()
    body = src[src.index("void exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    consts = [float(v) for v in re.findall(r"f2pack\(([0-9.e+-]+)f, \1f\)", body)]
    # the shifter 1.5 * 2^23 and its negative, the -1, then c3, c2, c1, c0 in Horner order
    poly = [v for v in consts if abs(v) < 2.0 and v != -1.0]
    want = np.asarray(c[::-1], dtype=np.float32)
    assert np.array_equal(np.asarray(poly, dtype=np.float32), want), (poly, want)
    f = np.linspace(-0.5, 0.5, 100001, dtype=np.float32)
    err = np.abs(m.horner_fp32(want[::-1], f).astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0).max()
    assert err < BOUND


@pytest.mark.gpu
def test_device_exp2_poly_within_its_bound():
    import token_skipping_sparse_b200 as S
    x = torch.linspace(-126.0, 0.0, 2_000_001, dtype=torch.float32, device="cuda")
    y = S.debug_exp2_poly(x).double().cpu()
    want = torch.exp2(x.double().cpu())
    assert float(((y / want) - 1).abs().max()) < BOUND
    # the special inputs: -inf and anything clamped to -127 give exactly 0, 0 gives 1
    sp = torch.tensor([float("-inf"), -1e30, -127.0, -500.0, 0.0, -1.0, -0.5], device="cuda")
    ys = S.debug_exp2_poly(sp).cpu()
    assert ys[:4].tolist() == [0.0, 0.0, 0.0, 0.0]
    assert ys[4].item() == 1.0
    assert abs(ys[5].item() - 0.5) <= BOUND * 0.5 and abs(ys[6].item() - 2 ** -0.5) <= BOUND
    low = torch.linspace(-127.0, -126.0, 10001, device="cuda")
    yl = S.debug_exp2_poly(low).cpu()
    assert torch.isfinite(yl).all() and (yl >= 0).all() and (yl < 2.0 ** -125).all()
    S.check_device_status()
