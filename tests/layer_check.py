"""Teacher-forced parity of one SPTS layer (helper of the GPU tests; not collected).

Every step of the layer is compared with the oracle on the inputs the GPU's
step itself received: K and the probe queries from the layer's input h, the
probe scores from the GPU's own K and probe queries, the attention rows from
the layer's input h, the O projection from the GPU's own O_sel, the LTP score and
the reduced FFN from the GPU's own h' (the output of the attention half), the
fused score and both selections from the GPU's own scores.  So every gate is
one call on the same inputs, at the per-call tolerance: 2e-2 max-abs for bf16
outputs (one bf16 ulp allowed where the output itself is stored in bf16),
1e-3 of the maximum for the fp32 scores, and bit equality for every integer
decision (a selection over given fp32 scores).  The selections are also
compared with the oracle's own scores, where they may differ only inside the
near-tie band (1e-3 of the threshold).

What the oracle's uninterrupted chain gives (its own selections and its own
roundings at every step) is reported as a drift statistic, not gated: the two
sides round their bf16 intermediates independently, so a composed output is
not one call on the same inputs.

Layers run through ``spts_layer_forward``; multi-layer pipelines (MSDP, the
Table B schedule) are replayed layer by layer on the GPU and then required to
be bit-identical to the pipeline call, so the pipeline inherits every per-layer
check.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle as O
from tests.gpu_util import assert_bf16_close, assert_close, band_check, np64

PER_CALL_TOL = 2e-2


def f64w(W):
    """CPU bf16 weight dict -> float64 numpy dict."""
    return {n: t.float().double().numpy() for n, t in W.items()}


def layer_desc(S, wl, k, sal_d=None):
    return S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, k, fuse=wl.fuse,
                        salient_rows=sal_d, salient_shift=wl.salient_shift if sal_d is not None else 0.0,
                        ltp_dout=wl.ltp_dout, ltp_top_m=wl.ltp_top_m, seq_pool=0, kv_active_only=wl.kv_active)


def gpu_layer_step(S, wl, hd, pd, Wd, k, sal_d=None):
    """One spts_layer_forward in place on the device tensors hd / pd.

    Returns (host copies of the input and of every output, the device outputs)."""
    h_in = hd.cpu()
    out = S.spts_layer_forward(hd, pd, layer_desc(S, wl, k, sal_d), Wd, outputs=True)
    S.check_device_status()
    g = {n: t.cpu() for n, t in out.items()}
    g.update(h_in=h_in, h_out=hd.cpu(), pos=pd.cpu())
    return g, out


def _norm_kv(wl, h, Wn, pos, chunk=8192):
    """xn, K, V of every row (row-wise definitions, evaluated in row chunks)."""
    N = h.shape[0]
    xn = np.empty((N, wl.D), np.float32)
    K = np.empty((N, wl.Hkv, wl.d), np.float32)
    V = np.empty((N, wl.Hkv, wl.d), np.float32)
    na = Wn.get("norm_attn")
    for a in range(0, N, chunk):
        b = min(N, a + chunk)
        x = O.bf16_round(O.rmsnorm(h[a:b], na, 1e-5))
        xn[a:b] = x
        K[a:b] = O.bf16_round(O.rope((x @ Wn["w_k"].T).reshape(b - a, wl.Hkv, wl.d), pos[a:b]))
        V[a:b] = O.bf16_round((x @ Wn["w_v"].T).reshape(b - a, wl.Hkv, wl.d))
    return xn, K, V


def _ltp(wl, x, Wn):
    if wl.ltp_top_m:
        return O.ltp_topm_scores(x, Wn["ltp_a"], Wn["ltp_b"], wl.ltp_top_m)
    return O.ltp_scores(x, Wn["ltp_a"], Wn["ltp_b"])


def _sample(n, extra, n_rows, rng):
    """All of range(n) when n_rows is None, else a sample plus the given rows."""
    if n_rows is None:
        return np.arange(n)
    return np.unique(np.concatenate([np.asarray(extra, np.int64),
                                     rng.choice(n, min(n, n_rows), replace=False)]))


def check_layer_step(wl, g, Wn, k, sal=None, n_rows=None, seed=0, drift=None, label=""):
    """Teacher-forced parity of one layer's GPU outputs ``g`` (from gpu_layer_step).

    ``Wn`` holds the float64 weights, ``k`` the active rows, ``sal`` the
    planted salient rows (numpy) or None.  ``n_rows`` None compares every row;
    otherwise each per-row step is compared on a sample of about n_rows rows
    (plus the first, the last and the probe rows).  ``drift`` (a dict) receives
    the composed-chain statistics.  Returns the number of near-tie differences
    of the two selections against the oracle's scores.
    """
    rng = np.random.default_rng(seed)
    h = g["h_in"].numpy().astype(np.float64)
    pos = g["pos"].numpy()
    N, P = h.shape[0], wl.P
    full = n_rows is None
    tag = f"{label}: " if label else ""

    # a1-a2: norm, K/V, probe queries.  K and the probe queries are bf16
    # intermediates: within 2e-2 or one bf16 ulp of the oracle's (a rounding
    # flip between the fp32 kernel and the fp64 oracle)
    xn, K, V = _norm_kv(wl, h, Wn, pos)
    qp = O.bf16_round(O.rope((xn[N - P:].astype(np.float64) @ Wn["w_q"].T).reshape(P, wl.Hq, wl.d), pos[N - P:]))
    if sal is not None and len(sal):
        K = O.inject_salience(K, qp, np.asarray(sal), wl.salient_shift, wl.Hkv)
    gk = g["k"].float().numpy()
    gqp = np64(g["q_probe"])
    salient = np.zeros(N, bool)
    if sal is not None and len(sal):
        salient[np.asarray(sal)] = True
    for a in range(0, N, 16384):
        b = min(N, a + 16384)
        plain = ~salient[a:b]
        assert_bf16_close(gk[a:b][plain], K[a:b][plain], PER_CALL_TOL, tag + "K")
        # salient keys are rounded to bf16 twice: after RoPE and after the shift
        assert_bf16_close(gk[a:b][~plain], K[a:b][~plain], PER_CALL_TOL, tag + "K (salient rows)", ulps=2)
    assert_bf16_close(gqp, qp, PER_CALL_TOL, tag + "probe queries")
    # a3-a4: the probe scores on the GPU's own keys and probe queries (a
    # one-ulp flip of one key element moves that key's weight in every probe
    # row, so the oracle's own K would not be the same input), the MHA selection
    s, _ = O.probe_scores(gqp, pos[N - P:], gk, pos)
    gs = g["s"].numpy()
    assert_close(gs, s, 1e-3 * s.max(), tag + "probe scores")
    assert abs(gs.astype(np.float64).sum() - P * wl.Hq) < 1e-3 * P * wl.Hq, tag + "probe score sum"
    ia = g["idx_attn"].numpy()
    assert np.array_equal(ia, O.select_topk(gs, k, P)[0]), tag + "MHA selection of the GPU's own scores"
    oidx, tau = O.select_topk(s.astype(np.float32), k, P)
    n_ties = band_check(ia, oidx, s, tau)

    # a5-a6: Q of the selected rows, reduced attention
    pick = _sample(k, [0, k - 1, *range(k - P, k)], None if full else n_rows, rng)
    rows = ia[pick]
    q = O.bf16_round(O.rope((xn[rows].astype(np.float64) @ Wn["w_q"].T).reshape(len(rows), wl.Hq, wl.d), pos[rows]))
    Kk, Vk, pk = (K[ia], V[ia], pos[ia]) if wl.kv_active else (K, V, pos)
    o = O.bf16_round(O.reduced_attention(q, pos[rows], Kk, Vk, pk))
    g_osel = np64(g["o_sel"][torch.from_numpy(pick)])
    assert_bf16_close(g_osel, o, PER_CALL_TOL, tag + "o_sel rows")

    # a7: O projection into the selected rows, on the GPU's own O_sel
    ha = g["h_attn"].numpy()
    want_ha = h[rows] + g_osel.reshape(len(rows), -1) @ Wn["w_o"].T
    assert_close(ha[rows], want_ha, PER_CALL_TOL, tag + "h after attention (selected rows)")
    skip = np.setdiff1d(np.arange(N), ia)
    assert np.array_equal(ha[skip], g["h_in"].numpy()[skip]), tag + "rows skipped by attention changed"
    if drift is not None:
        chain = h[rows] + o.reshape(len(rows), -1) @ Wn["w_o"].T
        drift["h_attn"] = max(drift.get("h_attn", 0.0), float(np.abs(ha[rows] - chain).max()))
    ho = g["h_out"].numpy()
    if not wl.F:
        assert np.array_equal(ho, ha), tag + "attention-only layer: h_out != h'"
        return n_ties

    # a8: LTP score of RMSNorm(h') on the GPU's own h'
    idf = g["idx_ffn"].numpy()
    rr = _sample(N, [*range(N - P, N), *idf[rng.choice(k, min(k, max(1, (n_rows or 0) // 2)), replace=False)]],
                 None if full else max(1, n_rows // 2), rng)
    x2 = O.bf16_round(O.rmsnorm(ha[rr].astype(np.float64), Wn.get("norm_ffn"), 1e-5))
    c = _ltp(wl, x2, Wn)
    gc = g["c"].numpy()
    assert_close(gc[rr], c, 1e-3 * c.max(), tag + "ltp scores")

    # a9: fusion and the FFN selection on the GPU's own scores (exact), and
    # against the oracle's scores (near-ties only) where the oracle has them all
    gf = g["f"].numpy()
    if wl.fuse == O.FUSE_SEQUENTIAL:
        assert np.array_equal(gf.view(np.uint32), gc.view(np.uint32)), tag + "sequential: f is c"
        want_idf = O.select_sequential(gs, gc, min(N, 2 * k), k, P)[0]
        assert np.array_equal(idf, want_idf), tag + "sequential FFN selection"
    else:
        f_want = O.fuse_scores(gs, gc, wl.fuse, 0.5, 0.5)
        assert np.array_equal(gf.view(np.uint32), f_want.view(np.uint32)), tag + "fused score (bitwise)"
        assert np.array_equal(idf, O.select_topk(f_want, k, P)[0]), tag + "FFN selection of the GPU's own scores"
        if full:
            f_or = O.fuse_scores(s.astype(np.float32), c.astype(np.float32), wl.fuse, 0.5, 0.5)
            oi, tf = O.select_topk(f_or, k, P)
            n_ties += band_check(idf, oi, f_or, tf)

    # a10: reduced FFN on the GPU's own h'
    fsel = rr[np.isin(rr, idf)]
    assert len(fsel) > 0
    want = O.reduced_ffn(ha[fsel].astype(np.float64), np.arange(len(fsel)), Wn.get("norm_ffn"), 1e-5,
                         Wn["w_gate"], Wn["w_up"], Wn["w_down"])
    assert_close(ho[fsel], want, PER_CALL_TOL, tag + "h out (reduced FFN rows)")
    skip = np.setdiff1d(np.arange(N), idf)
    assert np.array_equal(ho[skip], ha[skip]), tag + "rows skipped by the FFN changed"
    if drift is not None:
        # the oracle's own chain on these rows: its O_sel, then its FFN
        h1 = h[fsel].copy()
        at = np.isin(fsel, ia)
        if at.any():
            ra = fsel[at]
            qa = O.bf16_round(O.rope((xn[ra].astype(np.float64) @ Wn["w_q"].T).reshape(len(ra), wl.Hq, wl.d),
                                     pos[ra]))
            oa = O.bf16_round(O.reduced_attention(qa, pos[ra], Kk, Vk, pk))
            h1[at] += oa.reshape(len(ra), -1) @ Wn["w_o"].T
        chain = O.reduced_ffn(h1, np.arange(len(fsel)), Wn.get("norm_ffn"), 1e-5, Wn["w_gate"], Wn["w_up"],
                              Wn["w_down"])
        drift["h_out"] = max(drift.get("h_out", 0.0), float(np.abs(ho[fsel] - chain).max()))
    return n_ties
