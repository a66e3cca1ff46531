"""Parity at the full sizes of the workloads, in the launch configuration
bench.py times (the same inputs, the same C-ABI calls).

At these sizes the oracle computes every step whose inputs are synthetic in
full (norm, K/V projections, probe scores, the MHA selection), and the
per-row steps (reduced attention, O projection, LTP score, reduced FFN) for
sampled rows, one by one.  Everything else is checked through properties that
hold at any size: skipped rows are bit-exact, selections are valid top-k sets
of the kernel's own scores with the forced tail, and MSDP candidate sets nest.
"""

import numpy as np
import pytest
import torch

import oracle as O
from synthetic import WORKLOADS, keep_rows, make_hidden, make_layer_weights, salient_rows
from tests.gpu_util import assert_bf16_close, assert_close, band_check, np64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import token_skipping_sparse_b200 as S


PER_CALL_TOL = 2e-2     # bf16 outputs of one call given the same inputs
LAYER_OUT_TOL = 4e-2    # the layer output: two bf16-stored stages composed


def _f64(t):
    return t.float().double().numpy()


def _oracle_norm_kv(wl, h, W, pos, chunk=8192):
    """xn, K, V for every row (row-wise definitions, evaluated in row chunks)."""
    N = h.shape[0]
    xn = np.empty((N, wl.D), np.float32)
    K = np.empty((N, wl.Hkv, wl.d), np.float32)
    V = np.empty((N, wl.Hkv, wl.d), np.float32)
    for a in range(0, N, chunk):
        b = min(N, a + chunk)
        x = O.bf16_round(O.rmsnorm(h[a:b].astype(np.float64), None, 1e-5))
        xn[a:b] = x
        K[a:b] = O.bf16_round(O.rope((x @ W["w_k"].T).reshape(b - a, wl.Hkv, wl.d), pos[a:b]))
        V[a:b] = O.bf16_round((x @ W["w_v"].T).reshape(b - a, wl.Hkv, wl.d))
    return xn, K, V


def _check_topk_valid(idx, f, k, tail):
    """idx is the top-k set of f under the tie rule, tail forced, ascending."""
    idx = np.asarray(idx)
    Nc = len(f)
    assert len(idx) == k and np.all(np.diff(idx) > 0)
    assert set(range(Nc - tail, Nc)) <= set(idx.tolist())
    free = idx[idx < Nc - tail]
    sel = np.zeros(Nc - tail, bool)
    sel[free] = True
    fz = np.where(f[:Nc - tail] == 0, 0.0, f[:Nc - tail]).astype(np.float64)
    if sel.any() and (~sel).any():
        lo = fz[sel].min()
        hi = fz[~sel].max()
        assert lo >= hi
        if lo == hi:  # equal scores: every kept one precedes every dropped one
            assert np.where(sel & (fz == lo))[0].max() < np.where(~sel & (fz == hi))[0].min()


def _run_gpu_layer(wl, h, W, pos, sal, k=None):
    Wd = {n: t.cuda() for n, t in W.items()}
    sal_d = sal.cuda() if len(sal) else None
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, wl.k if k is None else k, fuse=wl.fuse,
                        salient_rows=sal_d, salient_shift=wl.salient_shift, ltp_dout=wl.ltp_dout, ltp_top_m=wl.ltp_top_m, seq_pool=0,
                        kv_active_only=wl.kv_active)
    hd = h.cuda()
    out = S.spts_layer_forward(hd, pos.cuda(), desc, Wd, outputs=True)
    S.check_device_status()
    res = {n: t.cpu() for n, t in out.items()}
    res["h_out"] = hd.cpu()
    del hd, Wd
    torch.cuda.empty_cache()
    return res


def _check_layer_sampled(wl, h, W, pos, sal, g, k, n_rows=40):
    """Sampled parity of one layer's GPU outputs `g` against the oracle."""
    rng = np.random.default_rng(0)
    Wn = {n: _f64(t) for n, t in W.items()}
    N, P = h.shape[0], wl.P
    pos_n = pos.numpy()
    h64 = h.numpy().astype(np.float64)
    xn, K, V = _oracle_norm_kv(wl, h.numpy(), Wn, pos_n)
    qp = O.bf16_round(O.rope((xn[N - P:].astype(np.float64) @ Wn["w_q"].T).reshape(P, wl.Hq, wl.d), pos_n[N - P:]))
    if len(sal):
        K = O.inject_salience(K, qp, sal.numpy(), wl.salient_shift, wl.Hkv)
    s, _ = O.probe_scores(qp, pos_n[N - P:], K, pos_n)
    gs = g["s"].numpy()
    assert_close(gs, s, 1e-3 * s.max(), "probe scores")
    assert abs(gs.astype(np.float64).sum() - P * wl.Hq) < 1e-3 * P * wl.Hq
    ia = g["idx_attn"].numpy()
    oidx, tau = O.select_topk(s.astype(np.float32), k, P)
    band_check(ia, oidx, s, tau)
    _check_topk_valid(ia, gs, k, P)

    # reduced attention and O projection on sampled selected rows
    pick = np.unique(np.concatenate([[0, len(ia) - 1], np.arange(len(ia) - P, len(ia)),
                                     rng.choice(len(ia), n_rows, replace=False)]))
    rows = ia[pick]
    q = O.bf16_round(O.rope((xn[rows].astype(np.float64) @ Wn["w_q"].T).reshape(len(rows), wl.Hq, wl.d),
                            pos_n[rows]))
    # the keys: every candidate, or (kv_active) the GPU's active rows
    Kk, Vk, pk = (K[ia], V[ia], pos_n[ia]) if wl.kv_active else (K, V, pos_n)
    o = O.bf16_round(O.reduced_attention(q, pos_n[rows], Kk, Vk, pk))
    assert_bf16_close(np64(g["o_sel"][pick]), o, 2e-2, "o_sel rows")
    h1_rows = h64[rows] + o.reshape(len(rows), -1) @ Wn["w_o"].T
    ha = g["h_attn"].numpy()
    assert_close(ha[rows], h1_rows, 2e-2, "h after attention (selected rows)")
    skip = np.setdiff1d(np.arange(N), ia)
    assert np.array_equal(ha[skip], h.numpy()[skip]), "rows skipped by attention changed"
    if not wl.F:
        return

    # LTP score on sampled rows (the oracle recomputes each row's h')
    def oracle_h1(rr):
        out = h64[rr].copy()
        sel = np.isin(rr, ia)
        if sel.any():
            rs = rr[sel]
            qq = O.bf16_round(O.rope((xn[rs].astype(np.float64) @ Wn["w_q"].T).reshape(len(rs), wl.Hq, wl.d),
                                     pos_n[rs]))
            oo = O.bf16_round(O.reduced_attention(qq, pos_n[rs], Kk, Vk, pk))
            out[sel] += oo.reshape(len(rs), -1) @ Wn["w_o"].T
        return out

    idf = g["idx_ffn"].numpy()
    rr = np.unique(np.concatenate([rng.choice(N, n_rows // 2, replace=False),
                                   idf[rng.choice(len(idf), n_rows // 2, replace=False)], np.arange(N - P, N)]))
    h1 = oracle_h1(rr)
    x2 = O.bf16_round(O.rmsnorm(h1, None, 1e-5))
    c = (O.ltp_topm_scores(x2, Wn["ltp_a"], Wn["ltp_b"], wl.ltp_top_m) if wl.ltp_top_m
         else O.ltp_scores(x2, Wn["ltp_a"], Wn["ltp_b"]))
    gc = g["c"].numpy()
    assert_close(gc[rr], c, 1e-3 * c.max(), "ltp scores (sampled rows)")
    if wl.fuse == O.FUSE_SEQUENTIAL:  # the pool by s, then the k by c (the kernel's own scores)
        want_f = O.select_sequential(gs, gc, min(N, 2 * k), k, P)[0]
        assert np.array_equal(idf, want_f), "sequential FFN selection"
    else:
        _check_topk_valid(idf, g["f"].numpy(), k, P)

    # reduced FFN on sampled rows: selected rows get the FFN delta, others stay
    ho = g["h_out"].numpy()
    fsel = rr[np.isin(rr, idf)]
    want = O.reduced_ffn(h1, np.where(np.isin(rr, idf))[0], None, 1e-5, Wn["w_gate"], Wn["w_up"], Wn["w_down"])
    # The layer output crosses two bf16-stored stages computed independently on
    # each side (O_sel, then the FFN input and activation), so one-ulp rounding
    # flips of the first stage reach the second: twice the per-call bound.
    assert_close(ho[rr], want, LAYER_OUT_TOL, "h out (sampled rows)")
    skip = np.setdiff1d(np.arange(N), idf)
    assert np.array_equal(ho[skip], ha[skip]), "rows skipped by the FFN changed"
    assert len(fsel) > 0


@pytest.mark.parametrize("name", ["attn_8k", "layer_32k", "layer_128k", "layer_32k_kv", "layer_128k_kv",
                                  "layer_32k_mul", "layer_32k_dlow", "layer_32k_rho", "layer_32k_std",
                                  "layer_32k_seq"])
def test_layer_full_size_sampled(name):
    wl = WORKLOADS[name]
    h = make_hidden(wl)
    W = make_layer_weights(wl)
    pos = torch.arange(wl.N, dtype=torch.int32)
    sal = salient_rows(wl.N, wl.P, wl.salient_frac, wl.seed)
    g = _run_gpu_layer(wl, h, W, pos, sal)
    _check_layer_sampled(wl, h, W, pos, sal, g, wl.k)


@pytest.mark.parametrize("name", ["layer_32k", "layer_128k"])
def test_reduced_ffn_full_size_sampled(name):
    """spts_reduced_ffn alone at the full sizes, on synthetic inputs."""
    wl = WORKLOADS[name]
    rng = np.random.default_rng(1)
    h = make_hidden(wl)
    W = make_layer_weights(wl)
    idx = np.sort(rng.choice(wl.N, wl.k, replace=False)).astype(np.int32)
    hd = h.cuda()
    S.spts_reduced_ffn(hd, torch.from_numpy(idx).cuda(), None, 1e-5, W["w_gate"].cuda(), W["w_up"].cuda(),
                       W["w_down"].cuda())
    S.check_device_status()
    got = hd.cpu().numpy()
    skip = np.setdiff1d(np.arange(wl.N), idx)
    assert np.array_equal(got[skip], h.numpy()[skip]), "rows outside idx changed"
    rows = idx[np.unique(np.concatenate([[0, len(idx) - 1], rng.choice(len(idx), 64, replace=False)]))]
    Wn = {n: _f64(W[n]) for n in ("w_gate", "w_up", "w_down")}
    want = O.reduced_ffn(h.numpy()[rows].astype(np.float64), np.arange(len(rows)), None, 1e-5, Wn["w_gate"],
                         Wn["w_up"], Wn["w_down"])
    assert_close(got[rows], want, PER_CALL_TOL, "reduced ffn rows")


def _msdp_gpu(wl, h, layers_cpu):
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, 0, fuse=wl.fuse)
    lw = [{n: t.cuda() for n, t in W.items()} for W in layers_cpu]
    ks = [keep_rows(r, wl.N) for r in wl.ratios]
    hd = h.cuda()
    pd = torch.arange(wl.N, dtype=torch.int32, device="cuda")
    n, sp = S.spts_msdp_forward(hd, pd, desc, lw, 2, ks, stage_pos=True)
    S.check_device_status()
    return hd[:n].cpu(), pd[:n].cpu(), [x.cpu().numpy() for x in sp], ks


def test_msdp_full_size_properties_and_first_layer():
    wl = WORKLOADS["msdp_32k"]
    h = make_hidden(wl)
    layers = [make_layer_weights(wl, i) for i in range(wl.layers)]
    h_out, pos_out, stage_pos, ks = _msdp_gpu(wl, h, layers)
    prev = set(range(wl.N))
    tail = set(range(wl.N - wl.P, wl.N))
    for s_pos, k in zip(stage_pos, ks):
        assert len(s_pos) == k and np.all(np.diff(s_pos) > 0)
        cur = set(s_pos.tolist())
        assert cur <= prev and tail <= cur
        prev = cur
    assert np.array_equal(pos_out.numpy(), stage_pos[-1])
    assert torch.isfinite(h_out).all()
    # the first layer (stage 1) in the same configuration, against the oracle
    pos = torch.arange(wl.N, dtype=torch.int32)
    sal = torch.zeros(0, dtype=torch.int32)
    wl1 = WORKLOADS["msdp_32k"]
    g = _run_gpu_layer(wl1, h, layers[0], pos, sal, k=ks[0])
    _check_layer_sampled(wl1, h, layers[0], pos, sal, g, ks[0])


def test_msdp_small_chain_matches_oracle():
    wl = WORKLOADS["msdp_small"]
    h = make_hidden(wl)
    layers = [make_layer_weights(wl, i) for i in range(wl.layers)]
    h_out, pos_out, stage_pos, ks = _msdp_gpu(wl, h, layers)
    ow = [O.LayerWeights(**{n: _f64(t) for n, t in W.items()}) for W in layers]
    cfg = O.LayerConfig(Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, P=wl.P, k=0, fuse=wl.fuse)
    tr = []
    oh, opos, pruned = O.msdp_forward(h.numpy().astype(np.float64), np.arange(wl.N), ow,
                                      O.MsdpConfig(layer=cfg, ratios=wl.ratios, layers_per_stage=2), tr)
    # stage by stage: the GPU's candidate set must match up to near-ties of the oracle's prune score
    cand = np.arange(wl.N)
    for s, (s_pos, k) in enumerate(zip(stage_pos, ks)):
        f = tr[2 * s + 1]["f"]
        okept, tau = O.select_topk(f, k, wl.P)
        want_pos = cand[okept]
        if not np.array_equal(s_pos, want_pos):
            gk = np.searchsorted(cand, s_pos)
            band_check(gk, okept, f, tau)
            return   # the chains diverge legitimately from here on
        cand = want_pos
    assert np.array_equal(pos_out.numpy(), opos)
    # eight layers of independently rounded stages on each side
    assert_close(h_out.numpy(), oh, 4 * LAYER_OUT_TOL, "msdp final hidden states")


def test_dense_layer_path_is_bit_identical_to_the_selection_path():
    # keep 1.0 without score outputs takes the dense path (no probe, LTP or
    # selections); asking for the scores forces the general path
    wl = WORKLOADS["layer_small"]
    h = make_hidden(wl)
    Wd = {n: t.cuda() for n, t in make_layer_weights(wl).items()}
    pos = torch.arange(wl.N, dtype=torch.int32, device="cuda")
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, wl.N, fuse=wl.fuse)
    h_fast = h.cuda()
    S.spts_layer_forward(h_fast, pos, desc, Wd)
    h_sel = h.cuda()
    out = S.spts_layer_forward(h_sel, pos, desc, Wd, outputs=True)
    S.check_device_status()
    assert torch.equal(out["idx_attn"].cpu(), torch.arange(wl.N, dtype=torch.int32))
    assert torch.equal(h_fast, h_sel)


def test_schedule_small_matches_oracle():
    # a Table-B-shaped schedule at small size: 2 full layers, three stages,
    # two full layers over the survivors
    wl = WORKLOADS["msdp_small"]
    n_layers, first_skip, ends, budgets, after = 9, 2, (3, 5, 6), (450, 300, 200), 120
    h = make_hidden(wl)
    layers = [make_layer_weights(wl, i) for i in range(n_layers)]
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, 0, fuse=wl.fuse)
    hd = h.cuda()
    pd = torch.arange(wl.N, dtype=torch.int32, device="cuda")
    n, sel = S.spts_schedule_forward(hd, pd, desc, [{k: t.cuda() for k, t in W.items()} for W in layers], first_skip,
                                     ends, budgets, after, selections=True)
    S.check_device_status()
    assert n == after
    ow = [O.LayerWeights(**{k: _f64(t) for k, t in W.items()}) for W in layers]
    cfg = O.LayerConfig(Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, P=wl.P, k=0, fuse=wl.fuse)
    tr = []
    oh, opos = O.schedule_forward(h.numpy().astype(np.float64), np.arange(wl.N), ow, cfg, first_skip, ends, budgets,
                                  after, tr)
    # layer by layer: the attention sets agree until a legitimate near-tie split
    for l, t in enumerate(tr):
        if not t["skip"]:
            assert sel[l] is None
            continue
        g = sel[l].cpu().numpy()
        assert len(g) == t["k"]
        if not np.array_equal(g, t["sel_pos"]):
            return   # the chains diverge from here on (checked per call elsewhere)
    assert np.array_equal(pd[:n].cpu().numpy(), opos)
    assert_close(hd[:n].cpu().numpy(), oh, 4 * LAYER_OUT_TOL, "schedule final hidden states")
