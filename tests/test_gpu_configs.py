"""Parity at the full sizes of the workloads, in the launch configuration
bench.py times (the same inputs, the same C-ABI calls), and of the
multi-layer pipelines.

Every layer is checked teacher-forced (tests/layer_check.py): each step
against the oracle on the inputs the GPU's step received, at the per-call
tolerance (2e-2 for bf16 outputs), with exact selections over the GPU's own
scores and near-tie-only differences against the oracle's scores.  At the
full sizes the oracle computes every step whose inputs are whole arrays in
full (norm, K/V projections, probe scores, both selections, the fused
score) and the per-row steps (reduced attention, O projection, LTP score,
reduced FFN) on sampled rows, one by one; skipped rows are bit-exact.

MSDP (8 layers, 4 stages) and the Table B schedule are replayed layer by
layer on the GPU -- every layer and every stage prune checked as above --
and the pipeline call must then be bit-identical to the replay.
"""

import numpy as np
import pytest
import torch

import oracle as O
from synthetic import WORKLOADS, keep_rows, make_hidden, make_layer_weights, salient_rows
from tests.gpu_util import assert_close
from tests.layer_check import PER_CALL_TOL, check_layer_step, f64w, gpu_layer_step

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import token_skipping_sparse_b200 as S


def _run_layer(wl, h, W, k=None, sal=None):
    Wd = {n: t.cuda() for n, t in W.items()}
    sal_d = sal.cuda() if sal is not None and len(sal) else None
    hd = h.cuda()
    pd = torch.arange(wl.N, dtype=torch.int32, device="cuda")
    g, _ = gpu_layer_step(S, wl, hd, pd, Wd, wl.k if k is None else k, sal_d)
    del hd, Wd
    torch.cuda.empty_cache()
    return g


@pytest.mark.parametrize("name", ["attn_8k", "layer_32k", "layer_128k", "layer_32k_kv", "layer_128k_kv",
                                  "layer_32k_mul", "layer_32k_dlow", "layer_32k_rho", "layer_32k_std",
                                  "layer_32k_seq"])
def test_layer_full_size_sampled(name):
    wl = WORKLOADS[name]
    h = make_hidden(wl)
    W = make_layer_weights(wl)
    sal = salient_rows(wl.N, wl.P, wl.salient_frac, wl.seed)
    g = _run_layer(wl, h, W, sal=sal)
    drift = {}
    check_layer_step(wl, g, f64w(W), wl.k, sal=sal.numpy(), n_rows=40, drift=drift, label=name)
    print(f"{name}: composed drift against the oracle's own chain {drift}")


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
    Wn = {n: W[n].float().double().numpy() for n in ("w_gate", "w_up", "w_down")}
    want = O.reduced_ffn(h.numpy()[rows].astype(np.float64), np.arange(len(rows)), None, 1e-5, Wn["w_gate"],
                         Wn["w_up"], Wn["w_down"])
    assert_close(got[rows], want, PER_CALL_TOL, "reduced ffn rows")


def _prune_step(wl, hd, pd, f_dev, g, k_next, label):
    """spts_stage_prune on the GPU state, checked exactly: the kept rows are
    the top-k_next of the GPU's own (already checked) fused score under the
    tie rule with the tail forced, and the compaction copies them bit for bit."""
    h_new, p_new, kept = S.spts_stage_prune(f_dev, k_next, wl.P, hd, pd)
    S.check_device_status()
    kept_n = kept.cpu().numpy()
    want, _ = O.select_topk(g["f"].numpy(), k_next, wl.P)
    assert np.array_equal(kept_n, want), f"{label}: stage prune selection"
    assert torch.equal(h_new.cpu(), g["h_out"][torch.from_numpy(want)]), f"{label}: pruned rows not copied exactly"
    assert torch.equal(p_new.cpu(), g["pos"][torch.from_numpy(want)]), f"{label}: pruned positions"
    return h_new, p_new


def _msdp_replay(wl, h, layers, n_rows):
    """MSDP layer by layer through spts_layer_forward / spts_stage_prune, each
    step checked teacher-forced; returns the final state and stage positions."""
    ks = [keep_rows(r, wl.N) for r in wl.ratios]
    hd = h.cuda()
    pd = torch.arange(wl.N, dtype=torch.int32, device="cuda")
    stage_pos, drift, ties, li = [], {}, 0, 0
    for s, k in enumerate(ks):
        for _ in range(2):
            Wd = {n: t.cuda() for n, t in layers[li].items()}
            g, out = gpu_layer_step(S, wl, hd, pd, Wd, k)
            ties += check_layer_step(wl, g, f64w(layers[li]), k, n_rows=n_rows, seed=li, drift=drift,
                                     label=f"layer {li} (stage {s})")
            del Wd
            li += 1
        hd, pd = _prune_step(wl, hd, pd, out["f"], g, k, f"stage {s}")
        stage_pos.append(pd.cpu().numpy())
    return hd.cpu(), pd.cpu(), stage_pos, ks, drift, ties


def _msdp_pipeline(wl, h, layers, ks):
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, 0, fuse=wl.fuse)
    lw = [{n: t.cuda() for n, t in W.items()} for W in layers]
    hd = h.cuda()
    pd = torch.arange(wl.N, dtype=torch.int32, device="cuda")
    n, sp = S.spts_msdp_forward(hd, pd, desc, lw, 2, ks, stage_pos=True)
    S.check_device_status()
    out = hd[:n].cpu(), pd[:n].cpu(), [x.cpu().numpy() for x in sp]
    del lw, hd, pd
    torch.cuda.empty_cache()
    return out


def _check_msdp(name, n_rows):
    wl = WORKLOADS[name]
    h = make_hidden(wl)
    layers = [make_layer_weights(wl, i) for i in range(wl.layers)]
    h_r, p_r, sp_r, ks, drift, ties = _msdp_replay(wl, h, layers, n_rows)
    tail = set(range(wl.N - wl.P, wl.N))
    prev = set(range(wl.N))
    for s_pos, k in zip(sp_r, ks):
        assert len(s_pos) == k and np.all(np.diff(s_pos) > 0)
        cur = set(s_pos.tolist())
        assert cur <= prev and tail <= cur, "candidate sets must nest and keep the probe tail"
        prev = cur
    # the pipeline call is the replay, bit for bit
    h_p, p_p, sp_p = _msdp_pipeline(wl, h, layers, ks)
    for s, (a, b) in enumerate(zip(sp_p, sp_r)):
        assert np.array_equal(a, b), f"spts_msdp_forward stage {s} candidates differ from the replay"
    assert torch.equal(p_p, p_r) and torch.equal(h_p, h_r), "spts_msdp_forward differs from the replay"
    return wl, h, layers, h_p, p_p, drift, ties


def test_msdp_full_size_all_layers():
    """Config 5 (8 layers, 4 stages, N = 32768): all 8 layers and all 4
    stage prunes compared with the oracle, each on the GPU's own input."""
    _, _, _, _, _, drift, ties = _check_msdp("msdp_32k", n_rows=24)
    print(f"msdp_32k: {ties} near-tie selection differences; composed drift {drift}")


def test_msdp_small_chain_matches_oracle():
    """The 8-layer MSDP chain at a small size, every row of every step."""
    wl, h, layers, h_p, p_p, drift, ties = _check_msdp("msdp_small", n_rows=None)
    # the oracle's uninterrupted chain: the same candidate sets unless a
    # near-tie split them (then the drift is not comparable); reported only
    ow = [O.LayerWeights(**f64w(W)) for W in layers]
    cfg = O.LayerConfig(Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, P=wl.P, k=0, fuse=wl.fuse)
    oh, opos, _ = O.msdp_forward(h.numpy().astype(np.float64), np.arange(wl.N), ow,
                                 O.MsdpConfig(layer=cfg, ratios=wl.ratios, layers_per_stage=2))
    same = np.array_equal(p_p.numpy(), opos)
    chain = float(np.abs(h_p.numpy() - oh).max()) if same else None
    print(f"msdp_small: {ties} near-tie differences; per-layer drift {drift}; "
          f"final candidates {'equal' if same else 'split by a near-tie'}; whole-chain drift {chain}")


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
    """A Table-B-shaped schedule at small size (2 full layers, three stages,
    two full layers over the survivors), replayed layer by layer with every
    step of every layer and every prune checked on the GPU's own inputs; the
    schedule call must then be bit-identical to the replay."""
    wl = WORKLOADS["msdp_small"]
    n_layers, first_skip, ends, budgets, after = 9, 2, (3, 5, 6), (450, 300, 200), 120
    h = make_hidden(wl)
    layers = [make_layer_weights(wl, i) for i in range(n_layers)]

    # the replay
    hd = h.cuda()
    pd = torch.arange(wl.N, dtype=torch.int32, device="cuda")
    sel_r, drift, ties, stage = [], {}, 0, 0
    for l in range(n_layers):
        Nc = hd.shape[0]
        skip = l >= first_skip and stage < len(ends) and l <= ends[stage]
        k = min(budgets[stage], Nc) if skip else Nc
        Wd = {n: t.cuda() for n, t in layers[l].items()}
        g, out = gpu_layer_step(S, wl, hd, pd, Wd, k)
        ties += check_layer_step(wl, g, f64w(layers[l]), k, n_rows=None, seed=l, drift=drift, label=f"layer {l}")
        sel_r.append(g["pos"].numpy()[g["idx_attn"].numpy()] if skip else None)
        if skip and l == ends[stage]:
            k_next = min(budgets[stage] if stage + 1 < len(ends) else after, Nc)
            hd, pd = _prune_step(wl, hd, pd, out["f"], g, k_next, f"stage {stage}")
            stage += 1
    assert hd.shape[0] == after

    # the schedule call
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, 0, fuse=wl.fuse)
    hs = h.cuda()
    ps = torch.arange(wl.N, dtype=torch.int32, device="cuda")
    n, sel = S.spts_schedule_forward(hs, ps, desc, [{k: t.cuda() for k, t in W.items()} for W in layers],
                                     first_skip, ends, budgets, after, selections=True)
    S.check_device_status()
    assert n == after
    for l in range(n_layers):
        if sel_r[l] is None:
            assert sel[l] is None, f"layer {l} is a full layer"
        else:
            assert np.array_equal(sel[l].cpu().numpy(), sel_r[l]), f"layer {l}: attention set differs from replay"
    assert torch.equal(ps[:n], pd) and torch.equal(hs[:n], hd), "spts_schedule_forward differs from the replay"

    # the oracle's uninterrupted chain, reported only
    ow = [O.LayerWeights(**f64w(W)) for W in layers]
    cfg = O.LayerConfig(Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, P=wl.P, k=0, fuse=wl.fuse)
    oh, opos = O.schedule_forward(h.numpy().astype(np.float64), np.arange(wl.N), ow, cfg, first_skip, ends, budgets,
                                  after)
    same = np.array_equal(pd.cpu().numpy(), opos)
    chain = float(np.abs(hd.cpu().numpy() - oh).max()) if same else None
    print(f"schedule: {ties} near-tie differences; per-layer drift {drift}; whole-chain drift {chain}")
