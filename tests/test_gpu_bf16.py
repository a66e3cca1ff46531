"""GPU parity of the bf16 tensor-core kernels (tcgen05) against the oracle:
PAP probe scores, the LTP score, reduced GQA attention and one full layer."""

import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_close, np64
from tests.layer_check import check_layer_step, f64w, gpu_layer_step

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import token_skipping_sparse_b200 as S

rng = np.random.default_rng(11)


def _positions(n, span_factor=3):
    return np.sort(rng.choice(n * span_factor, n, replace=False)).astype(np.int32)


@pytest.mark.parametrize("Nc,k,Hq,Hkv", [(1000, 300, 8, 2), (513, 200, 4, 4), (1000, 250, 8, 4),
                                         (1000, 300, 16, 2), (5000, 1500, 32, 8), (129, 1, 8, 2), (128, 128, 8, 2)])
def test_reduced_attention_bf16(Nc, k, Hq, Hkv):
    pos = _positions(Nc)
    sel = np.sort(rng.choice(Nc, k, replace=False))
    q = torch.randn(k, Hq, 128).to(torch.bfloat16)
    kk = torch.randn(Nc, Hkv, 128).to(torch.bfloat16)
    v = torch.randn(Nc, Hkv, 128).to(torch.bfloat16)
    o = S.spts_reduced_attention(q.cuda(), torch.from_numpy(pos[sel]).cuda(), kk.cuda(), v.cuda(),
                                 torch.from_numpy(pos).cuda())
    want = O.reduced_attention(np64(q), pos[sel], np64(kk), np64(v), pos)
    got = np64(o)
    assert_close(got, want, 2e-2, "reduced attention bf16")
    assert np.mean(np.abs(got - want)) < 2e-3


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (8, 4), (32, 8)])
def test_reduced_attention_bf16_lopsided_tile_pairs(Hq, Hkv):
    """A CTA's two Q tiles with very different key ranges: the first tile of
    each pair sees one or two key tiles, the second dozens, so for most key
    steps only the second tile runs and the K and V stages are recycled by
    its MMAs alone; the last pair is a single partial tile."""
    Nc, tq = 4096, 128 // (Hq // Hkv)
    pos = np.arange(Nc, dtype=np.int32) * 2 + 1
    early = np.arange(tq)                              # keys 0 .. tq-1
    late = np.arange(Nc - 40 * tq, Nc - 39 * tq)       # most of the keys
    tail = np.arange(Nc - 3 * tq // 2, Nc)             # last pair: one full tile and half of the next
    sel = np.concatenate([early, late, np.arange(Nc - 38 * tq, Nc - 36 * tq), tail]).astype(np.int64)
    assert np.all(np.diff(sel) > 0)
    k = len(sel)
    q = torch.randn(k, Hq, 128).to(torch.bfloat16)
    kk = torch.randn(Nc, Hkv, 128).to(torch.bfloat16)
    v = torch.randn(Nc, Hkv, 128).to(torch.bfloat16)
    o = S.spts_reduced_attention(q.cuda(), torch.from_numpy(pos[sel]).cuda(), kk.cuda(), v.cuda(),
                                 torch.from_numpy(pos).cuda())
    want = O.reduced_attention(np64(q), pos[sel], np64(kk), np64(v), pos)
    got = np64(o)
    assert_close(got, want, 2e-2, "reduced attention bf16, lopsided pairs")
    assert np.mean(np.abs(got - want)) < 2e-3


@pytest.mark.parametrize("Nc,P,Hq,Hkv", [(1000, 16, 8, 2), (3000, 64, 32, 8), (2000, 128, 32, 8), (300, 64, 8, 8),
                                         (700, 20, 8, 4), (2500, 80, 32, 8), (130, 100, 32, 8), (1000, 1, 32, 8)])
def test_probe_scores_bf16(Nc, P, Hq, Hkv):
    pos = _positions(Nc)
    q = torch.randn(P, Hq, 128).to(torch.bfloat16)
    kk = torch.randn(Nc, Hkv, 128).to(torch.bfloat16)
    s, g = S.spts_probe_scores(q.cuda(), torch.from_numpy(pos[-P:]).cuda(), kk.cuda(), torch.from_numpy(pos).cuda(),
                               group_scores=True)
    ws_, wg = O.probe_scores(np64(q), pos[-P:], np64(kk), pos)
    tol = 1e-3 * ws_.max() + 1e-5
    assert_close(s.cpu().numpy(), ws_, tol, "probe scores")
    assert_close(g.cpu().numpy(), wg, tol, "group scores")
    assert abs(float(s.double().sum()) - P * Hq) < 1e-3 * P * Hq


@pytest.mark.parametrize("Nc,D,r,Dout", [(1000, 1024, 64, 1024), (300, 4096, 256, 4096), (129, 512, 128, 768),
                                         (700, 4096, 192, 512)])
def test_ltp_scores_bf16(Nc, D, r, Dout):
    x = torch.randn(Nc, D).to(torch.bfloat16)
    A = (0.02 * torch.randn(r, D)).to(torch.bfloat16)
    B = (0.02 * torch.randn(Dout, r)).to(torch.bfloat16)
    c = S.spts_ltp_scores(x.cuda(), A.cuda(), B.cuda())
    want = O.ltp_scores(np64(x), np64(A), np64(B))
    assert_close(c.cpu().numpy(), want, 1e-3 * want.max(), "ltp scores")


@pytest.mark.parametrize("Nc,D,r,Dout,m", [(1000, 1024, 192, 512, 103), (300, 4096, 256, 256, 1),
                                           (129, 512, 64, 512, 512), (700, 4096, 192, 512, 52)])
def test_ltp_topm_scores_bf16(Nc, D, r, Dout, m):
    x = torch.randn(Nc, D).to(torch.bfloat16)
    A = (0.02 * torch.randn(r, D)).to(torch.bfloat16)
    B = (0.02 * torch.randn(Dout, r)).to(torch.bfloat16)
    c = S.spts_ltp_topm_scores(x.cuda(), A.cuda(), B.cuda(), m)
    want = O.ltp_topm_scores(np64(x), np64(A), np64(B), m)
    assert_close(c.cpu().numpy(), want, 1e-3 * want.max(), "top-m ltp scores")


def _layer_case(name):
    from synthetic import WORKLOADS, make_hidden, make_layer_weights, salient_rows
    wl = WORKLOADS[name]
    h = make_hidden(wl)
    W = make_layer_weights(wl)
    sal = salient_rows(wl.N, wl.P, wl.salient_frac, wl.seed)
    pos = torch.arange(wl.N, dtype=torch.int32)
    return wl, h, W, sal, pos


# the base layer and its variants: active-row keys only, Multiply fusion, one
# probe token, the channel-reduced LTP proxy
@pytest.mark.parametrize("name", ["layer_small", "layer_small_kv", "layer_small_mul", "layer_small_p1",
                                  "layer_small_dlow", "layer_small_rho", "layer_small_std", "layer_small_seq"])
def test_layer_small_matches_oracle(name):
    wl, h, W, sal, pos = _layer_case(name)
    _check_layer(wl, h, W, sal, pos, {n: t.cuda() for n, t in W.items()})


# Non-unit norm weights, distinct for the two norms (the FFN input is a full
# RMSNorm pass over h') or one shared vector (only the attention rows are
# renormalised, in place).
@pytest.mark.parametrize("shared", [False, True])
def test_layer_norm_weights(shared):
    wl, h, W, sal, pos = _layer_case("layer_small")
    g = torch.Generator().manual_seed(11)
    W["norm_attn"] = (1 + 0.2 * torch.randn(wl.D, generator=g)).to(torch.bfloat16)
    W["norm_ffn"] = W["norm_attn"] if shared else (1 + 0.2 * torch.randn(wl.D, generator=g)).to(torch.bfloat16)
    Wd = {n: t.cuda() for n, t in W.items() if n != "norm_ffn"}
    Wd["norm_ffn"] = Wd["norm_attn"] if shared else W["norm_ffn"].cuda()
    _check_layer(wl, h, W, sal, pos, Wd)


def _check_layer(wl, h, W, sal, pos, Wd):
    """Every step of the layer on its own inputs (tests/layer_check.py), all
    rows; then the oracle's uninterrupted chain, reported as drift."""
    hd = h.cuda()
    g, _ = gpu_layer_step(S, wl, hd, pos.cuda(), Wd, wl.k, sal.cuda() if len(sal) else None)
    drift = {}
    Wn = f64w(W)
    ties = check_layer_step(wl, g, Wn, wl.k, sal=sal.numpy(), n_rows=None, drift=drift, label=wl.name)
    ow = O.LayerWeights(**Wn)
    cfg = O.LayerConfig(Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, P=wl.P, k=wl.k, fuse=wl.fuse,
                        salient_rows=sal.numpy(), salient_shift=wl.salient_shift, kv_active=wl.kv_active,
                        ltp_top_m=wl.ltp_top_m)
    tr = {}
    O.layer_forward(np64(h), pos.numpy(), ow, cfg, tr)
    same = (np.array_equal(g["idx_attn"].numpy(), tr["idx_attn"])
            and np.array_equal(g["idx_ffn"].numpy(), tr["idx_ffn"]))
    chain = float(np.abs(g["h_out"].numpy() - tr["h_out"]).max()) if same else None
    print(f"{wl.name}: {ties} near-tie differences; drift {drift}; whole-layer drift {chain}")
