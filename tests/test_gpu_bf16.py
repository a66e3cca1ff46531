"""GPU parity of the bf16 tensor-core kernels (tcgen05) against the oracle:
PAP probe scores, the LTP score, reduced GQA attention and one full layer."""

import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_bf16_close, assert_close, band_check, np64

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
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, wl.k, fuse=wl.fuse,
                        salient_rows=sal.cuda(), salient_shift=wl.salient_shift, ltp_dout=wl.ltp_dout, ltp_top_m=wl.ltp_top_m, seq_pool=0,
                        kv_active_only=wl.kv_active)
    hd = h.cuda()
    out = S.spts_layer_forward(hd, pos.cuda(), desc, Wd, outputs=True)
    S.check_device_status()
    ow = O.LayerWeights(**{n: np64(t) for n, t in W.items()})
    cfg = O.LayerConfig(Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, P=wl.P, k=wl.k, fuse=wl.fuse,
                        salient_rows=sal.numpy(), salient_shift=wl.salient_shift, kv_active=wl.kv_active,
                        ltp_top_m=wl.ltp_top_m)
    tr = {}
    O.layer_forward(np64(h), pos.numpy(), ow, cfg, tr)
    s = out["s"].cpu().numpy()
    assert_close(s, tr["s"], 1e-3 * tr["s"].max(), "probe scores")
    ia = out["idx_attn"].cpu().numpy()
    band_check(ia, tr["idx_attn"], tr["s"], tr["tau_attn"])
    # reduced attention rows: oracle computes every row, compare at the GPU's picks
    pn = pos.numpy()
    q_all = O.bf16_round(O.rope((tr["xn"] @ ow.w_q.T).reshape(wl.N, wl.Hq, wl.d), pn))
    if wl.kv_active:  # the keys are the GPU's active rows
        o_sel = O.bf16_round(O.reduced_attention(q_all[ia], pn[ia], tr["k"][ia], tr["v"][ia], pn[ia]))
    else:
        o_sel = O.bf16_round(O.reduced_attention(q_all, pn, tr["k"], tr["v"], pn))[ia]
    assert_bf16_close(np64(out["o_sel"]), o_sel, 2e-2, "o_sel")
    ha = np64(out["h_attn"])
    same = np.array_equal(ia, tr["idx_attn"])
    if same:
        assert_close(ha, tr["h_attn"], 2e-2, "h after attention")
    # a8-a10 from the GPU's own h' (each step checked on the same input): LTP
    # within the per-call bound, then the fused score and the FFN set exactly
    # (the same fp32 operations on the same scores), then the reduced FFN
    x2 = O.bf16_round(O.rmsnorm(ha, ow.norm_ffn, cfg.eps))
    c_want = (O.ltp_topm_scores(x2, ow.ltp_a, ow.ltp_b, wl.ltp_top_m) if wl.ltp_top_m
              else O.ltp_scores(x2, ow.ltp_a, ow.ltp_b))
    c = out["c"].cpu().numpy()
    assert_close(c, c_want, 1e-3 * c_want.max(), "ltp scores")
    idf = out["idx_ffn"].cpu().numpy()
    if wl.fuse == O.FUSE_SEQUENTIAL:  # the pool by s, then the k by c; f is c
        assert np.array_equal(out["f"].cpu().numpy(), c)
        want_f = O.select_sequential(s.astype(np.float32), c.astype(np.float32), min(wl.N, 2 * wl.k), wl.k, wl.P)[0]
        assert np.array_equal(idf, want_f), "FFN selection"
    else:
        f_want = O.fuse_scores(s.astype(np.float32), c.astype(np.float32), wl.fuse, 0.5, 0.5)
        assert np.array_equal(out["f"].cpu().numpy().view(np.uint32), f_want.view(np.uint32)), "fused score"
        assert np.array_equal(idf, O.select_topk(f_want, wl.k, wl.P)[0]), "FFN selection"
    h_want = O.reduced_ffn(ha, idf, ow.norm_ffn, cfg.eps, ow.w_gate, ow.w_up, ow.w_down)
    assert_close(np64(hd), h_want, 2e-2, "h out (reduced FFN on the GPU's h')")
    # the composed layer against the oracle's own chain: two bf16-stored stages
    if same and np.array_equal(idf, tr["idx_ffn"]):
        assert_close(np64(hd), tr["h_out"], 4e-2, "h out (composed)")
