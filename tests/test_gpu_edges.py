"""Edge cases through the C ABI: empty and ragged inputs, single partial
tiles, and the degenerate cases of the method (keep ratio 1.0, k = P so only
the probe rows are kept, a single probe as in Table C's default)."""

import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_bf16_close, assert_close, np64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import token_skipping_sparse_b200 as S

rng = np.random.default_rng(3)


def test_select_all_equal_scores_takes_lowest_indices():
    s = torch.full((5000,), 0.125, device="cuda")
    idx = S.spts_select_topk(s, 700, 64)
    want = np.concatenate([np.arange(636), np.arange(5000 - 64, 5000)])
    assert np.array_equal(idx.cpu().numpy(), want)



@pytest.mark.parametrize("Nc,k,tail", [(100000, 20000, 128), (70000, 70000, 64), (70000, 64, 64), (50000, 1, 0),
                                       (30000, 9000, 64)])
def test_select_large_sets_on_the_grid_path(Nc, k, tail):
    # above 20K free candidates the selection runs on the grid; all-equal
    # scores put every key in one radix bin, few distinct values make long
    # runs of ties at the threshold
    for s in (np.full(Nc, 0.125, np.float32), rng.integers(0, 5, Nc).astype(np.float32) * 0.5):
        want, _ = O.select_topk(s, k, tail)
        idx = S.spts_select_topk(torch.from_numpy(s).cuda(), k, tail)
        assert np.array_equal(idx.cpu().numpy(), want)


def test_select_zero_scores_and_negative_zero():
    s = torch.zeros(300, device="cuda")
    s[::3] = -0.0
    idx = S.spts_select_topk(s, 100, 0)
    assert np.array_equal(idx.cpu().numpy(), np.arange(100))


def test_stage_prune_keep_all_and_keep_tail_only():
    Nc, D = 1000, 64
    scores = torch.rand(Nc, device="cuda")
    h = torch.randn(Nc, D, device="cuda")
    pos = torch.arange(Nc, dtype=torch.int32, device="cuda") * 3
    ho, po, kept = S.spts_stage_prune(scores, Nc, 16, h, pos)
    assert torch.equal(ho, h) and torch.equal(po, pos)
    ho, po, kept = S.spts_stage_prune(scores, 16, 16, h, pos)
    assert torch.equal(ho, h[-16:]) and torch.equal(po, pos[-16:])


def test_attention_single_partial_tile_and_first_position():
    Nc, k, Hq, Hkv = 100, 30, 8, 2
    pos = np.sort(rng.choice(1000, Nc, replace=False)).astype(np.int32)
    sel = np.sort(np.concatenate([[0], rng.choice(np.arange(1, Nc), k - 1, replace=False)]))
    q = torch.randn(k, Hq, 128).to(torch.bfloat16)
    kk = torch.randn(Nc, Hkv, 128).to(torch.bfloat16)
    v = torch.randn(Nc, Hkv, 128).to(torch.bfloat16)
    o = S.spts_reduced_attention(q.cuda(), torch.from_numpy(pos[sel]).cuda(), kk.cuda(), v.cuda(),
                                 torch.from_numpy(pos).cuda())
    want = O.reduced_attention(np64(q), pos[sel], np64(kk), np64(v), pos)
    assert_close(np64(o), want, 2e-2, "attention, one partial key tile")
    # the query at the first position sees only key 0: its output is v_0 (per KV group)
    v0 = np64(v)[0].repeat(Hq // Hkv, axis=0)
    assert_bf16_close(np64(o)[0], v0, 1e-6, "first-position query")


@pytest.mark.parametrize("n_blind", [3, 70])
def test_attention_queries_that_see_no_key_are_zero(n_blind):
    # keys start at position 1000; the first n_blind queries sit before them
    # (3: inside the first Q tile, 70: whole tiles of them), the rest among
    # the keys: the blind rows come out 0, the others match the oracle
    Nc, Hq, Hkv = 400, 8, 2
    pos = (1000 + np.sort(rng.choice(4000, Nc, replace=False))).astype(np.int32)
    blind = np.sort(rng.choice(1000, n_blind, replace=False)).astype(np.int32)
    seen = np.sort(rng.choice(pos, 90, replace=False)).astype(np.int32)
    q_pos = np.concatenate([blind, seen])
    m = len(q_pos)
    q = torch.randn(m, Hq, 128).to(torch.bfloat16)
    kk = torch.randn(Nc, Hkv, 128).to(torch.bfloat16)
    v = torch.randn(Nc, Hkv, 128).to(torch.bfloat16)
    o = np64(S.spts_reduced_attention(q.cuda(), torch.from_numpy(q_pos).cuda(), kk.cuda(), v.cuda(),
                                      torch.from_numpy(pos).cuda()))
    assert np.array_equal(o[:n_blind], np.zeros_like(o[:n_blind]))
    want = O.reduced_attention(np64(q)[n_blind:], seen, np64(kk), np64(v), pos)
    assert_close(o[n_blind:], want, 2e-2, "attention after the blind rows")


def test_probe_single_probe_and_all_keys_are_probes():
    for Nc, P in [(777, 1), (64, 64)]:
        pos = np.sort(rng.choice(5000, Nc, replace=False)).astype(np.int32)
        q = torch.randn(P, 32, 128).to(torch.bfloat16)
        kk = torch.randn(Nc, 8, 128).to(torch.bfloat16)
        s = S.spts_probe_scores(q.cuda(), torch.from_numpy(pos[-P:]).cuda(), kk.cuda(), torch.from_numpy(pos).cuda())
        want, _ = O.probe_scores(np64(q), pos[-P:], np64(kk), pos)
        assert_close(s.cpu().numpy(), want, 1e-3 * want.max() + 1e-6, f"probe P={P}")


def test_empty_inputs_launch_nothing():
    n0 = S.launch_count()
    x = torch.zeros(0, 512, device="cuda")
    S.spts_rmsnorm_rows(x)
    A = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda")
    S.spts_linear(A, W)
    h = torch.randn(10, 256, device="cuda")
    hb = h.clone()
    S.spts_reduced_ffn(h, torch.zeros(0, dtype=torch.int32, device="cuda"), None, 1e-5,
                       torch.zeros(128, 256, dtype=torch.bfloat16, device="cuda"),
                       torch.zeros(128, 256, dtype=torch.bfloat16, device="cuda"),
                       torch.zeros(256, 128, dtype=torch.bfloat16, device="cuda"))
    assert torch.equal(h, hb)
    S.spts_ltp_scores(torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda"),
                      torch.zeros(64, 256, dtype=torch.bfloat16, device="cuda"),
                      torch.zeros(256, 64, dtype=torch.bfloat16, device="cuda"))
    assert S.launch_count() == n0


def _small_layer(N, k, P):
    from synthetic import WORKLOADS, make_hidden, make_layer_weights, with_overrides
    wl = with_overrides(WORKLOADS["layer_small"], N=N, P=P, keep="1", salient_frac="0")
    h = make_hidden(wl)
    W = make_layer_weights(wl)
    pos = torch.arange(N, dtype=torch.int32) * 2 + 7
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, P, k, fuse=wl.fuse)
    hd = h.cuda()
    out = S.spts_layer_forward(hd, pos.cuda(), desc, {n: t.cuda() for n, t in W.items()}, outputs=True)
    ow = O.LayerWeights(**{n: np64(t) for n, t in W.items()})
    cfg = O.LayerConfig(Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, P=P, k=k, fuse=wl.fuse)
    tr = {}
    O.layer_forward(np64(h), pos.numpy(), ow, cfg, tr)
    return hd, out, tr


def test_layer_keep_ratio_one_is_the_dense_layer():
    N = 300
    hd, out, tr = _small_layer(N, N, 16)
    assert np.array_equal(out["idx_attn"].cpu().numpy(), np.arange(N))
    assert np.array_equal(out["idx_ffn"].cpu().numpy(), np.arange(N))
    assert_close(np64(hd), tr["h_out"], 2e-2, "dense layer")


def test_layer_keeps_only_the_probe_rows_when_k_equals_p():
    N, P = 400, 16
    hd, out, tr = _small_layer(N, P, P)
    assert np.array_equal(out["idx_attn"].cpu().numpy(), np.arange(N - P, N))
    assert np.array_equal(out["idx_ffn"].cpu().numpy(), np.arange(N - P, N))
    assert_close(np64(hd), tr["h_out"], 2e-2, "k = P layer")
