"""GPU parity of the single kernels against the CPU oracle (or, for the bare
GEMM epilogues, the plain fp64 definition), through the C ABI."""

import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_bf16_close, assert_close, bf16, np64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import token_skipping_sparse_b200 as S

rng = np.random.default_rng(7)


def _w(o, i, scale=0.02):
    return (scale * torch.randn(o, i)).to(torch.bfloat16)


# ---------------------------------------------------------------- GEMM epilogues
@pytest.mark.parametrize("M,K,N", [(300, 256, 512), (1000, 1024, 1024), (128, 64, 256), (1, 128, 256)])
def test_linear_store(M, K, N):
    A = torch.randn(M, K).to(torch.bfloat16)
    W = _w(N, K)
    out = S.spts_linear(A.cuda(), W.cuda())
    want = O.bf16_round(np64(A) @ np64(W).T)
    assert_bf16_close(np64(out), want, 1e-4, "linear store")



def test_linear_store_more_tiles_than_sm_pairs():
    # 40 x 4 tiles of 256 x 256 over at most 74 resident CTA pairs: every pair
    # runs several tiles through both TMEM accumulators; M is ragged.
    M, K, N = 10200, 256, 1024
    A = torch.randn(M, K).to(torch.bfloat16)
    W = _w(N, K)
    out = S.spts_linear(A.cuda(), W.cuda())
    want = O.bf16_round(np64(A) @ np64(W).T)
    assert_bf16_close(np64(out), want, 1e-4, "linear store, many tiles")


@pytest.mark.parametrize("epi", ["store", "rope", "swiglu", "scatter"])
def test_linear_whole_round_then_half_tiles(epi):
    # 10 x 8 = 80 two-SM tiles over 74 resident CTA pairs on a B200: one round
    # of whole 256 x 256 tiles, then the 6 tiles left run as 12 halves of 128
    # columns (N = 128 MMAs); M is ragged
    M, K, N = 2500, 128, 2048
    A = torch.randn(M, K).to(torch.bfloat16)
    Ad = A.cuda()
    if epi == "store":
        W = _w(N, K)
        got = np64(S.spts_linear(Ad, W.cuda()))
        want = O.bf16_round(np64(A) @ np64(W).T)
    elif epi == "rope":
        W = _w(N, K)
        pos = torch.from_numpy(np.sort(rng.choice(200000, M, replace=False)).astype(np.int32))
        got = np64(S.spts_linear(Ad, W.cuda(), S.EPI_ROPE, row_pos=pos.cuda(), theta=500000.0))
        want = O.bf16_round(O.rope((np64(A) @ np64(W).T).reshape(M, N // 128, 128), pos.numpy(),
                                   500000.0)).reshape(M, -1)
    elif epi == "swiglu":
        F = N // 2                                     # 8 tiles of 128 gate + 128 up columns
        Wg, Wu = _w(F, K, 0.1), _w(F, K, 0.1)
        got = np64(S.spts_linear(Ad, Wg.cuda(), S.EPI_SWIGLU, W2=Wu.cuda()))
        g, u = np64(A) @ np64(Wg).T, np64(A) @ np64(Wu).T
        want = O.bf16_round(g / (1 + np.exp(-g)) * u)
    else:
        W = _w(N, K)
        Nc = 3000
        h = torch.randn(Nc, N)
        rows = torch.from_numpy(rng.choice(Nc, M, replace=False).astype(np.int32))
        hd = h.cuda()
        S.spts_linear(Ad, W.cuda(), S.EPI_SCATTER_ADD, out=hd, rows=rows.cuda())
        want = np64(h)
        want[rows.numpy()] += np64(A) @ np64(W).T
        got = np64(hd)
        skip = np.setdiff1d(np.arange(Nc), rows.numpy())
        assert np.array_equal(got[skip], np64(h)[skip])
        assert_close(got, want, 1e-4, "scatter add, halves")
        return
    assert_bf16_close(got, want, 1e-4, f"linear {epi}, halves")


@pytest.mark.parametrize("lo,hi", [(0, 200000), (2 ** 24 - 170, 2 ** 24 + 163), (2 ** 30, 2 ** 31 - 1)])
def test_linear_rope(lo, hi):
    # positions below 2^24 take the fp32 two-product angle reduction, from
    # 2^24 on the fp64 one; the middle case straddles the switch
    M, K, H = 333, 512, 4
    A = torch.randn(M, K).to(torch.bfloat16)
    W = _w(H * 128, K)
    pos = torch.from_numpy(np.sort(rng.choice(np.arange(lo, hi), M, replace=False)).astype(np.int32))
    out = S.spts_linear(A.cuda(), W.cuda(), S.EPI_ROPE, row_pos=pos.cuda(), theta=500000.0)
    want = O.bf16_round(O.rope((np64(A) @ np64(W).T).reshape(M, H, 128), pos.numpy(), 500000.0)).reshape(M, -1)
    assert_bf16_close(np64(out), want, 1e-4, "linear rope")


def test_linear_swiglu():
    M, K, F = 257, 256, 384
    A = torch.randn(M, K).to(torch.bfloat16)
    Wg, Wu = _w(F, K, 0.1), _w(F, K, 0.1)
    out = S.spts_linear(A.cuda(), Wg.cuda(), S.EPI_SWIGLU, W2=Wu.cuda())
    g, u = np64(A) @ np64(Wg).T, np64(A) @ np64(Wu).T
    want = O.bf16_round(g / (1 + np.exp(-g)) * u)
    assert_bf16_close(np64(out), want, 1e-4, "linear swiglu")


@pytest.mark.parametrize("M,sort_rows", [(200, True), (200, False), (100, False), (1, True)])
def test_linear_scatter_add(M, sort_rows):
    # two-SM tiles (M > 128) and one-SM tiles, ragged last tiles, rows in any
    # order (they must only be unique)
    K, N, Nc = 384, 512, 700
    A = torch.randn(M, K).to(torch.bfloat16)
    W = _w(N, K)
    h = torch.randn(Nc, N)
    rows = rng.choice(Nc, M, replace=False)
    rows = torch.from_numpy((np.sort(rows) if sort_rows else rows).astype(np.int32))
    hd = h.cuda()
    S.spts_linear(A.cuda(), W.cuda(), S.EPI_SCATTER_ADD, out=hd, rows=rows.cuda())
    want = np64(h)
    want[rows.numpy()] += np64(A) @ np64(W).T
    got = np64(hd)
    skip = np.setdiff1d(np.arange(Nc), rows.numpy())
    assert np.array_equal(got[skip], np64(h)[skip])
    assert_close(got, want, 1e-4, "scatter add")


# ---------------------------------------------------------------- row ops
def test_rmsnorm_rows_with_gather():
    x = torch.randn(500, 1024) * 3
    w = torch.randn(1024).to(torch.bfloat16)
    rows = torch.from_numpy(rng.choice(500, 77, replace=False).astype(np.int32))
    y = S.spts_rmsnorm_rows(x.cuda(), w.cuda(), 1e-5, rows.cuda())
    want = O.bf16_round(O.rmsnorm(np64(x)[rows.numpy()], np64(w), 1e-5))
    assert_bf16_close(np64(y), want, 1e-5, "rmsnorm")


@pytest.mark.parametrize("lo,hi", [(0, 131072), (2 ** 24 - 45, 2 ** 24 + 45)])
def test_rope_inplace(lo, hi):
    x = torch.randn(90, 8, 128).to(torch.bfloat16)
    pos = torch.from_numpy(np.sort(rng.choice(np.arange(lo, hi), 90, replace=False)).astype(np.int32))
    y = S.spts_rope(x.cuda(), pos.cuda(), 500000.0)
    want = O.bf16_round(O.rope(np64(x), pos.numpy(), 500000.0))
    assert_bf16_close(np64(y), want, 1e-5, "rope")


def test_gather_rows_and_bad_index():
    src = torch.randn(100, 64).cuda()
    rows = torch.tensor([5, 99, 0, 42], dtype=torch.int32).cuda()
    assert torch.equal(S.spts_gather_rows(src, rows), src[rows.long()])
    ws = torch.zeros(256, dtype=torch.uint8).cuda()
    S.spts_gather_rows(src, torch.tensor([3, 100], dtype=torch.int32).cuda(), ws=ws)
    with pytest.raises(S.SptsError) as e:
        S.check_device_status(ws)
    assert e.value.status == S.ERR_INVALID
    S.check_device_status(ws)  # cleared


# ---------------------------------------------------------------- selection
@pytest.mark.parametrize("Nc,k,tail", [(1000, 300, 16), (1000, 1000, 16), (1000, 16, 16), (20544, 6163, 64),
                                       (20545, 6163, 64), (32768, 9830, 64), (49280, 9830, 64),
                                       (60000, 12000, 128), (131072, 26214, 128), (7, 3, 0), (1, 1, 1)])
@pytest.mark.parametrize("mode", [0, 1, 2, 3])
def test_select_topk_bit_exact(Nc, k, tail, mode):
    s = rng.random(Nc).astype(np.float32)
    c = (rng.random(Nc) * 30).astype(np.float32)
    s[rng.integers(0, Nc, Nc // 10)] = 0.25        # ties
    if Nc > 4:
        s[:3] = [0.0, -0.0, 0.0]
    f = O.fuse_scores(s, c, mode, 0.5, 0.5)
    want, tau = O.select_topk(f, k, tail)
    idx, fused, kth = S.spts_select_topk(torch.from_numpy(s).cuda(), k, tail, s_b=torch.from_numpy(c).cuda(),
                                         mode=mode, fused=True, kth=True)
    assert np.array_equal(fused.cpu().numpy().view(np.uint32), f.view(np.uint32))
    assert np.array_equal(idx.cpu().numpy(), want)
    if k > tail:
        assert kth.item() == tau
    else:
        assert np.isnan(kth.item())



@pytest.mark.parametrize("Nc,k_pool,k,tail", [(1000, 600, 300, 16), (60000, 24000, 12000, 128),
                                              (131072, 52428, 26214, 128), (500, 500, 100, 0), (300, 40, 40, 8)])
def test_select_sequential_matches_oracle(Nc, k_pool, k, tail):
    s = rng.random(Nc).astype(np.float32)
    c = (rng.random(Nc) * 30).astype(np.float32)
    c[rng.integers(0, Nc, Nc // 10)] = 7.0         # ties in the second criterion
    idx = S.spts_select_sequential(torch.from_numpy(s).cuda(), torch.from_numpy(c).cuda(), k_pool, k, tail)
    want, _ = O.select_sequential(s, c, k_pool, k, tail)
    assert np.array_equal(idx.cpu().numpy(), want)

def test_select_rejects_bad_sizes():
    s = torch.rand(10).cuda()
    with pytest.raises(S.SptsError) as e:
        S.spts_select_topk(s, 3, 5)
    assert e.value.status == S.ERR_SHAPE


def test_stage_prune_matches_oracle():
    Nc, D, keep, tail = 3000, 256, 1234, 16
    scores = rng.random(Nc).astype(np.float32)
    h = torch.randn(Nc, D)
    pos = torch.from_numpy(np.sort(rng.choice(10 ** 6, Nc, replace=False)).astype(np.int32))
    ho, po, kept = S.spts_stage_prune(torch.from_numpy(scores).cuda(), keep, tail, h.cuda(), pos.cuda())
    wh, wp, wk = O.stage_prune(scores, keep, tail, np64(h), pos.numpy())
    assert np.array_equal(kept.cpu().numpy(), wk)
    assert np.array_equal(po.cpu().numpy(), wp)
    assert np.array_equal(np64(ho), wh)


# ---------------------------------------------------------------- fp32 PAP + attention (tiny MHA case)
def test_tiny_f32_probe_select_attention():
    from synthetic import WORKLOADS, make_qkv_f32
    wl = WORKLOADS["tiny_f32"]
    q, k, v, pos, _ = make_qkv_f32(wl)
    P = wl.P
    s, group = S.spts_probe_scores(q[-P:].cuda(), pos[-P:].cuda(), k.cuda(), pos.cuda(), group_scores=True)
    ws_, wg = O.probe_scores(np64(q[-P:]), pos[-P:].numpy(), np64(k), pos.numpy())
    assert_close(s.cpu().numpy(), ws_, 1e-4, "probe scores")
    assert_close(group.cpu().numpy(), wg, 1e-4, "group scores")
    assert abs(float(s.double().sum()) - P * wl.Hq) < 1e-3
    idx = S.spts_select_topk(s, wl.k, P)
    oidx, tau = O.select_topk(ws_.astype(np.float32), wl.k, P)
    from tests.gpu_util import band_check
    band_check(idx.cpu().numpy(), oidx, ws_, tau)
    il = idx.long()
    o = S.spts_reduced_attention(q.cuda()[il].contiguous(), pos.cuda()[il].contiguous(), k.cuda(), v.cuda(),
                                 pos.cuda())
    # the oracle attends every row; the GPU rows are compared at the indices it selected
    want_all = O.reduced_attention(np64(q), pos.numpy(), np64(k), np64(v), pos.numpy())
    assert_close(np64(o), want_all[idx.cpu().numpy()], 1e-4, "attention f32")


# ---------------------------------------------------------------- reduced FFN
def test_reduced_ffn_small():
    Nc, D, F, k = 600, 512, 640, 200
    h = torch.randn(Nc, D)
    wg, wu, wd = _w(F, D, 0.05), _w(F, D, 0.05), _w(D, F, 0.05)
    nw = (1 + 0.1 * torch.randn(D)).to(torch.bfloat16)
    idx = torch.from_numpy(np.sort(rng.choice(Nc, k, replace=False)).astype(np.int32))
    hd = h.cuda()
    S.spts_reduced_ffn(hd, idx.cuda(), nw.cuda(), 1e-5, wg.cuda(), wu.cuda(), wd.cuda())
    want = O.reduced_ffn(np64(h), idx.numpy(), np64(nw), 1e-5, np64(wg), np64(wu), np64(wd))
    got = np64(hd)
    skip = np.setdiff1d(np.arange(Nc), idx.numpy())
    assert np.array_equal(got[skip], np64(h)[skip])
    assert_close(got, want, 2e-2, "reduced ffn")


# ---------------------------------------------------------------- synthetic salience
@pytest.mark.parametrize("Nc,Hq,Hkv,d,P,n_rows", [(3000, 32, 8, 128, 64, 655), (500, 4, 4, 64, 16, 10),
                                                  (700, 32, 8, 128, 1, 129), (300, 8, 2, 128, 128, 1)])
def test_inject_salience_matches_oracle(Nc, Hq, Hkv, d, P, n_rows):
    # several row chunks per KV head with a ragged last chunk, fewer query
    # vectors than slices (P = 1), and a single row
    g = torch.Generator().manual_seed(Nc + P)
    k = torch.randn(Nc, Hkv, d, generator=g).to(torch.bfloat16)
    q = torch.randn(P, Hq, d, generator=g).to(torch.bfloat16)
    rows = np.sort(np.random.default_rng(Nc).choice(Nc, n_rows, replace=False)).astype(np.int32)
    kd = k.cuda()
    S.spts_inject_salience(kd, q.cuda(), torch.from_numpy(rows).cuda(), 3.0)
    want = O.inject_salience(np64(k), np64(q), rows, 3.0, Hkv)
    got = np64(kd)
    assert np.array_equal(np.delete(got, rows, axis=0), np.delete(np64(k), rows, axis=0))
    # the kernel forms k + shift*u in fp32 (|k| + shift <~ 8): its rounding
    # error, below 2^-20, decides the result only where the sum cancels to
    # near zero; elsewhere within one bf16 ulp of the fp64 oracle
    assert_bf16_close(got, want, 2.0 ** -20, "salient keys")


# ---------------------------------------------------------------- bounded waits
def test_bounded_wait_timeout_reports_and_context_survives():
    A = torch.randn(512, 4096).to(torch.bfloat16).cuda()
    W = _w(1024, 4096).cuda()
    ws = torch.zeros(256, dtype=torch.uint8).cuda()
    old = S.get_wait_limit_ns()
    try:
        S.set_wait_limit_ns(0)
        S.spts_linear(A, W, ws=ws)
        with pytest.raises(S.SptsError) as e:
            S.check_device_status(ws)
        assert e.value.status == S.ERR_TIMEOUT
    finally:
        S.set_wait_limit_ns(old)
    out = S.spts_linear(A, W, ws=ws)
    S.check_device_status(ws)
    want = O.bf16_round(np64(A) @ np64(W).T)
    assert_bf16_close(np64(out), want, 1e-4, "linear after timeout")
