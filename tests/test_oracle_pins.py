"""Pins of the CPU oracle against things other than itself.

Each test checks an oracle function against a library routine it does not
use, a closed form, an invariant, brute force on tiny inputs, or values
printed in "Probe and Skip: Self-Predictive Token Skipping for Efficient
Long-Context LLM Inference" (Tables A and 5).  The cases are chosen so that a
dropped term, a wrong sign or index, or a transposed operand fails one of them.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O

rng = np.random.default_rng(12345)


def _sdpa(q, k, v, mask):
    """torch SDPA in fp64: q [H, m, d], k/v [H, n, d], mask [m, n] bool."""
    return F.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k),
                                          torch.from_numpy(v), attn_mask=torch.from_numpy(mask)).numpy()


# ---------------------------------------------------------------- bf16
def test_bf16_round_matches_torch_on_fp32_values():
    x = rng.standard_normal(200000).astype(np.float32) * np.float32(3.0)
    x[:5] = [0.0, -0.0, 1e-39, -3e-40, 65504.0]
    # exact ties: a bf16 value plus half of its ulp, representable in fp32
    base = torch.randn(1000).to(torch.bfloat16).float().numpy()
    ties = (base + np.sign(base) * np.float32(2.0) ** (np.floor(np.log2(np.abs(base))) - 8)).astype(np.float32)
    allx = np.concatenate([x, ties])
    want = torch.from_numpy(allx).to(torch.bfloat16).double().numpy()
    got = O.bf16_round(allx.astype(np.float64))
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_matches_torch():
    x = rng.standard_normal((37, 96)) * 2.5
    w = rng.standard_normal(96)
    want = F.rms_norm(torch.from_numpy(x), (96,), torch.from_numpy(w), eps=1e-5).numpy()
    np.testing.assert_allclose(O.rmsnorm(x, w, 1e-5), want, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- RoPE
def test_rope_rotate_half_closed_form():
    # d = 4: pairs (0, 2) with frequency 1 and (1, 3) with frequency theta**-0.5.
    theta = 10000.0
    x = np.zeros((1, 1, 4)); x[0, 0, 0] = 1.0
    p = 3
    y = O.rope(x, np.array([p]), theta)[0, 0]
    np.testing.assert_allclose(y, [math.cos(p), 0.0, math.sin(p), 0.0], atol=1e-15)
    x = np.zeros((1, 1, 4)); x[0, 0, 3] = 1.0
    y = O.rope(x, np.array([p]), theta)[0, 0]
    a = p * theta ** -0.5
    np.testing.assert_allclose(y, [0.0, -math.sin(a), 0.0, math.cos(a)], atol=1e-15)


def test_rope_matches_complex_rotation_and_is_relative():
    d, theta = 128, 500000.0
    x = rng.standard_normal((5, 3, d))
    pos = np.array([0, 1, 77, 4096, 131071])
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    freq = theta ** (-np.arange(0, d, 2) / d)
    zr = z * np.exp(1j * pos[:, None, None] * freq[None, None, :])
    want = np.concatenate([zr.real, zr.imag], axis=-1)
    np.testing.assert_allclose(O.rope(x, pos, theta), want, rtol=1e-9, atol=1e-9)
    q, k = rng.standard_normal((1, 1, d)), rng.standard_normal((1, 1, d))
    a = np.sum(O.rope(q, [100], theta) * O.rope(k, [40], theta))
    b = np.sum(O.rope(q, [1100], theta) * O.rope(k, [1040], theta))
    assert abs(a - b) < 1e-9


# ---------------------------------------------------------------- PAP
def _probe_case(Nc=70, P=5, Hq=8, Hkv=2, d=16, gaps=True):
    pos = np.cumsum(rng.integers(1, 4, Nc)) if gaps else np.arange(Nc)
    q = rng.standard_normal((P, Hq, d))
    k = rng.standard_normal((Nc, Hkv, d))
    return q, k, pos


def test_probe_scores_match_sdpa_with_identity_values():
    """Column sums of the causal softmax rows, via SDPA with V = I."""
    Nc, P, Hq, Hkv, d = 70, 5, 8, 2, 16
    q, k, pos = _probe_case(Nc, P, Hq, Hkv, d)
    ppos = pos[-P:]
    s, group = O.probe_scores(q, ppos, k, pos)
    kk = np.repeat(k, Hq // Hkv, axis=1).transpose(1, 0, 2)          # [Hq, Nc, d]
    ident = np.broadcast_to(np.eye(Nc), (Hq, Nc, Nc)).copy()
    mask = pos[None, :] <= ppos[:, None]
    a = _sdpa(q.transpose(1, 0, 2).copy(), kk.copy(), ident, mask)     # [Hq, P, Nc] weights
    want_group = a.sum(axis=1).reshape(Hkv, Hq // Hkv, Nc).sum(axis=1)
    np.testing.assert_allclose(group, want_group, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s, a.sum(axis=(0, 1)), rtol=1e-12, atol=1e-12)


def test_probe_scores_invariants_and_equal_keys_closed_form():
    Nc, P, Hq, Hkv, d = 50, 4, 4, 1, 8
    q, _, pos = _probe_case(Nc, P, Hq, Hkv, d, gaps=False)
    k = np.tile(rng.standard_normal(d), (Nc, Hkv, 1))               # all keys equal
    s, group = O.probe_scores(q, pos[-P:], k, pos)
    # every visible key gets 1 / (number visible) from each (head, probe) row
    want = np.zeros(Nc)
    for p in pos[-P:]:
        want[: p + 1] += Hq / (p + 1)
    np.testing.assert_allclose(s, want, rtol=1e-13)
    q, k, pos = _probe_case(300, 7, 8, 2, 16)
    s, group = O.probe_scores(q, pos[-7:], k, pos)
    assert abs(s.sum() - 7 * 8) < 1e-9
    np.testing.assert_allclose(group.sum(axis=1), [7 * 4, 7 * 4], rtol=1e-12)
    assert np.all(s >= 0)


# ---------------------------------------------------------------- LTP
def test_ltp_identity_proxy_is_leading_norm():
    D, r = 32, 8
    x = O.bf16_round(rng.standard_normal((10, D)))
    A = np.zeros((r, D)); A[:, :r] = np.eye(r)
    B = A.T.copy()                                                    # [D, r]
    np.testing.assert_allclose(O.ltp_scores(x, A, B), np.linalg.norm(x[:, :r], axis=1), rtol=1e-15)



def test_ltp_topm_brute_force_and_limits():
    # the sum of the m largest |y| equals the best m-subset sum (brute force),
    # the L1 norm at m = D_low and the largest |y| at m = 1
    import itertools
    x = O.bf16_round(rng.standard_normal((5, 16)))
    A = O.bf16_round(rng.standard_normal((4, 16)) * 0.3)
    B = O.bf16_round(rng.standard_normal((7, 4)) * 0.3)
    y = O.bf16_round(x @ A.T) @ B.T
    for m in (1, 3, 7):
        got = O.ltp_topm_scores(x, A, B, m)
        want = [max(sum(abs(row[j]) for j in sub) for sub in itertools.combinations(range(7), m)) for row in y]
        np.testing.assert_allclose(got, want, rtol=1e-14)
    np.testing.assert_allclose(O.ltp_topm_scores(x, A, B, 7), np.abs(y).sum(axis=1), rtol=1e-14)
    np.testing.assert_allclose(O.ltp_topm_scores(x, A, B, 1), np.abs(y).max(axis=1), rtol=1e-14)
    with pytest.raises(ValueError):
        O.ltp_topm_scores(x, A, B, 8)

def test_ltp_matches_torch_on_exact_intermediates():
    # integer inputs keep x A^T exact in bf16, so the rounding is a no-op
    D, r, Dout = 24, 6, 40
    x = rng.integers(-1, 2, (9, D)).astype(np.float64)
    A = rng.integers(-1, 2, (r, D)).astype(np.float64)
    B = rng.standard_normal((Dout, r))
    y = torch.from_numpy(x) @ torch.from_numpy(A).T @ torch.from_numpy(B).T
    want = torch.linalg.vector_norm(y, dim=1).numpy()
    np.testing.assert_allclose(O.ltp_scores(x, A, B), want, rtol=1e-13)


# ---------------------------------------------------------------- fusion
def test_fuse_modes_exact_values():
    s = np.array([1, 2, 4, 8], np.float32)
    c = np.array([8, 4, 2, 1], np.float32)
    f = O.fuse_scores(s, c, O.FUSE_MAXNORM_ADD, 0.5, 0.5)
    np.testing.assert_array_equal(f, np.array([0.5625, 0.375, 0.375, 0.5625], np.float32))
    # unequal weights: 0.25 s/8 + 0.75 c/8, exact in fp32
    f = O.fuse_scores(s, c, O.FUSE_MAXNORM_ADD, 0.25, 0.75)
    np.testing.assert_array_equal(f, np.array([0.78125, 0.4375, 0.3125, 0.34375], np.float32))
    f = O.fuse_scores(s, c, O.FUSE_MULTIPLY)
    np.testing.assert_array_equal(f, (torch.from_numpy(s) * torch.from_numpy(c)).numpy())
    np.testing.assert_array_equal(O.fuse_scores(s, c, O.FUSE_NONE), s)
    z = np.zeros(4, np.float32)
    np.testing.assert_array_equal(O.fuse_scores(s, z, O.FUSE_MAXNORM_ADD, 0.5, 0.5),
                                  np.float32(0.5) * (s / np.float32(8)))
    # max-normalisation makes the ranking invariant to scaling one term by 2**j
    s2 = rng.random(100).astype(np.float32); c2 = rng.random(100).astype(np.float32)
    f1 = O.fuse_scores(s2, c2, O.FUSE_MAXNORM_ADD, 0.3, 0.7)
    f2 = O.fuse_scores(s2 * np.float32(64), c2, O.FUSE_MAXNORM_ADD, 0.3, 0.7)
    np.testing.assert_array_equal(f1, f2)


# ---------------------------------------------------------------- select
def _brute_topk(f, k, tail):
    n = len(f)
    free = list(range(n - tail))
    ok = []
    for sub in itertools.combinations(free, k - tail):
        S = set(sub)
        good = all((f[i] > f[j]) or (f[i] == f[j] and i < j) for i in S for j in free if j not in S)
        if good:
            ok.append(sorted(sub) + list(range(n - tail, n)))
    assert len(ok) == 1
    return np.array(ok[0])


@pytest.mark.parametrize("n,k,tail", [(10, 4, 0), (10, 4, 2), (9, 9, 3), (8, 3, 3), (11, 1, 0), (7, 0, 0)])
def test_select_topk_brute_force_with_ties(n, k, tail):
    for trial in range(20):
        f = rng.integers(0, 4, n).astype(np.float32)                 # many ties
        if trial % 3 == 0:
            f[rng.integers(0, n)] = -0.0
        idx, tau = O.select_topk(f, k, tail)
        np.testing.assert_array_equal(idx, _brute_topk(f, k, tail))
        if k - tail > 0:
            assert tau == min(f[i] for i in idx[: k - tail])



def test_fuse_std_add_is_weighted_zscores():
    # Std-Add reduces to the library z-score (population std) of each score
    from scipy.stats import zscore
    s = rng.random(500).astype(np.float32)
    c = (rng.random(500) * 30).astype(np.float32)
    f = O.fuse_scores(s, c, O.FUSE_STD_ADD, 0.25, 0.75)
    want = 0.25 * zscore(s.astype(np.float64)) + 0.75 * zscore(c.astype(np.float64))
    np.testing.assert_allclose(f, want, rtol=0, atol=2e-6)
    # a constant score has std 0 and contributes nothing
    f0 = O.fuse_scores(np.full(500, 0.3, np.float32), c, O.FUSE_STD_ADD, 0.5, 0.5)
    np.testing.assert_allclose(f0, 0.5 * zscore(c.astype(np.float64)), rtol=0, atol=2e-6)


@pytest.mark.parametrize("k_pool", [20, 33, 60])
def test_select_sequential_reductions(k_pool):
    # pool of everything: the selection by c alone; pool of size k: the
    # selection by s alone; otherwise a subset of the pool holding the tail
    n, k, tail = 60, 20, 4
    s = rng.random(n).astype(np.float32)
    c = rng.random(n).astype(np.float32)
    c[rng.integers(0, n, 10)] = 0.5
    idx, _ = O.select_sequential(s, c, k_pool, k, tail)
    pool, _ = O.select_topk(s, k_pool, tail)
    assert len(idx) == k and np.all(np.diff(idx) > 0)
    assert set(idx) <= set(pool) and set(range(n - tail, n)) <= set(idx)
    if k_pool == n:
        assert np.array_equal(idx, O.select_topk(c, k, tail)[0])
    if k_pool == k:
        assert np.array_equal(idx, pool)
    # brute force inside the pool: no dropped pool member beats a kept one
    free_pool = [i for i in pool if i < n - tail]
    kept = [i for i in idx if i < n - tail]
    dropped = [i for i in free_pool if i not in kept]
    for a in kept:
        for b in dropped:
            assert c[a] > c[b] or (c[a] == c[b] and a < b)

def test_select_keep_all_and_errors():
    f = rng.random(33).astype(np.float32)
    idx, _ = O.select_topk(f, 33, 5)
    np.testing.assert_array_equal(idx, np.arange(33))
    with pytest.raises(ValueError):
        O.select_topk(f, 3, 5)
    with pytest.raises(ValueError):
        O.select_topk(np.array([1.0, np.nan], np.float32), 1, 0)


# ---------------------------------------------------------------- attention
def test_reduced_attention_matches_sdpa_rows():
    Nc, Hq, Hkv, d = 90, 8, 2, 16
    pos = np.cumsum(rng.integers(1, 3, Nc))
    k = rng.standard_normal((Nc, Hkv, d)); v = rng.standard_normal((Nc, Hkv, d))
    sel = np.sort(rng.choice(Nc, 23, replace=False))
    q = rng.standard_normal((23, Hq, d))
    got = O.reduced_attention(q, pos[sel], k, v, pos)
    kk = np.repeat(k, Hq // Hkv, axis=1).transpose(1, 0, 2).copy()
    vv = np.repeat(v, Hq // Hkv, axis=1).transpose(1, 0, 2).copy()
    mask = pos[None, :] <= pos[sel][:, None]
    want = _sdpa(q.transpose(1, 0, 2).copy(), kk, vv, mask).transpose(1, 0, 2)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_reduced_attention_special_cases():
    Nc, H, d = 40, 2, 8
    pos = np.arange(Nc)
    k = rng.standard_normal((Nc, H, d))
    v = np.broadcast_to(rng.standard_normal((1, H, d)), (Nc, H, d)).copy()
    q = rng.standard_normal((5, H, d))
    out = O.reduced_attention(q, pos[[0, 3, 9, 20, 39]], k, v, pos)
    np.testing.assert_allclose(out, np.broadcast_to(v[:1], out.shape), rtol=1e-13)
    v = rng.standard_normal((Nc, H, d))
    out = O.reduced_attention(q[:1], pos[:1], k, v, pos)            # query at pos 0 sees only key 0
    np.testing.assert_allclose(out[0], v[0], rtol=1e-14)


def test_attention_residual_rows():
    Nc, D, Hq, d = 30, 32, 4, 8
    h = rng.standard_normal((Nc, D))
    idx = np.array([2, 5, 6, 29])
    o = O.bf16_round(rng.standard_normal((4, Hq, d)))
    wo = rng.standard_normal((D, Hq * d))
    out = O.attention_residual(h, idx, o, wo)
    skip = np.setdiff1d(np.arange(Nc), idx)
    assert np.array_equal(out[skip], h[skip])
    want = h[idx] + F.linear(torch.from_numpy(o.reshape(4, -1)), torch.from_numpy(wo)).numpy()
    np.testing.assert_allclose(out[idx], want, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- FFN
def test_reduced_ffn_rows_match_torch_swiglu():
    Nc, D, Fh = 25, 32, 48
    h = rng.standard_normal((Nc, D))
    wg, wu = rng.standard_normal((Fh, D)) * 0.2, rng.standard_normal((Fh, D)) * 0.2
    wd = rng.standard_normal((D, Fh)) * 0.2
    nw = rng.standard_normal(D)
    idx = np.array([0, 4, 11, 24])
    out = O.reduced_ffn(h, idx, nw, 1e-5, wg, wu, wd)
    skip = np.setdiff1d(np.arange(Nc), idx)
    assert np.array_equal(out[skip], h[skip])
    x = F.rms_norm(torch.from_numpy(h[idx]), (D,), torch.from_numpy(nw), eps=1e-5)
    x = torch.from_numpy(O.bf16_round(x.numpy()))
    act = F.silu(F.linear(x, torch.from_numpy(wg))) * F.linear(x, torch.from_numpy(wu))
    act = torch.from_numpy(O.bf16_round(act.numpy()))
    want = h[idx] + F.linear(act, torch.from_numpy(wd)).numpy()
    np.testing.assert_allclose(out[idx], want, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- layer
def _tiny_layer(N=48, Hq=4, Hkv=2, d=8, Fh=24, r=4, P=3, k=None):
    D = Hq * d
    def w(o, i):
        return O.bf16_round(rng.standard_normal((o, i)) * 0.2)
    W = O.LayerWeights(w_q=w(Hq * d, D), w_k=w(Hkv * d, D), w_v=w(Hkv * d, D), w_o=w(D, Hq * d),
                       w_gate=w(Fh, D), w_up=w(Fh, D), w_down=w(D, Fh), ltp_a=w(r, D), ltp_b=w(D, r))
    h = O.bf16_round(rng.standard_normal((N, D)))
    pos = np.arange(N) * 2 + 5
    cfg = O.LayerConfig(Hq=Hq, Hkv=Hkv, d=d, P=P, k=N if k is None else k)
    return h, pos, W, cfg


def _dense_layer_torch(h, pos, W, cfg):
    """The dense Llama layer written with torch fp64 routines (keep = 1.0)."""
    B = O.bf16_round
    T = torch.from_numpy
    N, D = h.shape
    Hq, Hkv, d = cfg.Hq, cfg.Hkv, cfg.d
    x = B(F.rms_norm(T(h), (D,), eps=cfg.eps).numpy())
    q = B(O.rope(F.linear(T(x), T(W.w_q)).numpy().reshape(N, Hq, d), pos))
    k = B(O.rope(F.linear(T(x), T(W.w_k)).numpy().reshape(N, Hkv, d), pos))
    v = B(F.linear(T(x), T(W.w_v)).numpy().reshape(N, Hkv, d))
    kk = np.repeat(k, Hq // Hkv, axis=1).transpose(1, 0, 2).copy()
    vv = np.repeat(v, Hq // Hkv, axis=1).transpose(1, 0, 2).copy()
    o = B(F.scaled_dot_product_attention(T(q.transpose(1, 0, 2).copy()), T(kk), T(vv),
                                         is_causal=True).numpy().transpose(1, 0, 2))
    h1 = h + F.linear(T(o.reshape(N, -1)), T(W.w_o)).numpy()
    x2 = B(F.rms_norm(T(h1), (D,), eps=cfg.eps).numpy())
    act = B((F.silu(F.linear(T(x2), T(W.w_gate))) * F.linear(T(x2), T(W.w_up))).numpy())
    return h1 + F.linear(T(act), T(W.w_down)).numpy()


def test_layer_keep_all_equals_dense_layer():
    h, pos, W, cfg = _tiny_layer()
    out, _ = O.layer_forward(h, pos, W, cfg)
    np.testing.assert_allclose(out, _dense_layer_torch(h, pos, W, cfg), rtol=1e-11, atol=1e-11)



def test_layer_kv_active_keep_all_equals_dense_layer():
    # with every row active, the active-row keys are all keys: the dense layer
    h, pos, W, cfg = _tiny_layer()
    cfg.kv_active = True
    out, _ = O.layer_forward(h, pos, W, cfg)
    np.testing.assert_allclose(out, _dense_layer_torch(h, pos, W, cfg), rtol=1e-11, atol=1e-11)


def test_layer_kv_active_attention_is_dense_attention_of_the_active_rows():
    # with keys restricted to the active rows, each selected query attends as
    # in a dense causal layer run on the subsequence of the selected rows
    h, pos, W, cfg = _tiny_layer(N=64, k=21, P=3)
    cfg.kv_active = True
    tr = {}
    O.layer_forward(h, pos, W, cfg, tr)
    idx = tr["idx_attn"]
    T = torch.from_numpy
    Hq, Hkv, d, m = cfg.Hq, cfg.Hkv, cfg.d, len(idx)
    x = T(tr["xn"][idx])
    k = O.bf16_round(O.rope(F.linear(x, T(W.w_k)).numpy().reshape(m, Hkv, d), pos[idx]))
    v = O.bf16_round(F.linear(x, T(W.w_v)).numpy().reshape(m, Hkv, d))
    kk = np.repeat(k, Hq // Hkv, axis=1).transpose(1, 0, 2).copy()
    vv = np.repeat(v, Hq // Hkv, axis=1).transpose(1, 0, 2).copy()
    q = tr["q_sel"].transpose(1, 0, 2).copy()
    want = F.scaled_dot_product_attention(T(q), T(kk), T(vv), is_causal=True).numpy().transpose(1, 0, 2)
    np.testing.assert_allclose(tr["o_sel"], O.bf16_round(want), rtol=0, atol=1e-12)

def test_layer_skipped_rows_pass_through():
    h, pos, W, cfg = _tiny_layer(N=64, k=20, P=4)
    tr = {}
    out, f = O.layer_forward(h, pos, W, cfg, tr)
    touched = np.union1d(tr["idx_attn"], tr["idx_ffn"])
    skip = np.setdiff1d(np.arange(64), touched)
    assert len(skip) > 0
    assert np.array_equal(out[skip], h[skip])
    assert set(range(60, 64)) <= set(tr["idx_attn"]) and set(range(60, 64)) <= set(tr["idx_ffn"])
    assert len(tr["idx_attn"]) == 20 and np.all(np.diff(tr["idx_attn"]) > 0)


def _top_k_rows(score, k, tail):
    """Top-k by plain sorting (largest first, ties to the lower index), the
    last `tail` rows forced, ascending."""
    n = len(score)
    free = sorted(range(n - tail), key=lambda i: (-float(score[i]), i))[: k - tail]
    return np.array(sorted(free) + list(range(n - tail, n)))


@pytest.mark.parametrize("w_a,w_b", [(0.0, 1.0), (1.0, 0.0)])
def test_layer_selection_wiring(w_a, w_b):
    # with one fusion weight zero, the FFN rows are the top-k of one score:
    # of the LTP score of RMSNorm(h') (h' = the attention output) for w_a =
    # 0, of the probe score for w_b = 0 (the attention rows); attention
    # changes exactly its rows of h, the FFN exactly its rows of h'
    h, pos, W, cfg = _tiny_layer(N=40, k=12, P=3)
    cfg.w_a, cfg.w_b = w_a, w_b
    tr = {}
    out, _ = O.layer_forward(h, pos, W, cfg, tr)
    # the probes are the last P rows, at their own positions
    Hq, d = cfg.Hq, cfg.d
    q_probe = O.bf16_round(O.rope((tr["xn"][-3:] @ W.w_q.T).reshape(3, Hq, d), pos[-3:]))
    np.testing.assert_allclose(tr["s"], O.probe_scores(q_probe, pos[-3:], tr["k"], pos)[0], rtol=1e-12)
    want_a = _top_k_rows(tr["s"].astype(np.float32), 12, 3)
    assert np.array_equal(tr["idx_attn"], want_a)
    assert np.array_equal(np.nonzero(np.any(tr["h_attn"] != h, axis=1))[0], want_a)
    c = O.ltp_scores(O.bf16_round(O.rmsnorm(tr["h_attn"], W.norm_ffn, cfg.eps)), W.ltp_a, W.ltp_b)
    # the LTP score itself, not only its ranking, is that of RMSNorm(h')
    np.testing.assert_allclose(tr["c"], c, rtol=1e-12, atol=0)
    want_f = _top_k_rows(c.astype(np.float32), 12, 3) if w_a == 0 else want_a
    assert np.array_equal(tr["idx_ffn"], want_f)
    assert np.array_equal(np.nonzero(np.any(out != tr["h_attn"], axis=1))[0], want_f)


def test_msdp_all_ratios_one_is_dense_stack_and_sets_nest():
    h, pos, W0, cfg = _tiny_layer(N=40, P=2)
    layers = [W0] + [_tiny_layer(N=40, P=2)[2] for _ in range(3)]
    m = O.MsdpConfig(layer=cfg, ratios=("1", "1"), layers_per_stage=2)
    out, opos, pruned = O.msdp_forward(h, pos, layers, m)
    ref = h
    for W in layers:
        ref = _dense_layer_torch(ref, pos, W, cfg)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-10)
    assert np.array_equal(opos, pos) and all(len(p[0]) == 0 for p in pruned)
    # nested candidate sets, tail always kept
    m = O.MsdpConfig(layer=cfg, ratios=("0.8", "0.6", "0.4", "0.25"), layers_per_stage=1)
    layers = [_tiny_layer(N=40, P=2)[2] for _ in range(4)]
    tr = []
    out, opos, pruned = O.msdp_forward(h, pos, layers, m, tr)
    assert len(opos) == 10
    sizes = [40]
    seen = set(pos.tolist())
    for (ppos, _), lt in zip(pruned, tr):
        seen -= set(ppos.tolist())
        sizes.append(len(seen))
    assert sizes == [40, 32, 24, 16, 10]
    assert set(opos.tolist()) == seen and {pos[-1], pos[-2]} <= seen


def test_msdp_prunes_by_the_last_layers_fused_score():
    # at each stage boundary the candidates kept are the top-k_s of the
    # stage's last layer's fused score (plain sorting, tail forced)
    h, pos, W0, cfg = _tiny_layer(N=40, P=2)
    layers = [_tiny_layer(N=40, P=2)[2] for _ in range(6)]
    m = O.MsdpConfig(layer=cfg, ratios=("0.75", "0.5", "0.3"), layers_per_stage=2)
    tr = []
    out, opos, pruned = O.msdp_forward(h, pos, layers, m, tr)
    cand = pos
    for s_i, r in enumerate(m.ratios):
        k_s = O.keep_count(r, 40)
        last = tr[2 * s_i + 1]
        keep = _top_k_rows(last["f"], k_s, 2)
        nxt = cand[keep]
        assert np.array_equal(np.sort(pruned[s_i][0]), np.setdiff1d(cand, nxt))
        cand = nxt
    assert np.array_equal(opos, cand)


def test_stage_prune_worked_example():
    scores = np.array([0.1, 0.9, 0.5, 0.9, 0.3, 0.2], np.float32)
    h = np.arange(12.0).reshape(6, 2)
    pos = np.array([3, 8, 9, 20, 21, 30])
    # keep 4, tail 1: the top 3 of the first 5 (0.9 at 1 and 3, then 0.5 at 2), then row 5
    ho, po, kept = O.stage_prune(scores, 4, 1, h, pos)
    assert list(kept) == [1, 2, 3, 5] and list(po) == [8, 9, 20, 30]
    np.testing.assert_array_equal(ho, h[[1, 2, 3, 5]])


def test_schedule_without_skipping_is_the_dense_stack_and_sets_nest():
    # budgets and the final count at least N: every layer is a full layer
    h, pos, W0, cfg = _tiny_layer(N=40, P=2)
    layers = [W0] + [_tiny_layer(N=40, P=2)[2] for _ in range(5)]
    out, opos = O.schedule_forward(h, pos, layers, cfg, 1, (2, 4), (40, 50), 40)
    want = h
    for W in layers:
        want = _dense_layer_torch(want, pos, W, cfg)
    np.testing.assert_allclose(out, want, rtol=1e-10, atol=1e-10)
    assert np.array_equal(opos, pos)
    # with budgets: k per layer, candidate sets nest, the tail survives
    tr = []
    out, opos = O.schedule_forward(h, pos, layers, cfg, 1, (2, 4), (30, 20), 10, tr)
    assert [t["k"] for t in tr] == [40, 30, 30, 20, 20, 10]
    assert [len(t["cand"]) for t in tr] == [40, 40, 40, 30, 30, 10]
    assert [t["skip"] for t in tr] == [False, True, True, True, True, False]
    for t in tr:
        assert set(t["sel_pos"]) <= set(t["cand"]) and set(pos[-2:]) <= set(t["sel_pos"])
    for a, b in zip(tr, tr[1:]):
        assert set(b["cand"]) <= set(a["cand"])
    assert np.array_equal(opos, tr[-1]["cand"]) and out.shape == (10, h.shape[1])
    # more survivors than the last stage's budget: the layers after the last
    # stage are still full layers over every survivor
    tr = []
    out, opos = O.schedule_forward(h, pos, layers, cfg, 1, (2, 4), (30, 20), 25, tr)
    assert [t["k"] for t in tr] == [40, 30, 30, 20, 20, 25]
    assert [len(t["cand"]) for t in tr] == [40, 40, 40, 30, 30, 25]
    assert not tr[-1]["skip"] and np.array_equal(np.sort(tr[-1]["sel_pos"]), np.sort(tr[-1]["cand"]))


# ---------------------------------------------------------------- synthetic salience
def test_inject_salience_closed_form():
    # two probes x two heads of one KV group: mean (0.5, 0.5, 0, 0) -> unit (1, 1, 0, 0)/sqrt(2)
    q = np.zeros((2, 2, 4))
    q[0, :, 0] = 1.0
    q[1, :, 1] = 1.0
    k = np.zeros((5, 1, 4))
    k[:, 0, 3] = 0.5
    out = O.inject_salience(k, q, np.array([1, 3]), 3.0, 1)
    add = 3.0 / math.sqrt(2.0)
    want = k.copy()
    want[[1, 3], 0, 0] = torch.tensor(add, dtype=torch.float32).to(torch.bfloat16).item()
    want[[1, 3], 0, 1] = want[1, 0, 0]
    np.testing.assert_array_equal(out, want)
    # two KV groups of two heads each (heads 0-1 read group 0, heads 2-3
    # group 1): each group's keys move along its own heads' mean direction
    q = np.zeros((1, 4, 4))
    q[0, 0:2, 0] = 1.0
    q[0, 2:4, 1] = 1.0
    k = np.zeros((3, 2, 4))
    out = O.inject_salience(k, q, np.array([2]), 2.0, 2)
    want = np.zeros_like(k)
    want[2, 0, 0] = 2.0
    want[2, 1, 1] = 2.0
    np.testing.assert_array_equal(out, want)


# ---------------------------------------------------------------- accounting
def _golden(golden_dir, name):
    rows = []
    for line in open(os.path.join(golden_dir, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(line.split())
    return rows


def test_table_a_ltp_cost(golden_dir):
    rows = _golden(golden_dir, "table_a_ltp_cost.txt")
    assert len(rows) == 6
    for d_low, r, printed, flag in rows:
        macs = O.ltp_proxy_macs(4096, int(d_low), None if r == "/" else int(r))
        if flag == "ok":
            assert round(macs / 1000) == int(printed)
        else:
            assert round(macs / 1000) != int(printed) and macs == 884736


def test_table5_kv_cache(golden_dir):
    rows = _golden(golden_dir, "table5_kv_cache.txt")
    assert len(rows) == 4
    for n, full, pap, saving in rows:
        n = int(n)
        f_ = O.kv_cache_gib(n, with_pap=False)
        p_ = O.kv_cache_gib(n)
        assert f"{f_:.2f}" == full
        assert abs(p_ - float(pap)) <= 0.005 + 1e-12
        assert f"{100 * (1 - p_ / f_):.1f}" == saving


def test_keep_counts_exact():
    assert [O.keep_count(r, n) for r, n in [("0.25", 512), ("0.4", 8192), ("0.3", 32768), ("0.2", 131072)]] \
        == [128, 3276, 9830, 26214]
    assert [O.keep_count(r, 32768) for r in ("0.8", "0.6", "0.4", "0.25")] == [26214, 19660, 13107, 8192]
