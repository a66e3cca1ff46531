"""The fp32 timed mode of the oracle (oracle/timed.py) computes the same layer
as the fp64 oracle: checked on the CPU at small sizes.

The timed mode exists only to time whole layers at full size on the host; it
is pinned here to oracle.spts, which carries the pins to the pages and to
library routines.  Same inputs, fp32 against fp64: scores within fp32
rounding, selections equal up to near-ties of the fp64 scores, outputs within
the bf16 path's per-call bound (both sides round the same operands to bf16).
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
from oracle import timed as T
from synthetic import WORKLOADS, make_hidden, make_layer_weights, salient_rows
from tests.gpu_util import band_check


def _f64(W):
    return {n: t.float().double().numpy() for n, t in W.items()}


@pytest.mark.parametrize("name", ["layer_small", "layer_small_mul", "layer_small_p1"])
def test_timed_layer_matches_fp64_oracle(name):
    wl = WORKLOADS[name]
    h = make_hidden(wl)
    W = make_layer_weights(wl)
    sal = salient_rows(wl.N, wl.P, wl.salient_frac, wl.seed)
    pos = torch.arange(wl.N)
    ho, s, c, f, ia, idf = T.layer_forward(h, pos, {n: t.float() for n, t in W.items()}, wl.Hq, wl.Hkv, wl.P, wl.k,
                                           wl.fuse, salient_rows=sal.long(), salient_shift=wl.salient_shift)
    cfg = O.LayerConfig(Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, P=wl.P, k=wl.k, fuse=wl.fuse, salient_rows=sal.numpy(),
                        salient_shift=wl.salient_shift)
    tr = {}
    O.layer_forward(h.double().numpy(), pos.numpy(), O.LayerWeights(**_f64(W)), cfg, tr)
    assert np.abs(s.numpy() - tr["s"]).max() <= 1e-4 * tr["s"].max()
    band_check(ia.numpy(), tr["idx_attn"], tr["s"], tr["tau_attn"])
    assert np.abs(c.numpy() - tr["c"]).max() <= 1e-3 * tr["c"].max()
    band_check(idf.numpy(), tr["idx_ffn"], tr["f"], tr["tau_ffn"])
    assert np.array_equal(ia.numpy(), tr["idx_attn"]) and np.array_equal(idf.numpy(), tr["idx_ffn"]), \
        "these seeds have no near-tie at the threshold"
    assert np.abs(ho.double().numpy() - tr["h_out"]).max() <= 2e-2


def test_timed_attention_only_layer_matches_fp64_oracle():
    """The attention-only layer (the 8K configuration's steps): h after the
    O projection, the probe scores and the MHA selection."""
    wl = WORKLOADS["layer_small"]
    h = make_hidden(wl)
    W = make_layer_weights(wl)
    sal = salient_rows(wl.N, wl.P, wl.salient_frac, wl.seed)
    pos = torch.arange(wl.N)
    ho, s, c, f, ia, idf = T.layer_forward(h, pos, {n: t.float() for n, t in W.items()}, wl.Hq, wl.Hkv, wl.P, wl.k,
                                           wl.fuse, salient_rows=sal.long(), salient_shift=wl.salient_shift,
                                           ffn=False)
    assert c is None and f is None and idf is None
    cfg = O.LayerConfig(Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, P=wl.P, k=wl.k, fuse=wl.fuse, salient_rows=sal.numpy(),
                        salient_shift=wl.salient_shift, ffn=False)
    tr = {}
    want, _ = O.layer_forward(h.double().numpy(), pos.numpy(), O.LayerWeights(**_f64(W)), cfg, tr)
    assert np.abs(s.numpy() - tr["s"]).max() <= 1e-4 * tr["s"].max()
    assert np.array_equal(ia.numpy(), tr["idx_attn"])
    assert np.abs(ho.double().numpy() - tr["h_attn"]).max() <= 2e-2
    assert np.abs(ho.double().numpy() - want).max() <= 2e-2
    rest = np.setdiff1d(np.arange(wl.N), ia.numpy())
    assert torch.equal(ho[rest], h[rest])


def test_timed_attention_key_range_is_exact():
    """Each slab reads keys up to its last query's position only: the same
    result as masked attention over every key (brute force, fp64 oracle)."""
    g = torch.Generator().manual_seed(5)
    Nc, m, Hq, Hkv, d = 700, 300, 4, 2, 64
    key_pos = torch.sort(torch.randperm(3 * Nc, generator=g)[:Nc]).values
    sel = torch.sort(torch.randperm(Nc, generator=g)[:m]).values
    q = torch.randn(m, Hq, d, generator=g)
    kk = torch.randn(Nc, Hkv, d, generator=g)
    vv = torch.randn(Nc, Hkv, d, generator=g)
    for slab in (1, 37, 1024):
        o = T._attention(q, key_pos[sel], kk, vv, key_pos, Hq // Hkv, slab=slab)
        want = O.reduced_attention(q.double().numpy(), key_pos[sel].numpy(), kk.double().numpy(),
                                   vv.double().numpy(), key_pos.numpy(), 1.0 / math.sqrt(d))
        assert np.abs(o.double().numpy() - want).max() < 1e-5


def test_timed_topk_rule():
    f = torch.tensor([0.5, 0.9, 0.5, 0.1, 0.9, 0.2, 0.3], dtype=torch.float32)
    assert T._topk(f, 4, 2).tolist() == [1, 4, 5, 6]          # the tail forced, then 0.9, 0.9
    assert T._topk(f, 5, 2).tolist() == [0, 1, 4, 5, 6]       # equal 0.5s: the lower index first
    for k in range(2, 8):
        assert np.array_equal(T._topk(f, k, 2).numpy(), O.select_topk(f.numpy(), k, 2)[0])
