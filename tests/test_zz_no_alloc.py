"""The allocation-free stage prune (spts_stage_prune_noalloc) on the GPU.

Some callers cannot allocate device memory when they call the library -- a
plugin inside a host framework that reserved all GPU memory up front, or a
latency-critical loop that cannot take cudaMalloc's implicit
synchronisation.  For them spts_stage_prune_noalloc keeps its index scratch
in a fixed device array inside the library.  These tests call it through the
C ABI and compare it with the workspace-based spts_stage_prune on the same
inputs, and with the oracle's stage prune; the results are integer indices
and copied rows, so they must match exactly.  The calls come in pairs on one
device -- the larger first, so the smaller one meets stale indices past its
k_keep in the shared array -- with and without caller-supplied kept indices.
After the set-up call (Nc == 0), repeated calls must leave the device's free
memory unchanged.  This file is named to run last.
"""

import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import token_skipping_sparse_b200 as S


def _case(Nc, D, seed):
    g = torch.Generator().manual_seed(seed)
    scores = torch.rand(Nc, generator=g)
    scores[torch.randint(0, Nc, (Nc // 20,), generator=g)] = 0.5     # ties
    h = torch.randn(Nc, D, generator=g)
    pos = torch.sort(torch.randperm(4 * Nc, generator=g)[:Nc]).values.to(torch.int32)
    return scores.cuda(), h.cuda(), pos.cuda()


def _setup():
    S.check(S.lib.spts_stage_prune_noalloc(None, 0, 0, 0, None, None, 0, None, None, None, S.stream_ptr()))


def _raw_call(scores, keep, tail, h, pos, h_out, pos_out, kept=None):
    """The C entry point with caller-owned outputs (nothing allocated here)."""
    return S.lib.spts_stage_prune_noalloc(S.ptr(scores), scores.shape[0], keep, tail, S.ptr(h), S.ptr(pos),
                                          h.shape[1], S.ptr(h_out), S.ptr(pos_out), S.ptr(kept), S.stream_ptr())


CASES = [(100000, 64, 30000, 64, 1), (5000, 256, 1234, 16, 2)]   # the larger call first


def test_noalloc_prune_matches_workspace_prune_and_oracle_on_two_calls():
    _setup()
    for use_kept in (False, True):
        for Nc, D, keep, tail, seed in CASES:
            scores, h, pos = _case(Nc, D, seed)
            want_h, want_pos, want_kept = S.spts_stage_prune(scores, keep, tail, h, pos)
            kept = torch.full((keep,), -1, dtype=torch.int32, device="cuda") if use_kept else None
            got_h, got_pos = S.spts_stage_prune_noalloc(scores, keep, tail, h, pos, kept=kept)
            torch.cuda.synchronize()
            assert torch.equal(got_pos, want_pos)
            assert torch.equal(got_h, want_h)
            if use_kept:
                assert torch.equal(kept, want_kept)
            # the oracle's prune: top-k_keep by score, tail forced, ties to the lower index
            o_h, o_pos, o_kept = O.stage_prune(scores.cpu().numpy(), keep, tail, h.cpu().numpy(), pos.cpu().numpy())
            assert np.array_equal(got_pos.cpu().numpy(), o_pos)
            assert np.array_equal(got_h.cpu().numpy(), o_h)


def test_noalloc_prune_takes_no_device_memory_after_setup():
    Nc, D, keep, tail, seed = CASES[0]
    scores, h, pos = _case(Nc, D, seed)
    h_out = torch.empty(keep, D, device="cuda")
    pos_out = torch.empty(keep, dtype=torch.int32, device="cuda")
    _setup()
    S.check(_raw_call(scores, keep, tail, h, pos, h_out, pos_out))
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(5):
        S.check(_raw_call(scores, keep, tail, h, pos, h_out, pos_out))
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    want_h, want_pos, _ = S.spts_stage_prune(scores, keep, tail, h, pos)
    assert torch.equal(h_out, want_h) and torch.equal(pos_out, want_pos)


def test_noalloc_prune_rejects_oversize_and_leaves_context_usable():
    n = S.NOALLOC_MAX_NC + 1
    scores = torch.zeros(n, device="cuda")
    h = torch.zeros(n, 4, device="cuda")
    pos = torch.arange(n, dtype=torch.int32, device="cuda")
    with pytest.raises(S.SptsError) as e:
        S.spts_stage_prune_noalloc(scores, 8, 0, h, pos)
    assert e.value.status == S.ERR_SHAPE
    scores, h, pos = _case(3000, 32, 3)
    got_h, got_pos = S.spts_stage_prune_noalloc(scores, 100, 4, h, pos)
    want_h, want_pos, _ = S.spts_stage_prune(scores, 100, 4, h, pos)
    assert torch.equal(got_h, want_h) and torch.equal(got_pos, want_pos)
    assert np.all(np.diff(got_pos.cpu().numpy()) > 0)
