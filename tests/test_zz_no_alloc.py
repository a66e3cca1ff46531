"""The allocation-free stage prune (spts_stage_prune_noalloc) on the GPU.

Some callers cannot allocate device memory when they call the library -- a
plugin inside a host framework that reserved all GPU memory up front, or a
latency-critical loop that cannot take cudaMalloc's implicit
synchronisation.  For them spts_stage_prune_noalloc keeps its index scratch
in a fixed device array inside the library.  These tests call it through the
C ABI twice in a row and compare each result with the workspace-based
spts_stage_prune on the same inputs; the results are integer indices and
copied rows, so they must match exactly.  This file is named to run last.
"""

import numpy as np
import pytest
import torch

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


def test_noalloc_prune_matches_workspace_prune_on_two_calls():
    for Nc, D, keep, tail, seed in [(100000, 64, 30000, 64, 1), (5000, 256, 1234, 16, 2)]:
        scores, h, pos = _case(Nc, D, seed)
        want_h, want_pos, want_kept = S.spts_stage_prune(scores, keep, tail, h, pos)
        got_h, got_pos = S.spts_stage_prune_noalloc(scores, keep, tail, h, pos)
        torch.cuda.synchronize()
        assert torch.equal(got_pos, want_pos)
        assert torch.equal(got_h, want_h)
        assert torch.equal(pos[want_kept.long()], got_pos)


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
