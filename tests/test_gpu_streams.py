"""The layer's side-stream overlap (V and probe-Q projections on a second
stream) must not change any result: the same kernels run on the same data,
so outputs are bit-identical to the all-on-one-stream run (which
spts_layer_forward uses when given any of the stage events 1..7), on the
default stream and on a caller's non-default stream."""

import pytest
import torch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import token_skipping_sparse_b200 as S


def _case():
    from synthetic import WORKLOADS, make_hidden, make_layer_weights, salient_rows
    wl = WORKLOADS["layer_small"]
    W = {n: t.cuda() for n, t in make_layer_weights(wl).items()}
    sal = salient_rows(wl.N, wl.P, wl.salient_frac, wl.seed).cuda()
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, wl.k, fuse=wl.fuse, salient_rows=sal,
                        salient_shift=wl.salient_shift)
    return wl, make_hidden(wl).cuda(), W, torch.arange(wl.N, dtype=torch.int32, device="cuda"), desc


def _outs(wl, desc):
    k = desc.k
    return dict(s=torch.empty(wl.N, device="cuda"), idx_attn=torch.empty(k, dtype=torch.int32, device="cuda"),
                idx_ffn=torch.empty(k, dtype=torch.int32, device="cuda"))


def test_side_stream_overlap_is_bit_identical():
    wl, h0, W, pos, desc = _case()
    h_seq = h0.clone()
    o_seq = _outs(wl, desc)
    S.spts_layer_forward(h_seq, pos, desc, W, outputs=o_seq, events=S.stage_events())
    h_par = h0.clone()
    o_par = _outs(wl, desc)
    S.spts_layer_forward(h_par, pos, desc, W, outputs=o_par)
    torch.cuda.synchronize()
    S.check_device_status()
    assert torch.equal(h_seq, h_par)
    for n in o_seq:
        assert torch.equal(o_seq[n], o_par[n]), n


def test_layer_on_a_caller_stream_joins_before_return():
    wl, h0, W, pos, desc = _case()
    ref = h0.clone()
    S.spts_layer_forward(ref, pos, desc, W)
    st = torch.cuda.Stream()
    h = h0.clone()
    torch.cuda.synchronize()
    with torch.cuda.stream(st):
        for _ in range(3):                 # back to back on the caller's stream
            hh = h0.clone()
            S.spts_layer_forward(hh, pos, desc, W)
        out = hh.clone()                   # ordered after the layer on st
    st.synchronize()
    assert torch.equal(out, ref)


def _pair_events(first):
    """Stage-event list with only events `first` and `first + 1` set (each
    recorded once so that its CUDA handle exists)."""
    evs = [None] * S.LAYER_STAGE_EVENTS
    for i in (first, first + 1):
        evs[i] = torch.cuda.Event(enable_timing=True)
        evs[i].record()
    torch.cuda.synchronize()
    return evs


@pytest.mark.parametrize("stage", ["reduced_attention", "gate_up_swiglu"])
def test_timing_one_kernel_keeps_the_result_and_times_it(stage):
    """Events around one kernel past the side stream's join (how bench.py
    times the dominant kernel inside its timed region): the layer's outputs
    are bit-identical to the run without events, and the pair measures a
    positive time no longer than the whole layer."""
    wl, h0, W, pos, desc = _case()
    i = S.LAYER_STAGES.index(stage)
    assert i >= 8  # events 1..7 would switch the layer to one stream
    ref, o_ref = h0.clone(), _outs(wl, desc)
    S.spts_layer_forward(ref, pos, desc, W, outputs=o_ref)
    evs = _pair_events(i)
    whole = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    h, o = h0.clone(), _outs(wl, desc)
    whole[0].record()
    S.spts_layer_forward(h, pos, desc, W, outputs=o, events=evs)
    whole[1].record()
    torch.cuda.synchronize()
    S.check_device_status()
    assert torch.equal(h, ref)
    for n in o:
        assert torch.equal(o[n], o_ref[n]), n
    t = evs[i].elapsed_time(evs[i + 1])
    assert 0.0 < t <= whole[0].elapsed_time(whole[1])
