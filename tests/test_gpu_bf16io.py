"""spts_layer_forward_bf16io: the layer on a residual stream held in bf16 at
the boundary.  It runs the same kernels on an fp32 copy of h, so its output
must be the fp32 layer's output rounded to bf16 (nearest even), bit for bit,
and every row the layer skipped keeps its input bits."""

import pytest
import torch

from synthetic import WORKLOADS, make_hidden, make_layer_weights, salient_rows

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import token_skipping_sparse_b200 as S


@pytest.mark.parametrize("name,keep_all", [("layer_small", False), ("layer_small_kv", False),
                                           ("layer_small_mul", False), ("layer_small_rho", False),
                                           ("layer_small", True)])
def test_bf16_boundary_is_the_fp32_layer_rounded(name, keep_all):
    wl = WORKLOADS[name]
    h = make_hidden(wl)                       # bf16 values held in fp32: exact in bf16
    W = {n: t.cuda() for n, t in make_layer_weights(wl).items()}
    sal = salient_rows(wl.N, wl.P, wl.salient_frac, wl.seed).cuda()
    k = wl.N if keep_all else wl.k
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, k, fuse=wl.fuse,
                        salient_rows=None if keep_all else sal, salient_shift=wl.salient_shift,
                        ltp_dout=wl.ltp_dout, ltp_top_m=wl.ltp_top_m, kv_active_only=wl.kv_active)
    pos = torch.arange(wl.N, dtype=torch.int32, device="cuda")
    hf = h.cuda()
    S.spts_layer_forward(hf, pos, desc, W)
    hb = h.to(torch.bfloat16).cuda()
    S.spts_layer_forward_bf16io(hb, pos, desc, W)
    S.check_device_status()
    assert torch.equal(hb.view(torch.int16), hf.to(torch.bfloat16).view(torch.int16))
    changed = (hf != h.cuda()).any(dim=1)
    assert changed.any()
    unchanged = ~changed
    assert torch.equal(hb[unchanged].view(torch.int16), h.to(torch.bfloat16).cuda()[unchanged].view(torch.int16))


def test_bf16_boundary_rejects_misaligned_h():
    wl = WORKLOADS["layer_small"]
    W = {n: t.cuda() for n, t in make_layer_weights(wl).items()}
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, wl.k, fuse=wl.fuse)
    buf = torch.zeros(wl.N * wl.D + 8, dtype=torch.bfloat16, device="cuda")
    h = buf[1:1 + wl.N * wl.D].view(wl.N, wl.D)          # 2-byte offset: not 16-byte aligned
    pos = torch.arange(wl.N, dtype=torch.int32, device="cuda")
    with pytest.raises(S.SptsError) as e:
        S.spts_layer_forward_bf16io(h, pos, desc, W)
    assert e.value.status == S.ERR_INVALID
