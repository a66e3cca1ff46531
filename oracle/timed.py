"""fp32 timed mode of the oracle: one whole SPTS layer on the host's cores.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: used by
``bench.py``'s CPU baseline and reference legs to time a full-size layer,
and by ``tests/`` (which pin it to the fp64 oracle).  The product never
imports it.

What it computes is the layer of "Probe and Skip: Self-Predictive Token
Skipping for Efficient Long-Context LLM Inference" in the order of Fig. 2:
the PAP probe scores (Fig. 2(a)), the MHA selection, reduced attention over
the selected rows, the O projection into them, the LTP score of the FFN input
(Fig. 2(b), Table 6), the fused FFN selection (Table D) and the reduced FFN
-- the same definitions and readings as ``oracle.spts.layer_forward``, with
the same bf16 roundings of the product operands, but in fp32 with plain
torch CPU operations (matrix products, softmax, sort), so that a 32K-token
layer runs in seconds on all host threads instead of minutes in fp64 numpy.
Each softmax row is formed whole and masked (no online softmax); the only
restructuring is that reduced attention processes one head and a slab of
query rows at a time, over the keys up to the slab's last query position
(every later key is masked for the whole slab), so the logits fit in host
memory.
"""

from __future__ import annotations

import math

import torch

FUSE_NONE, FUSE_MAXNORM_ADD, FUSE_MULTIPLY = 0, 1, 2


def _bf16(x):
    """Round-to-nearest-even to bf16, held in fp32."""
    return x.to(torch.bfloat16).float()


def _rmsnorm(x, eps=1e-5):
    return x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + eps)


def _rope(x, pos, theta=500000.0):
    """Rotate-half RoPE at the given positions; x [m, H, d] fp32."""
    d = x.shape[-1]
    inv = theta ** (-torch.arange(0, d // 2, dtype=torch.float64) * 2.0 / d)
    ang = pos.to(torch.float64)[:, None] * inv[None, :]
    cos, sin = ang.cos().float()[:, None, :], ang.sin().float()[:, None, :]
    a, b = x[..., : d // 2], x[..., d // 2:]
    return torch.cat([a * cos - b * sin, a * sin + b * cos], dim=-1)


def _topk(f, k, tail):
    """The last ``tail`` rows forced, the top k - tail of the rest by score
    (ties to the lower index), ascending."""
    n = f.shape[0]
    order = torch.argsort(-f[: n - tail], stable=True)[: k - tail]
    return torch.cat([torch.sort(order).values, torch.arange(n - tail, n)])


def _salience(kk, qp, rows, shift, Hkv):
    """Synthetic-workload step: shift the planted keys toward the mean probe query of their group."""
    G = qp.shape[1] // Hkv
    for g in range(Hkv):
        m = qp[:, g * G:(g + 1) * G, :].reshape(-1, qp.shape[-1]).double().mean(0)
        kk[rows, g, :] = _bf16(kk[rows, g, :] + (shift * m / m.norm()).float())
    return kk


def _attention(q, q_pos, kk, vv, key_pos, G, slab=1024):
    """Causal GQA softmax attention of the rows q [m, Hq, d] over all keys
    kk / vv [Nc, Hkv, d] with pos_key <= pos_query; one head and at most
    ``slab`` query rows per softmax block.  Query and key positions ascend,
    so a block's keys past its last query's position are masked for every
    row of the block: they are left out of its products (an exact step)."""
    m, Hq, d = q.shape
    scale = 1.0 / math.sqrt(d)
    out = torch.empty(m, Hq, d)
    for a in range(0, m, slab):
        b = min(m, a + slab)
        n_vis = int(torch.searchsorted(key_pos, q_pos[b - 1], right=True))
        hidden = key_pos[None, :n_vis] > q_pos[a:b, None]
        for h in range(Hq):
            logits = (q[a:b, h, :] @ kk[:n_vis, h // G, :].T) * scale
            logits.masked_fill_(hidden, float("-inf"))
            out[a:b, h, :] = torch.softmax(logits, dim=1) @ vv[:n_vis, h // G, :]
    return out


def layer_forward(h, pos, W, Hq, Hkv, P, k, fuse=FUSE_MAXNORM_ADD, w_a=0.5, w_b=0.5, salient_rows=None,
                  salient_shift=0.0, ffn=True):
    """One SPTS layer in fp32 on the host: h [Nc, D] fp32 (updated copy
    returned), pos [Nc] int64 ascending, W a dict of fp32 weights (nn.Linear
    layout; norm weights taken as ones).  Returns (h_out, s, c, f, idx_attn, idx_ffn);
    ffn=False is the attention-only layer (steps a1..a7: c, f and idx_ffn None)."""
    Nc, D = h.shape
    d = W["w_q"].shape[0] // Hq
    G = Hq // Hkv
    xn = _bf16(_rmsnorm(h))
    kk = _bf16(_rope((xn @ W["w_k"].T).view(Nc, Hkv, d), pos))
    vv = _bf16((xn @ W["w_v"].T).view(Nc, Hkv, d))
    qp = _bf16(_rope((xn[Nc - P:] @ W["w_q"].T).view(P, Hq, d), pos[Nc - P:]))
    if salient_rows is not None and len(salient_rows):
        kk = _salience(kk, qp, salient_rows, salient_shift, Hkv)
    # PAP: per (head, probe) causal softmax over every key, summed (Fig. 2(a))
    hidden = pos[None, :] > pos[Nc - P:, None]
    s = torch.zeros(Nc, dtype=torch.float64)
    for hh in range(Hq):
        logits = (qp[:, hh, :] @ kk[:, hh // G, :].T) / math.sqrt(d)
        logits.masked_fill_(hidden, float("-inf"))
        s += torch.softmax(logits, dim=1).sum(0).double()
    s = s.float()
    idx_a = _topk(s, k, P)
    q_sel = _bf16(_rope((xn[idx_a] @ W["w_q"].T).view(k, Hq, d), pos[idx_a]))
    o_sel = _bf16(_attention(q_sel, pos[idx_a], kk, vv, pos, G))
    h1 = h.clone()
    h1[idx_a] += o_sel.view(k, Hq * d) @ W["w_o"].T
    if not ffn:
        return h1, s, None, None, idx_a, None
    # LTP score of the FFN input (Fig. 2(b)): || (x A^T) B^T ||_2
    x2 = _bf16(_rmsnorm(h1))
    c = (_bf16(x2 @ W["ltp_a"].T) @ W["ltp_b"].T).norm(dim=1)
    if fuse == FUSE_MULTIPLY:
        f = s * c
    elif fuse == FUSE_MAXNORM_ADD:
        f = w_a * (s / s.max()) + w_b * (c / c.max())
    else:
        f = s.clone()
    idx_f = _topk(f, k, P)
    x = x2[idx_f]
    act = _bf16(torch.nn.functional.silu(x @ W["w_gate"].T) * (x @ W["w_up"].T))
    h2 = h1.clone()
    h2[idx_f] += act @ W["w_down"].T
    return h2, s, c, f, idx_a, idx_f
