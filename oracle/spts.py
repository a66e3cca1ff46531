"""fp64 CPU oracle of the SPTS prefill layer (test infrastructure only).

Source of every definition below: "Probe and Skip: Self-Predictive Token
Skipping for Efficient Long-Context LLM Inference" (Wu, Wang, Jin, Chen, Wang;
2026), abstract and the captions of Fig. 2 / Fig. 3 / Fig. A, with the
fusion names of Table D, the proxy criterion of Table 6 and the stage layout
of Table B.  The pages print no equations, so each step states the reading it
takes; the full list of readings is kept with the design notes.

Conventions (the reading of a Llama-3.1-8B-shaped layer):
  * rows are tokens; ``pos`` holds each row's original position (ascending);
  * weights use the nn.Linear layout [out, in], so y = x @ W.T;
  * GQA: query head h reads KV head h // (Hq // Hkv); scale = 1/sqrt(d);
  * causal masking is by original position: key j is visible to a query at
    position p when pos_j <= p;
  * RoPE is rotate-half (pairs i, i + d/2), theta = 500000, at original
    positions, no frequency scaling;
  * RMSNorm eps = 1e-5.

Precision: all arithmetic is fp64.  The bf16 layer stores some tensors in
bf16 between operations; the oracle rounds (round-to-nearest-even) exactly
those tensors and nothing else: every operand of a matrix product (normed
activations, projected Q/K/V, the attention output, the LTP intermediate,
the SwiGLU activation).  The residual stream stays unrounded.  Where a float
decides an integer (the fused score that top-k ranks), the decision is taken
in fp32 with the same operation order as the library, as the product does.

Parity status: every public function is pinned in
``tests/test_oracle_pins.py``; none is "parity unpinned".
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from .accounting import keep_count

__all__ = [
    "bf16_round", "rmsnorm", "rope", "probe_scores", "ltp_scores", "ltp_topm_scores", "fuse_scores",
    "select_topk", "reduced_attention", "attention_residual", "reduced_ffn",
    "stage_prune", "inject_salience", "LayerWeights", "LayerConfig", "layer_forward",
    "msdp_forward", "MsdpConfig", "FUSE_NONE", "FUSE_MAXNORM_ADD", "FUSE_MULTIPLY", "FUSE_STD_ADD",
    "FUSE_SEQUENTIAL", "select_sequential", "schedule_forward",
]

FUSE_NONE = 0
FUSE_MAXNORM_ADD = 1
FUSE_MULTIPLY = 2
FUSE_STD_ADD = 3
FUSE_SEQUENTIAL = 4    # layer setting: select_sequential


# --------------------------------------------------------------------------
# bf16 rounding (storage precision of the bf16 path)
# --------------------------------------------------------------------------
def bf16_round(x):
    """Round to the nearest bf16 value, ties to even, returned as float64.

    bf16 keeps 8 significant bits and fp32's exponent range.  Written from the
    definition: scale so that the kept bits are the integer part, round half
    to even (np.rint), scale back.  Below 2**-126 the quantum stays 2**-133
    (bf16 subnormals).  Magnitudes that round beyond the largest finite bf16
    become inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    finite = np.isfinite(x) & (x != 0)
    xf = x[finite]
    _, e = np.frexp(xf)                      # xf = m * 2**e, 0.5 <= |m| < 1
    q = np.maximum(e - 8, -133)              # exponent of the last kept bit
    r = np.ldexp(np.rint(np.ldexp(xf, -q)), q)
    r[np.abs(r) >= 2.0 ** 128] = np.copysign(np.inf, r[np.abs(r) >= 2.0 ** 128])
    out[finite] = r
    return out


# --------------------------------------------------------------------------
# Glue of the Llama-shaped layer
# --------------------------------------------------------------------------
def rmsnorm(x, w=None, eps=1e-5):
    """RMSNorm of each row: x / sqrt(mean(x**2) + eps) * w."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    if w is not None:
        y = y * np.asarray(w, dtype=np.float64)
    return y


def rope(x, pos, theta=500000.0):
    """Rotate-half rotary embedding of x [rows, H, d] at positions pos [rows].

    Pair (i, i + d/2) turns by angle pos * theta**(-2i/d).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    inv_freq = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / d)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]   # [rows, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# --------------------------------------------------------------------------
# Partial Attention Probing (Fig. 2(a); probe length: Table C)
# --------------------------------------------------------------------------
def probe_scores(q_probe, probe_pos, k, key_pos, scale=None):
    """Per-key importance from a few probe queries.

    Fig. 2(a): PAP pre-computes a small fraction of attention -- the rows of
    the probe queries (the last P candidates; Table C sweeps P) against every
    key -- and ranks keys by it.  Reading: each (head, probe) row is a causal
    softmax over keys, and the score of key j is the plain sum of its weights
    over all heads and probes.

    q_probe [P, Hq, d], probe_pos [P], k [Nc, Hkv, d], key_pos [Nc].
    Returns (s [Nc], group_scores [Hkv, Nc]); group g sums the heads that
    read KV head g.  Every row sums to 1, so sum(s) = P * Hq.
    """
    q_probe = np.asarray(q_probe, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    P, Hq, d = q_probe.shape
    Nc, Hkv, _ = k.shape
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    visible = np.asarray(key_pos)[None, :] <= np.asarray(probe_pos)[:, None]   # [P, Nc]
    group = np.zeros((Hkv, Nc), dtype=np.float64)
    for h in range(Hq):
        g = h // G
        logits = scale * (q_probe[:, h, :] @ k[:, g, :].T)                   # [P, Nc]
        logits = np.where(visible, logits, -np.inf)
        m = np.max(logits, axis=1, keepdims=True)
        e = np.where(visible, np.exp(logits - m), 0.0)
        a = e / np.sum(e, axis=1, keepdims=True)
        group[g] += a.sum(axis=0)
    return group.sum(axis=0), group


# --------------------------------------------------------------------------
# Low-rank Transformation Probing (Fig. 2(b), Table 6, Table A)
# --------------------------------------------------------------------------
def ltp_scores(x, A, B):
    """FFN-change score from the low-rank proxy: c_i = || (x_i A^T) B^T ||_2.

    Fig. 2(b): a low-rank proxy network probes each token's transformation.
    Reading: the proxy is the product X A^T B^T with A [r, D], B [Dout, r];
    the score is the L2 norm of the predicted change per row.  The rank-r
    intermediate is an operand of the second product, so it is rounded to
    bf16 as the bf16 path stores it; x is taken as given (already bf16).
    """
    x = np.asarray(x, dtype=np.float64)
    t = bf16_round(x @ np.asarray(A, dtype=np.float64).T)
    y = t @ np.asarray(B, dtype=np.float64).T
    return np.sqrt(np.sum(y * y, axis=1))


def ltp_topm_scores(x, A, B, m):
    """Top-rho channel saliency of the proxy output (Table E, with D_low of
    Table A).

    Reading: the proxy predicts the token's change y_i = (x_i A^T) B^T over
    the D_low output channels; the token's saliency is the sum of its m =
    ceil(rho * D_low) largest |y_ij|.  The intermediate is bf16-rounded as in
    ltp_scores.
    """
    x = np.asarray(x, dtype=np.float64)
    t = bf16_round(x @ np.asarray(A, dtype=np.float64).T)
    y = np.abs(t @ np.asarray(B, dtype=np.float64).T)
    m = int(m)
    if not 1 <= m <= y.shape[1]:
        raise ValueError("need 1 <= m <= D_low")
    return np.sort(y, axis=1)[:, y.shape[1] - m:].sum(axis=1)


# --------------------------------------------------------------------------
# Score fusion (Table D; criterion C*S of Table 6) -- decided in fp32
# --------------------------------------------------------------------------
def fuse_scores(s, c, mode, w_a=0.5, w_b=0.5):
    """Fused FFN-selection score, computed in fp32 as the library ranks it.

    Table D names the strategies; Table 6 writes the default as C * S.
      NONE:        f = s
      MULTIPLY:    f = s * c
      MAXNORM_ADD: f = w_a * (s / max s) + w_b * (c / max c), each max over
                   all candidates; a term whose max is 0 contributes 0.
      STD_ADD:     f = w_a * ((s - mean s) / std s) + w_b * ((c - mean c) / std c)
                   (reading of the name "Std-Add"): population mean and
                   standard deviation over all candidates, exact in fp64 and
                   rounded to fp32; a term whose std is 0 contributes 0.
    Each operation rounds to fp32 (no fused multiply-add), in this order.
    """
    s = np.asarray(s, dtype=np.float32)
    if mode == FUSE_NONE:
        return s.copy()
    c = np.asarray(c, dtype=np.float32)
    if mode == FUSE_MULTIPLY:
        return (s * c).astype(np.float32)
    if mode == FUSE_MAXNORM_ADD:
        ms = np.float32(np.max(s)) if s.size else np.float32(0)
        mc = np.float32(np.max(c)) if c.size else np.float32(0)
        ta = (np.float32(w_a) * (s / ms)).astype(np.float32) if ms > 0 else np.zeros_like(s)
        tb = (np.float32(w_b) * (c / mc)).astype(np.float32) if mc > 0 else np.zeros_like(c)
        return (ta + tb).astype(np.float32)
    if mode == FUSE_STD_ADD:
        def standardised(x, w):
            x64 = x.astype(np.float64)
            mu = math.fsum(x64) / len(x64)
            sd = math.sqrt(math.fsum((x64 - mu) ** 2) / len(x64))
            mu32, sd32 = np.float32(mu), np.float32(sd)
            if not sd32 > 0:
                return np.zeros_like(x)
            return (np.float32(w) * ((x - mu32).astype(np.float32) / sd32).astype(np.float32)).astype(np.float32)
        return (standardised(s, w_a) + standardised(c, w_b)).astype(np.float32)
    raise ValueError(f"unknown fusion mode {mode}")


# --------------------------------------------------------------------------
# Token selection (Fig. 2(a)/(b): the informative tokens)
# --------------------------------------------------------------------------
def select_topk(f, k, force_tail):
    """Indices of the k informative tokens, ascending.

    Reading: the last ``force_tail`` candidates (the probe rows) are always
    kept (Fig. 3(b) singles out the last token); the other k - force_tail are
    the largest scores among the rest, equal scores going to the lower index.
    -0 counts as +0.  Returns (idx int64 [k], tau) where tau is the score of
    the last non-forced pick (nan when every pick is forced).
    """
    f = np.asarray(f, dtype=np.float32)
    Nc = f.shape[0]
    if not (0 <= force_tail <= k <= Nc):
        raise ValueError("need 0 <= force_tail <= k <= Nc")
    if np.any(~np.isfinite(f)):
        raise ValueError("scores must be finite")
    f = np.where(f == 0, np.float32(0), f)
    n_free = Nc - force_tail
    k_free = k - force_tail
    order = np.argsort(-f[:n_free].astype(np.float64), kind="stable")
    chosen = np.sort(order[:k_free])
    idx = np.concatenate([chosen, np.arange(n_free, Nc)]).astype(np.int64)
    tau = float(f[order[k_free - 1]]) if k_free > 0 else float("nan")
    return idx, tau


def select_sequential(s, c, k_pool, k, force_tail):
    """Sequential Select of Table D (reading: the pages only name it).

    The attention-based score narrows the candidates first and the
    transformation score decides second: the pool is select_topk(s, k_pool),
    then the k of the pool with the largest c under the same rules (the
    forced tail stays, ties go to the lower index).  Returns (indices
    ascending, threshold of the second selection).
    """
    pool, _ = select_topk(np.asarray(s, dtype=np.float32), k_pool, force_tail)
    local, tau = select_topk(np.asarray(c, dtype=np.float32)[pool], k, force_tail)
    return pool[local], tau


# --------------------------------------------------------------------------
# Reduced attention (Fig. 2(a): the informative tokens attend)
# --------------------------------------------------------------------------
def reduced_attention(q_sel, q_pos, k, v, key_pos, scale=None):
    """Exact causal GQA attention of the selected queries against all keys.

    Reduced attention runs only for the selected rows; for them it is plain
    softmax attention over every candidate key j with pos_j <= pos_i.
    q_sel [m, Hq, d], q_pos [m], k/v [Nc, Hkv, d], key_pos [Nc] -> [m, Hq, d].
    """
    q_sel = np.asarray(q_sel, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    m, Hq, d = q_sel.shape
    Nc, Hkv, _ = k.shape
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    visible = np.asarray(key_pos)[None, :] <= np.asarray(q_pos)[:, None]     # [m, Nc]
    out = np.zeros((m, Hq, d), dtype=np.float64)
    for h in range(Hq):
        g = h // G
        logits = scale * (q_sel[:, h, :] @ k[:, g, :].T)
        logits = np.where(visible, logits, -np.inf)
        mx = np.max(logits, axis=1, keepdims=True)
        e = np.where(visible, np.exp(logits - mx), 0.0)
        out[:, h, :] = (e @ v[:, g, :]) / np.sum(e, axis=1, keepdims=True)
    return out


def attention_residual(h, idx, o_sel, w_o):
    """h' = h; h'[idx] += O_sel W_o^T (skipped rows pass through unchanged)."""
    h = np.array(h, dtype=np.float64, copy=True)
    o = bf16_round(np.asarray(o_sel, dtype=np.float64).reshape(len(idx), -1))
    h[np.asarray(idx)] += o @ np.asarray(w_o, dtype=np.float64).T
    return h


# --------------------------------------------------------------------------
# Reduced FFN (Fig. 2(b): reduced feed-forward on the selected rows)
# --------------------------------------------------------------------------
def _silu(z):
    return z / (1.0 + np.exp(-z))


def reduced_ffn(h, idx, norm_w, eps, w_gate, w_up, w_down):
    """h'' = h; for i in idx: h''_i += W_down (silu(W_gate x_i) * (W_up x_i)).

    x_i = RMSNorm(h_i) * norm_w.  x and the SwiGLU activation are the two
    product operands the bf16 path stores, so both are rounded to bf16.
    """
    h = np.array(h, dtype=np.float64, copy=True)
    idx = np.asarray(idx)
    x = bf16_round(rmsnorm(h[idx], norm_w, eps))
    g = x @ np.asarray(w_gate, dtype=np.float64).T
    u = x @ np.asarray(w_up, dtype=np.float64).T
    act = bf16_round(_silu(g) * u)
    h[idx] += act @ np.asarray(w_down, dtype=np.float64).T
    return h


# --------------------------------------------------------------------------
# Multi-Stage Delayed Pruning (Fig. 2(c), Fig. A, Table B)
# --------------------------------------------------------------------------
def stage_prune(scores, k_keep, force_tail, h, pos):
    """Prune the candidate set at a stage boundary.

    Fig. 2(c): candidates stay fixed inside a stage and shrink at its end.
    Reading: keep the top k_keep candidates by the stage's last fused score
    (tail forced, ties to the lower index), in ascending order, and compact
    the hidden rows and their positions.  Returns (h_out, pos_out, kept_idx).
    """
    kept, _ = select_topk(scores, k_keep, force_tail)
    return np.asarray(h)[kept].copy(), np.asarray(pos)[kept].copy(), kept


# --------------------------------------------------------------------------
# The composed layer and the MSDP pipeline
# --------------------------------------------------------------------------
@dataclass
class LayerWeights:
    w_q: np.ndarray            # [Hq*d, D]
    w_k: np.ndarray            # [Hkv*d, D]
    w_v: np.ndarray            # [Hkv*d, D]
    w_o: np.ndarray            # [D, Hq*d]
    w_gate: np.ndarray | None = None   # [F, D]
    w_up: np.ndarray | None = None     # [F, D]
    w_down: np.ndarray | None = None   # [D, F]
    ltp_a: np.ndarray | None = None    # [r, D]
    ltp_b: np.ndarray | None = None    # [Dout, r]
    norm_attn: np.ndarray | None = None  # [D] (None = ones)
    norm_ffn: np.ndarray | None = None   # [D] (None = ones)


@dataclass
class LayerConfig:
    Hq: int
    Hkv: int
    d: int
    P: int
    k: int                     # active rows per selection
    fuse: int = FUSE_MAXNORM_ADD
    w_a: float = 0.5
    w_b: float = 0.5
    ffn: bool = True           # False: attention-only layer (a1..a7)
    eps: float = 1e-5
    theta: float = 500000.0
    salient_rows: np.ndarray | None = None   # workload recipe, not SPTS
    salient_shift: float = 0.0
    kv_active: bool = False    # reduced attention over the active rows' keys only
    ltp_top_m: int = 0         # > 0: LTP saliency = sum of the top m |y| (Table E); 0: L2 norm
    seq_pool: int = 0          # FUSE_SEQUENTIAL: pool size (0: min(Nc, 2k))


def inject_salience(kk, q_probe, rows, shift, Hkv):
    """Synthetic-workload step (not part of SPTS): make some keys salient.

    Adds shift * unit(mean of the group's probe queries) to K[rows, g] for
    every KV group g, then stores K back in bf16.
    """
    kk = np.array(kk, dtype=np.float64, copy=True)
    P, Hq, d = q_probe.shape
    G = Hq // Hkv
    for g in range(Hkv):
        mean = q_probe[:, g * G:(g + 1) * G, :].reshape(-1, d).mean(axis=0)
        u = mean / np.linalg.norm(mean)
        kk[rows, g, :] = bf16_round(kk[rows, g, :] + shift * u)
    return kk


def layer_forward(h, pos, W: LayerWeights, cfg: LayerConfig, trace: dict | None = None):
    """One SPTS layer (the order of Fig. 2: PAP -> reduced MHA -> LTP -> reduced FFN).

    h [Nc, D] residual stream (fp64, unrounded), pos [Nc] ascending.
    Returns (h_out, fused score of the FFN selection (fp32)).  When ``trace``
    is a dict it receives every intermediate, for sampled comparisons.
    """
    h = np.asarray(h, dtype=np.float64)
    pos = np.asarray(pos)
    Nc, D = h.shape
    Hq, Hkv, d, P, k = cfg.Hq, cfg.Hkv, cfg.d, cfg.P, cfg.k
    t = trace if trace is not None else {}

    xn = bf16_round(rmsnorm(h, W.norm_attn, cfg.eps))
    kk = bf16_round(rope((xn @ W.w_k.T).reshape(Nc, Hkv, d), pos, cfg.theta))
    vv = bf16_round((xn @ W.w_v.T).reshape(Nc, Hkv, d))
    pp = pos[Nc - P:]
    q_probe = bf16_round(rope((xn[Nc - P:] @ W.w_q.T).reshape(P, Hq, d), pp, cfg.theta))
    if cfg.salient_rows is not None and len(cfg.salient_rows):
        kk = inject_salience(kk, q_probe, np.asarray(cfg.salient_rows), cfg.salient_shift, Hkv)
    s, group = probe_scores(q_probe, pp, kk, pos)
    s32 = s.astype(np.float32)
    idx_a, tau_a = select_topk(s32, k, P)
    q_sel = bf16_round(rope((xn[idx_a] @ W.w_q.T).reshape(k, Hq, d), pos[idx_a], cfg.theta))
    if cfg.kv_active:
        # the KV-cache reading behind Table 5 and Fig. A(c): a skipping layer
        # keeps K and V of its active tokens only, so the selected queries
        # attend, causally by original position, to the selected keys
        o_sel = bf16_round(reduced_attention(q_sel, pos[idx_a], kk[idx_a], vv[idx_a], pos[idx_a]))
    else:
        o_sel = bf16_round(reduced_attention(q_sel, pos[idx_a], kk, vv, pos))
    h1 = attention_residual(h, idx_a, o_sel, W.w_o)
    t.update(xn=xn, k=kk, v=vv, q_probe=q_probe, s=s, group=group, idx_attn=idx_a,
             tau_attn=tau_a, q_sel=q_sel, o_sel=o_sel, h_attn=h1)
    if not cfg.ffn:
        return h1, s32
    x_ffn = bf16_round(rmsnorm(h1, W.norm_ffn, cfg.eps))
    c = (ltp_topm_scores(x_ffn, W.ltp_a, W.ltp_b, cfg.ltp_top_m) if cfg.ltp_top_m > 0
         else ltp_scores(x_ffn, W.ltp_a, W.ltp_b))
    if cfg.fuse == FUSE_SEQUENTIAL:
        pool = cfg.seq_pool if cfg.seq_pool > 0 else min(Nc, 2 * k)
        f = c.astype(np.float32)
        idx_f, tau_f = select_sequential(s32, f, pool, k, P)
    else:
        f = fuse_scores(s32, c.astype(np.float32), cfg.fuse, cfg.w_a, cfg.w_b)
        idx_f, tau_f = select_topk(f, k, P)
    h2 = reduced_ffn(h1, idx_f, W.norm_ffn, cfg.eps, W.w_gate, W.w_up, W.w_down)
    t.update(x_ffn=x_ffn, c=c, f=f, idx_ffn=idx_f, tau_ffn=tau_f, h_out=h2)
    return h2, f


@dataclass
class MsdpConfig:
    layer: LayerConfig
    ratios: tuple = (0.8, 0.6, 0.4, 0.25)
    layers_per_stage: int = 2


def msdp_forward(h, pos, layers, mcfg: MsdpConfig, trace: list | None = None):
    """Multi-Stage Delayed Pruning over len(ratios) stages.

    Reading of Fig. 2(c) / Fig. A / Table B: stage s holds a candidate set
    C_s (C_1 = every token).  Each layer of the stage picks k_s = floor(r_s N)
    active rows afresh from C_s for both reduced attention and reduced FFN;
    rows of C_s that a layer skips pass through on the residual.  At the end
    of the stage C_{s+1} = top-k_s of C_s by the fused score of the stage's
    last layer (tail kept), so pruning is delayed to the stage boundary.

    Returns (h_final [k_last, D], pos_final, pruned) where ``pruned`` lists,
    per stage, (positions, last hidden rows) of the rows that left.
    """
    h = np.asarray(h, dtype=np.float64)
    pos = np.asarray(pos)
    N = h.shape[0]
    li = 0
    pruned = []
    for r in mcfg.ratios:
        k_s = keep_count(r, N)
        f = None
        for _ in range(mcfg.layers_per_stage):
            cfg = LayerConfig(**{**mcfg.layer.__dict__, "k": k_s})
            tr = {} if trace is not None else None
            h, f = layer_forward(h, pos, layers[li], cfg, tr)
            if trace is not None:
                trace.append(tr)
            li += 1
        keep_mask = np.zeros(h.shape[0], dtype=bool)
        h_new, pos_new, kept = stage_prune(f, k_s, mcfg.layer.P, h, pos)
        keep_mask[kept] = True
        pruned.append((pos[~keep_mask].copy(), h[~keep_mask].copy()))
        h, pos = h_new, pos_new
    return h, pos, pruned


def schedule_forward(h, pos, layers, cfg: LayerConfig, first_skip, stage_ends, budgets, after_last,
                     trace: list | None = None):
    """A per-layer skipping schedule of Table B (reading).

    Layers before ``first_skip`` are full layers (every token active).
    Stage s runs the layers up to ``stage_ends[s]``; each selects
    k = min(budgets[s], |C_s|) active rows from the stage's candidates C_s.
    At a stage end the candidates are pruned to the top budgets[s] by that
    layer's fused score (after the last stage to the top ``after_last``),
    the probe tail kept; the layers after the last stage are full layers over
    the survivors (Fig. A(c): skipped tokens are computed again later, pruned
    ones are gone).  Returns (h of the survivors, their positions); ``trace``
    receives per layer its k, its candidates' positions and the positions of
    its attention set.
    """
    h = np.asarray(h, dtype=np.float64)
    pos = np.asarray(pos)
    stage = 0
    for l, W in enumerate(layers):
        Nc = h.shape[0]
        skip = l >= first_skip and stage < len(stage_ends) and l <= stage_ends[stage]
        k = min(budgets[stage], Nc) if skip else Nc
        c = LayerConfig(**{**cfg.__dict__, "k": k, "salient_rows": None})
        tr = {}
        h, f = layer_forward(h, pos, W, c, tr)
        if trace is not None:
            trace.append(dict(layer=l, k=k, skip=skip, cand=pos.copy(), sel_pos=pos[tr["idx_attn"]], f=f))
        if skip and l == stage_ends[stage]:
            k_next = min(budgets[stage] if stage + 1 < len(stage_ends) else after_last, Nc)
            kept, _ = select_topk(f, k_next, cfg.P)
            h, pos = h[kept], pos[kept]
            stage += 1
    return h, pos
