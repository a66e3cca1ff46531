"""Seeded synthetic workloads for the SPTS prefill path.

This module only draws random inputs (and the positions of the synthetic
"salient" keys); it holds none of the method's arithmetic.  The tests, the
bench and the smoke check take their inputs from here and hand the same
arrays to the CUDA library and to the CPU oracle.

The real workloads of the method -- LongBench prompts through a trained
LLaMA-3.1-8B-Instruct -- are not available offline, so these stand in for
them: a Llama-3.1-8B-shaped layer (32 query / 8 KV heads of 128, hidden 4096,
SwiGLU 14336) with random N(0, 0.02) weights, N(0, 1) hidden states, and a
small fraction of keys made salient.  Every draw is from a CPU
``torch.Generator`` so the values are identical on every machine.
"""

from __future__ import annotations

from dataclasses import dataclass, replace
from fractions import Fraction

import torch

__all__ = ["Workload", "WORKLOADS", "keep_rows", "salient_rows", "make_qkv_f32",
           "make_hidden", "make_layer_weights", "FUSE_NONE", "FUSE_MAXNORM_ADD", "FUSE_MULTIPLY",
           "FUSE_STD_ADD", "FUSE_SEQUENTIAL"]

FUSE_NONE, FUSE_MAXNORM_ADD, FUSE_MULTIPLY, FUSE_STD_ADD, FUSE_SEQUENTIAL = 0, 1, 2, 3, 4


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    Hq: int
    Hkv: int
    d: int
    P: int
    keep: str                 # keep ratio as an exact decimal string
    dtype: str = "bf16"       # "f32": Q/K/V given directly; "bf16": a full layer
    D: int = 0                # hidden size (Hq * d for the Llama shape)
    F: int = 0                # FFN hidden size (0: attention-only layer)
    r: int = 0                # LTP rank
    salient_frac: str = "0"
    salient_shift: float = 0.0
    fuse: int = FUSE_MAXNORM_ADD
    layers: int = 1
    ratios: tuple = ()
    seed: int = 1000
    ltp_dout: int = 0         # LTP proxy output channels (0: D)
    kv_active: bool = False   # reduced attention over the active rows' keys only
    ltp_top_m: int = 0        # LTP saliency = sum of the top m |y| (0: L2 norm)
    # per-layer skipping schedule (first_skip, stage_ends, budgets, after_last); () for none
    schedule: tuple = ()

    @property
    def k(self) -> int:
        return keep_rows(self.keep, self.N)


def keep_rows(ratio, n) -> int:
    """floor(ratio * n) in exact arithmetic."""
    r = Fraction(str(ratio))
    return (r.numerator * int(n)) // r.denominator


WORKLOADS = {
    # PAP + select + reduced attention on given fp32 Q/K/V (MHA).
    "tiny_f32": Workload("tiny_f32", N=512, Hq=4, Hkv=4, d=64, P=16, keep="0.25", dtype="f32",
                         salient_frac="0.02", salient_shift=3.0, seed=1001),
    # Llama-3.1-8B-shaped attention-only layer at 8K tokens.
    "attn_8k": Workload("attn_8k", N=8192, Hq=32, Hkv=8, d=128, P=64, keep="0.4", D=4096,
                        salient_frac="0.02", salient_shift=3.0, seed=1002),
    # Full SPTS layer (PAP + LTP) at 32K and 128K tokens.
    "layer_32k": Workload("layer_32k", N=32768, Hq=32, Hkv=8, d=128, P=64, keep="0.3", D=4096,
                          F=14336, r=256, salient_frac="0.02", salient_shift=3.0, seed=1003),
    "layer_128k": Workload("layer_128k", N=131072, Hq=32, Hkv=8, d=128, P=128, keep="0.2", D=4096,
                           F=14336, r=256, salient_frac="0.01", salient_shift=4.0, seed=1004),
    # MSDP: 8 layers in 4 stages of 2, candidate ratios 0.8/0.6/0.4/0.25.
    "msdp_32k": Workload("msdp_32k", N=32768, Hq=32, Hkv=8, d=128, P=64, keep="0.8", D=4096,
                         F=14336, r=256, layers=8, ratios=("0.8", "0.6", "0.4", "0.25"), seed=1005),
    # Small shapes for full element-by-element parity (ragged N, several tiles).
    "layer_small": Workload("layer_small", N=1000, Hq=8, Hkv=2, d=128, P=16, keep="0.3", D=1024,
                            F=1536, r=64, salient_frac="0.02", salient_shift=3.0, seed=1101),
    "msdp_small": Workload("msdp_small", N=600, Hq=8, Hkv=2, d=128, P=16, keep="0.8", D=1024,
                           F=1024, r=64, layers=8, ratios=("0.8", "0.6", "0.4", "0.25"), seed=1102),
}
# Variants of the layer workloads (the same inputs, one setting changed):
#   _kv    keys and values of the active rows only in the reduced attention;
#   _mul   the Multiply fusion f = s * c for the FFN selection;
#   _p1    a single probe token;
#   _dlow  the channel-reduced LTP proxy, D_low = 512 output channels, r = 192;
#   _rho   that proxy with top-rho saliency, rho = 0.2: the top 103 of 512 |y|;
#   _std   the Std-Add fusion; _seq the Sequential Select (pool 2k).
for _base in ("layer_32k", "layer_128k", "layer_small"):
    _w = WORKLOADS[_base]
    WORKLOADS[_base + "_kv"] = replace(_w, name=_base + "_kv", kv_active=True)
    WORKLOADS[_base + "_mul"] = replace(_w, name=_base + "_mul", fuse=FUSE_MULTIPLY)
    WORKLOADS[_base + "_p1"] = replace(_w, name=_base + "_p1", P=1)
    WORKLOADS[_base + "_dlow"] = replace(_w, name=_base + "_dlow", ltp_dout=512, r=192)
    WORKLOADS[_base + "_rho"] = replace(_w, name=_base + "_rho", ltp_dout=512, r=192, ltp_top_m=103)
    WORKLOADS[_base + "_std"] = replace(_w, name=_base + "_std", fuse=FUSE_STD_ADD)
    WORKLOADS[_base + "_seq"] = replace(_w, name=_base + "_seq", fuse=FUSE_SEQUENTIAL)
del _base, _w
# The 32-layer LLaMA-3.1-8B-shaped schedule of Table B (skipping in layers
# 10..28, stages ending at 13/18/23/28 with budgets 9K/7K/4K/2K, 1K tokens
# after) at Table 4's context lengths, with the pages' default settings: one
# probe token, the Multiply fusion, the (D_low 512, r 192) proxy with top-rho
# 0.2, and active-row keys in the skipping layers.  Random weights.
for _n in (8, 16, 24, 32):
    WORKLOADS[f"llama32_{_n}k"] = Workload(
        f"llama32_{_n}k", N=_n * 1024, Hq=32, Hkv=8, d=128, P=1, keep="1", D=4096, F=14336, r=192,
        fuse=FUSE_MULTIPLY, layers=32, seed=1200 + _n, ltp_dout=512, ltp_top_m=103, kv_active=True,
        schedule=(10, (13, 18, 23, 28), (9 * 1024, 7 * 1024, 4 * 1024, 2 * 1024), 1024))
del _n


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def salient_rows(n, p, frac, seed):
    """floor(frac * n) distinct rows drawn from [0, n - p), sorted."""
    count = keep_rows(frac, n)
    if count == 0:
        return torch.zeros(0, dtype=torch.int32)
    g = _gen(seed + 7)
    perm = torch.randperm(n - p, generator=g)[:count]
    return torch.sort(perm).values.to(torch.int32)


def make_qkv_f32(wl: Workload):
    """fp32 Q, K, V [N, H, d] ~ N(0, 1) with salient keys (the tiny MHA case).

    Salience: for each head, the keys at ``salient_rows`` get
    shift * unit(mean of that head's probe queries), the probes being the last
    P rows.  Returns (q, k, v, pos int32, salient rows).
    """
    g = _gen(wl.seed)
    q = torch.randn(wl.N, wl.Hq, wl.d, generator=g, dtype=torch.float32)
    k = torch.randn(wl.N, wl.Hkv, wl.d, generator=g, dtype=torch.float32)
    v = torch.randn(wl.N, wl.Hkv, wl.d, generator=g, dtype=torch.float32)
    rows = salient_rows(wl.N, wl.P, wl.salient_frac, wl.seed)
    if len(rows):
        G = wl.Hq // wl.Hkv
        for gidx in range(wl.Hkv):
            mean = q[wl.N - wl.P:, gidx * G:(gidx + 1) * G, :].reshape(-1, wl.d).double().mean(0)
            u = (mean / mean.norm()).float()
            k[rows.long(), gidx, :] += wl.salient_shift * u
    pos = torch.arange(wl.N, dtype=torch.int32)
    return q, k, v, pos, rows


def make_hidden(wl: Workload, n=None):
    """Residual-stream input h [n, D]: N(0, 1) values rounded to bf16, held in fp32."""
    n = wl.N if n is None else n
    g = _gen(wl.seed)
    return torch.randn(n, wl.D, generator=g, dtype=torch.float32).to(torch.bfloat16).float()


def make_layer_weights(wl: Workload, layer: int = 0, device="cpu"):
    """bf16 weights of one Llama-shaped layer, nn.Linear layout, ~N(0, 0.02).

    ``device`` draws them there (a different stream of values than on the
    CPU: used where only timing needs them).  Keys: w_q [Hq*d, D], w_k / w_v [Hkv*d, D], w_o [D, Hq*d]; when F > 0 also
    w_gate / w_up [F, D], w_down [D, F], ltp_a [r, D], ltp_b [D_low, r] (D_low =
    ltp_dout, else D).  Norm
    weights are ones.
    """
    g = torch.Generator(device=device)
    g.manual_seed(int(wl.seed * 1000 + 17 + 101 * layer))
    D, hd, kd = wl.D, wl.Hq * wl.d, wl.Hkv * wl.d

    def w(o, i):
        return (0.02 * torch.randn(o, i, generator=g, dtype=torch.float32, device=device)).to(torch.bfloat16)

    out = dict(w_q=w(hd, D), w_k=w(kd, D), w_v=w(kd, D), w_o=w(D, hd))
    if wl.F:
        out.update(w_gate=w(wl.F, D), w_up=w(wl.F, D), w_down=w(D, wl.F),
                   ltp_a=w(wl.r, D), ltp_b=w(wl.ltp_dout or D, wl.r))
    out["norm_attn"] = torch.ones(D, dtype=torch.bfloat16, device=device)
    out["norm_ffn"] = torch.ones(D, dtype=torch.bfloat16, device=device)
    return out


def with_overrides(wl: Workload, **kw) -> Workload:
    return replace(wl, **kw)
