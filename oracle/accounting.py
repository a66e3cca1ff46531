"""Closed-form cost accounting of SPTS (test infrastructure only).

Two tables of "Probe and Skip: Self-Predictive Token Skipping for Efficient
Long-Context LLM Inference" print numbers that follow from the method's
shapes alone, with no trained weights:

* Table A -- per-token, per-projection cost of the LTP proxy for output width
  D_low and rank r on a 4096-wide model;
* Table 5 -- KV-cache size of LLaMA-3.1-8B at 8K..32K tokens with and without
  PAP, under the skipping schedule of Table B.

Both are reproduced here and pinned against the printed values in
``tests/golden/``.
"""

from __future__ import annotations

from fractions import Fraction

__all__ = ["keep_count", "ltp_proxy_macs", "kv_cache_gib", "LLAMA31_8B_SCHEDULE"]


def keep_count(ratio, n):
    """floor(ratio * n) in exact arithmetic (ratio given as str/float/Fraction)."""
    r = Fraction(str(ratio)) if not isinstance(ratio, Fraction) else ratio
    return (r.numerator * int(n)) // r.denominator


def ltp_proxy_macs(d_model, d_low, r):
    """Multiply-accumulates per token of one proxy projection (Table A).

    With a rank-r decomposition the proxy maps d_model -> r -> d_low, costing
    r * (d_model + d_low); without one ("/" in Table A, r=None) it is a dense
    d_model x d_low map.  Table A calls these counts FLOPs.
    """
    if r is None:
        return d_model * d_low
    return r * (d_model + d_low)


# Table B, LLaMA-3.1-8B-Instruct row: 32 layers, tokens skipped in layers
# 10..28, stages ending at layers 13/18/23/28 with active budgets
# 9K/7K/4K/2K, and 1K tokens left after the last stage (K = 1024).
LLAMA31_8B_SCHEDULE = dict(
    layers=32, first_skip=10, stage_ends=(13, 18, 23, 28),
    budgets=(9 * 1024, 7 * 1024, 4 * 1024, 2 * 1024), after_last=1024,
    kv_heads_counted=32, head_dim=128, bytes_per_value=2,
)


def kv_cache_gib(n_tokens, schedule=LLAMA31_8B_SCHEDULE, with_pap=True):
    """KV-cache size in GiB for one sequence (Table 5 reading).

    Reading: a skipping layer caches only the tokens active in it (Fig. A(c)).
    Layers before the first skipping layer cache every token; layers of stage
    s cache min(budget_s, n); layers after the last stage cache the tokens
    that survived it.  Table 5's figures match when K and V are counted at 32
    heads of 128 values in 2 bytes, i.e. 16 KiB per token per layer.
    """
    per_token = 2 * schedule["kv_heads_counted"] * schedule["head_dim"] * schedule["bytes_per_value"]
    L = schedule["layers"]
    if not with_pap:
        return L * n_tokens * per_token / 2 ** 30
    total = schedule["first_skip"] * n_tokens
    start = schedule["first_skip"]
    for end, budget in zip(schedule["stage_ends"], schedule["budgets"]):
        total += (end - start + 1) * min(budget, n_tokens)
        start = end + 1
    total += (L - start) * min(schedule["after_last"], n_tokens)
    return total * per_token / 2 ** 30
