"""KV-cache accounting of a token-skipping prefill (host-side helper).

A skipping layer computes K and V only for the tokens active in it, so that
is all it can cache (the reading of Table 5 and Fig. A(c) of "Probe and Skip:
Self-Predictive Token Skipping for Efficient Long-Context LLM Inference").
With multi-stage delayed pruning (Table B), layers before the first skipping
layer cache every token, each layer of stage s caches the stage's active
budget, and the layers after the last stage cache the tokens that survived.

``cached_tokens_per_layer`` gives the per-layer counts of a schedule and
``kv_cache_bytes`` turns any such list into bytes; the LLaMA-3.1-8B-Instruct
schedule of Table B is ``LLAMA31_8B``.  Table 5 counts K and V at 32 heads of
128 values in 2 bytes (16 KiB per token and layer).
"""

from __future__ import annotations

from dataclasses import dataclass

__all__ = ["SkipSchedule", "LLAMA31_8B", "cached_tokens_per_layer", "kv_cache_bytes", "kv_cache_gib"]


@dataclass(frozen=True)
class SkipSchedule:
    layers: int
    first_skip: int              # index of the first skipping layer
    stage_ends: tuple            # last layer index of each stage (ascending)
    budgets: tuple               # active tokens of each stage
    after_last: int              # tokens kept after the last stage
    kv_heads: int = 32           # heads counted per K and per V
    head_dim: int = 128
    bytes_per_value: int = 2


# Table B, LLaMA-3.1-8B-Instruct: 32 layers, skipping from layer 10, stages
# ending at layers 13/18/23/28 with budgets 9K/7K/4K/2K, 1K tokens after.
LLAMA31_8B = SkipSchedule(layers=32, first_skip=10, stage_ends=(13, 18, 23, 28),
                          budgets=(9 * 1024, 7 * 1024, 4 * 1024, 2 * 1024), after_last=1024)


def cached_tokens_per_layer(n_tokens: int, sched: SkipSchedule = LLAMA31_8B, skipping: bool = True) -> list:
    """Tokens whose K and V layer l holds after a prefill of n_tokens."""
    n = int(n_tokens)
    if not skipping:
        return [n] * sched.layers
    if len(sched.stage_ends) != len(sched.budgets):
        raise ValueError("one budget per stage")
    out = []
    for layer in range(sched.layers):
        if layer < sched.first_skip:
            out.append(n)
            continue
        stage = next((s for s, end in enumerate(sched.stage_ends) if layer <= end), None)
        out.append(min(n, sched.budgets[stage] if stage is not None else sched.after_last))
    return out


def kv_cache_bytes(per_layer_tokens, sched: SkipSchedule = LLAMA31_8B) -> int:
    """Bytes of K and V for the given cached-token count of every layer."""
    per_token = 2 * sched.kv_heads * sched.head_dim * sched.bytes_per_value
    return sum(int(t) for t in per_layer_tokens) * per_token


def kv_cache_gib(n_tokens: int, sched: SkipSchedule = LLAMA31_8B, skipping: bool = True) -> float:
    """KV cache of one sequence in GiB (the "GB" of Table 5)."""
    return kv_cache_bytes(cached_tokens_per_layer(n_tokens, sched, skipping), sched) / 2 ** 30
