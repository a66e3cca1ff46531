"""The oracle's pins must catch plausible mistakes.

Each case swaps one oracle function for a deliberately broken version (a
flipped sign, a missing term, a wrong axis or index, a transposed operand, a
tie broken the wrong way), on the CPU, and runs the pins of
``test_oracle_pins`` that cover that function: at least one must fail.  A
mutant no pin catches is a gap in the pins.
"""

import math

import numpy as np
import pytest

import oracle as O
import oracle.spts as OS
import tests.test_oracle_pins as PINS

_ORIG = {n: getattr(OS, n) for n in ("rmsnorm", "rope", "probe_scores", "ltp_scores", "ltp_topm_scores",
                                     "fuse_scores", "select_topk", "select_sequential", "reduced_attention",
                                     "attention_residual", "reduced_ffn", "inject_salience", "stage_prune")}


# ---------------------------------------------------------------- mutants
def _rmsnorm_wrong_axis(x, w=None, eps=1e-5):
    x = np.asarray(x, dtype=np.float64)
    y = x / np.sqrt(np.mean(x * x, axis=0, keepdims=True) + eps)
    return y if w is None else y * np.asarray(w, dtype=np.float64)


def _rmsnorm_eps_outside_root(x, w=None, eps=1e-5):
    x = np.asarray(x, dtype=np.float64)
    y = x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps)
    return y if w is None else y * np.asarray(w, dtype=np.float64)


def _rmsnorm_drops_weight(x, w=None, eps=1e-5):
    return _ORIG["rmsnorm"](x, None, eps)


def _rope_backwards(x, pos, theta=500000.0):
    return _ORIG["rope"](x, -np.asarray(pos), theta)


def _rope_rotation(x, pos, theta, inv_freq, interleaved):
    x = np.asarray(x, dtype=np.float64)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    if interleaved:
        x1, x2 = x[..., 0::2], x[..., 1::2]
        out = np.empty_like(x)
        out[..., 0::2], out[..., 1::2] = x1 * c - x2 * s, x2 * c + x1 * s
        return out
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def _rope_half_exponent(x, pos, theta=500000.0):   # theta**(-i/d) instead of theta**(-2i/d)
    d = np.asarray(x).shape[-1]
    return _rope_rotation(x, pos, theta, theta ** (-np.arange(d // 2) / d), False)


def _rope_interleaved_pairs(x, pos, theta=500000.0):   # pairs (2i, 2i+1) instead of (i, i + d/2)
    d = np.asarray(x).shape[-1]
    return _rope_rotation(x, pos, theta, theta ** (-np.arange(0, d, 2) / d), True)


def _probe_unmasked(q_probe, probe_pos, k, key_pos, scale=None):
    return _ORIG["probe_scores"](q_probe, np.full(len(probe_pos), np.max(key_pos)), k, key_pos, scale)


def _probe_unscaled(q_probe, probe_pos, k, key_pos, scale=None):
    return _ORIG["probe_scores"](q_probe, probe_pos, k, key_pos, 1.0)


def _probe_mask_after_softmax(q_probe, probe_pos, k, key_pos, scale=None):
    # each row normalised over every key, the future keys zeroed afterwards
    q_probe, k = np.asarray(q_probe, dtype=np.float64), np.asarray(k, dtype=np.float64)
    P, Hq, d = q_probe.shape
    Nc, Hkv, _ = k.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    visible = np.asarray(key_pos)[None, :] <= np.asarray(probe_pos)[:, None]
    group = np.zeros((Hkv, Nc))
    for h in range(Hq):
        g = h // (Hq // Hkv)
        logits = scale * (q_probe[:, h, :] @ k[:, g, :].T)
        e = np.exp(logits - logits.max(axis=1, keepdims=True))
        group[g] += np.where(visible, e / e.sum(axis=1, keepdims=True), 0.0).sum(axis=0)
    return group.sum(axis=0), group


def _ltp_squared(x, A, B):
    return _ORIG["ltp_scores"](x, A, B) ** 2


def _topm_one_short(x, A, B, m):
    return _ORIG["ltp_topm_scores"](x, A, B, max(1, int(m) - 1))


def _fuse_weights_swapped(s, c, mode, w_a=0.5, w_b=0.5):
    return _ORIG["fuse_scores"](s, c, mode, w_b, w_a)


def _fuse_maxnorm_weights_swapped(s, c, mode, w_a=0.5, w_b=0.5):
    return _ORIG["fuse_scores"](s, c, mode, *((w_b, w_a) if mode == O.FUSE_MAXNORM_ADD else (w_a, w_b)))


def _fuse_c_not_normalised(s, c, mode, w_a=0.5, w_b=0.5):
    if mode != O.FUSE_MAXNORM_ADD:
        return _ORIG["fuse_scores"](s, c, mode, w_a, w_b)
    s = np.asarray(s, dtype=np.float32)
    c = np.asarray(c, dtype=np.float32)
    ms = np.float32(np.max(s))
    ta = (np.float32(w_a) * (s / ms)).astype(np.float32) if ms > 0 else np.zeros_like(s)
    return (ta + np.float32(w_b) * c).astype(np.float32)


def _select_ties_high(f, k, force_tail):
    f = np.asarray(f, dtype=np.float32)
    Nc = len(f)
    if not (0 <= force_tail <= k <= Nc) or np.any(~np.isfinite(f)):
        raise ValueError("bad selection arguments")
    n_free, k_free = Nc - force_tail, k - force_tail
    order = np.lexsort((-np.arange(n_free), -f[:n_free].astype(np.float64)))   # ties to the higher index
    idx = np.concatenate([np.sort(order[:k_free]), np.arange(n_free, Nc)]).astype(np.int64)
    return idx, float(f[order[k_free - 1]]) if k_free > 0 else float("nan")


def _select_tail_not_forced(f, k, force_tail):
    idx, tau = _ORIG["select_topk"](f, k, 0)
    return idx, tau


def _attention_strictly_causal(q_sel, q_pos, k, v, key_pos, scale=None):
    return _ORIG["reduced_attention"](q_sel, np.asarray(q_pos) - 1, k, v, key_pos, scale)


def _attention_heads_modulo(q_sel, q_pos, k, v, key_pos, scale=None):   # GQA group h % Hkv
    q_sel, k, v = (np.asarray(a, dtype=np.float64) for a in (q_sel, k, v))
    m, Hq, d = q_sel.shape
    Hkv = k.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    visible = np.asarray(key_pos)[None, :] <= np.asarray(q_pos)[:, None]
    out = np.zeros((m, Hq, d))
    for h in range(Hq):
        g = h % Hkv
        logits = np.where(visible, scale * (q_sel[:, h, :] @ k[:, g, :].T), -np.inf)
        e = np.where(visible, np.exp(logits - logits.max(axis=1, keepdims=True)), 0.0)
        out[:, h, :] = (e @ v[:, g, :]) / e.sum(axis=1, keepdims=True)
    return out


def _residual_untransposed(h, idx, o_sel, w_o):
    h = np.array(h, dtype=np.float64, copy=True)
    o = O.bf16_round(np.asarray(o_sel, dtype=np.float64).reshape(len(idx), -1))
    h[np.asarray(idx)] += o @ np.asarray(w_o, dtype=np.float64)
    return h


def _ffn(h, idx, norm_w, eps, w_gate, w_up, w_down, act_fn, normalise):
    h = np.array(h, dtype=np.float64, copy=True)
    idx = np.asarray(idx)
    x = O.bf16_round(_ORIG["rmsnorm"](h[idx], norm_w, eps) if normalise else h[idx])
    g, u = x @ np.asarray(w_gate).T, x @ np.asarray(w_up).T
    h[idx] += O.bf16_round(act_fn(g) * u) @ np.asarray(w_down).T
    return h


def _ffn_relu(h, idx, norm_w, eps, w_gate, w_up, w_down):
    return _ffn(h, idx, norm_w, eps, w_gate, w_up, w_down, lambda z: np.maximum(z, 0.0), True)


def _ffn_unnormalised(h, idx, norm_w, eps, w_gate, w_up, w_down):
    return _ffn(h, idx, norm_w, eps, w_gate, w_up, w_down, lambda z: z / (1.0 + np.exp(-z)), False)


def _salience_not_unit(kk, q_probe, rows, shift, Hkv):
    kk = np.array(kk, dtype=np.float64, copy=True)
    P, Hq, d = q_probe.shape
    G = Hq // Hkv
    for g in range(Hkv):
        mean = q_probe[:, g * G:(g + 1) * G, :].reshape(-1, d).mean(axis=0)
        kk[rows, g, :] = O.bf16_round(kk[rows, g, :] + shift * mean)
    return kk


def _sequential_scores_swapped(s, c, k_pool, k, force_tail):   # pool by c, decided by s
    return _ORIG["select_sequential"](c, s, k_pool, k, force_tail)


def _sequential_pool_local(s, c, k_pool, k, force_tail):   # indices into the pool, not the candidates
    pool, _ = _ORIG["select_topk"](np.asarray(s, dtype=np.float32), k_pool, force_tail)
    return _ORIG["select_topk"](np.asarray(c, dtype=np.float32)[pool], k, force_tail)


def _stage_prune_lowest(scores, k_keep, force_tail, h, pos):
    return _ORIG["stage_prune"](-np.asarray(scores, dtype=np.float32), k_keep, force_tail, h, pos)


def _source_with(fn, old, new):
    """An oracle function with one line of its source changed."""
    import inspect
    import textwrap
    src = textwrap.dedent(inspect.getsource(fn))
    assert src.count(old) == 1, old
    ns = dict(vars(OS))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)  # noqa: S102
    return ns[fn.__name__]


_ORIG_LAYER = OS.layer_forward
_ORIG_MSDP = OS.msdp_forward
_ORIG_SCHEDULE = OS.schedule_forward


def _layer_with(old, new):
    return _source_with(_ORIG_LAYER, old, new)
_LAYER_PINS = ["test_layer_keep_all_equals_dense_layer", "test_layer_skipped_rows_pass_through",
               ("test_layer_selection_wiring", (0.0, 1.0)), ("test_layer_selection_wiring", (1.0, 0.0))]


_ORIG_PROBE = OS.probe_scores
_ORIG_BF16 = OS.bf16_round
_ORIG_TOPM = OS.ltp_topm_scores
_ORIG_FFN = OS.reduced_ffn
_ORIG_RESIDUAL = OS.attention_residual
_ORIG_SALIENCE = OS.inject_salience

# name -> (oracle function, mutant, pins that cover it)
MUTANTS = {
    "rmsnorm over the wrong axis": ("rmsnorm", _rmsnorm_wrong_axis, ["test_rmsnorm_matches_torch"]),
    "bf16 ties rounded away from zero": (
        "bf16_round",
        _source_with(_ORIG_BF16, "np.rint(np.ldexp(xf, -q))", "np.trunc(np.ldexp(xf, -q) + np.copysign(0.5, xf))"),
        ["test_bf16_round_matches_torch_on_fp32_values"]),
    "bf16 truncates": (
        "bf16_round", _source_with(_ORIG_BF16, "np.rint(np.ldexp(xf, -q))", "np.trunc(np.ldexp(xf, -q))"),
        ["test_bf16_round_matches_torch_on_fp32_values"]),
    "bf16 keeps one bit too few": (
        "bf16_round", _source_with(_ORIG_BF16, "q = np.maximum(e - 8, -133)", "q = np.maximum(e - 7, -133)"),
        ["test_bf16_round_matches_torch_on_fp32_values"]),
    "rmsnorm eps outside the root": ("rmsnorm", _rmsnorm_eps_outside_root, ["test_rmsnorm_matches_torch"]),
    "rmsnorm drops its weight": ("rmsnorm", _rmsnorm_drops_weight, ["test_rmsnorm_matches_torch"]),
    "rope turns backwards": ("rope", _rope_backwards,
                             ["test_rope_rotate_half_closed_form", "test_rope_matches_complex_rotation_and_is_relative"]),
    "rope frequency exponent halved": ("rope", _rope_half_exponent,
                                       ["test_rope_rotate_half_closed_form",
                                        "test_rope_matches_complex_rotation_and_is_relative"]),
    "rope pairs interleaved": ("rope", _rope_interleaved_pairs,
                               ["test_rope_rotate_half_closed_form",
                                "test_rope_matches_complex_rotation_and_is_relative"]),
    "probe without the causal mask": ("probe_scores", _probe_unmasked,
                                      ["test_probe_scores_match_sdpa_with_identity_values",
                                       "test_probe_scores_invariants_and_equal_keys_closed_form"]),
    "probe without 1/sqrt(d)": ("probe_scores", _probe_unscaled,
                                ["test_probe_scores_match_sdpa_with_identity_values"]),
    "probe heads grouped modulo": (
        "probe_scores", _source_with(_ORIG_PROBE, "        g = h // G", "        g = h % Hkv"),
        ["test_probe_scores_match_sdpa_with_identity_values"]),
    "probe mask applied after the softmax": (
        "probe_scores", _probe_mask_after_softmax,
        ["test_probe_scores_match_sdpa_with_identity_values",
         "test_probe_scores_invariants_and_equal_keys_closed_form"]),
    "ltp squared norm": ("ltp_scores", _ltp_squared,
                         ["test_ltp_identity_proxy_is_leading_norm", "test_ltp_matches_torch_on_exact_intermediates"]),
    "top-m sums the smallest": (
        "ltp_topm_scores",
        _source_with(_ORIG_TOPM, "np.sort(y, axis=1)[:, y.shape[1] - m:]", "np.sort(y, axis=1)[:, :m]"),
        ["test_ltp_topm_brute_force_and_limits"]),
    "top-m of signed values": (
        "ltp_topm_scores",
        _source_with(_ORIG_TOPM, "y = np.abs(t @ np.asarray(B, dtype=np.float64).T)",
                     "y = t @ np.asarray(B, dtype=np.float64).T"),
        ["test_ltp_topm_brute_force_and_limits"]),
    "FFN gate and up swapped": (
        "reduced_ffn", _source_with(_ORIG_FFN, "act = bf16_round(_silu(g) * u)", "act = bf16_round(_silu(u) * g)"),
        ["test_reduced_ffn_rows_match_torch_swiglu"]),
    "top-m one short": ("ltp_topm_scores", _topm_one_short, ["test_ltp_topm_brute_force_and_limits"]),
    "fusion weights swapped": ("fuse_scores", _fuse_weights_swapped,
                               ["test_fuse_modes_exact_values", "test_fuse_std_add_is_weighted_zscores"]),
    "MaxNorm-Add weights swapped": ("fuse_scores", _fuse_maxnorm_weights_swapped, ["test_fuse_modes_exact_values"]),
    "fusion without max-normalising c": ("fuse_scores", _fuse_c_not_normalised, ["test_fuse_modes_exact_values"]),
    "selection ties to the higher index": ("select_topk", _select_ties_high,
                                           [("test_select_topk_brute_force_with_ties", (10, 4, 0)),
                                            ("test_select_topk_brute_force_with_ties", (10, 4, 2))]),
    "selection tail not forced": ("select_topk", _select_tail_not_forced,
                                  [("test_select_topk_brute_force_with_ties", (10, 4, 2)),
                                   "test_select_keep_all_and_errors"]),
    "attention excludes the query's own position": ("reduced_attention", _attention_strictly_causal,
                                                    ["test_reduced_attention_matches_sdpa_rows",
                                                     "test_reduced_attention_special_cases"]),
    "attention heads grouped modulo": ("reduced_attention", _attention_heads_modulo,
                                       ["test_reduced_attention_matches_sdpa_rows"]),
    "O projection untransposed": ("attention_residual", _residual_untransposed, ["test_attention_residual_rows"]),
    "O projection without the bf16 operand": (
        "attention_residual",
        _source_with(_ORIG_RESIDUAL, "o = bf16_round(np.asarray(o_sel, dtype=np.float64).reshape(len(idx), -1))",
                     "o = np.asarray(o_sel, dtype=np.float64).reshape(len(idx), -1) * (1 + 2.0 ** -9)"),
        ["test_attention_residual_rows"]),
    "salience grouped by the wrong heads": (
        "inject_salience",
        _source_with(_ORIG_SALIENCE, "mean = q_probe[:, g * G:(g + 1) * G, :]", "mean = q_probe[:, g::Hkv, :]"),
        ["test_inject_salience_closed_form"]),
    "FFN with relu": ("reduced_ffn", _ffn_relu, ["test_reduced_ffn_rows_match_torch_swiglu"]),
    "FFN without its norm": ("reduced_ffn", _ffn_unnormalised, ["test_reduced_ffn_rows_match_torch_swiglu"]),
    "LTP scores the rows before attention": (
        "layer_forward", _layer_with("rmsnorm(h1, W.norm_ffn", "rmsnorm(h, W.norm_ffn"), _LAYER_PINS),
    "FFN runs on the attention rows": (
        "layer_forward", _layer_with("reduced_ffn(h1, idx_f,", "reduced_ffn(h1, idx_a,"), _LAYER_PINS),
    "probe rows not forced into the attention set": (
        "layer_forward", _layer_with("select_topk(s32, k, P)", "select_topk(s32, k, 0)"), _LAYER_PINS),
    "probes taken from the first rows": (
        "layer_forward", _layer_with("pp = pos[Nc - P:]", "pp = pos[:P]"), _LAYER_PINS),
    "FFN built on the pre-attention stream": (
        "layer_forward", _layer_with("h2 = reduced_ffn(h1,", "h2 = reduced_ffn(h,"), _LAYER_PINS),
    "stage prune keeps the lowest scores": ("stage_prune", _stage_prune_lowest,
                                            ["test_stage_prune_worked_example",
                                             "test_msdp_prunes_by_the_last_layers_fused_score"]),
    "active-row keys at the candidates' positions": (
        "layer_forward",
        _layer_with("reduced_attention(q_sel, pos[idx_a], kk[idx_a], vv[idx_a], pos[idx_a])",
                    "reduced_attention(q_sel, pos[idx_a], kk[idx_a], vv[idx_a], pos[:len(idx_a)])"),
        ["test_layer_kv_active_attention_is_dense_attention_of_the_active_rows",
         "test_layer_kv_active_keep_all_equals_dense_layer"]),
    "active-row flag ignored": (
        "layer_forward",
        _layer_with("    if cfg.kv_active:", "    if False:"),
        ["test_layer_kv_active_attention_is_dense_attention_of_the_active_rows",
         "test_layer_kv_active_keep_all_equals_dense_layer"]),
    "MSDP prunes by the stage's first layer": (
        "msdp_forward",
        _source_with(OS.msdp_forward, "            h, f = layer_forward(h, pos, layers[li], cfg, tr)",
                     "            h, f_l = layer_forward(h, pos, layers[li], cfg, tr)\n"
                     "            f = f_l if f is None else f"),
        ["test_msdp_prunes_by_the_last_layers_fused_score", "test_msdp_all_ratios_one_is_dense_stack_and_sets_nest"]),
    "salience direction not normalised": ("inject_salience", _salience_not_unit, ["test_inject_salience_closed_form"]),
    "sequential select with the scores swapped": (
        "select_sequential", _sequential_scores_swapped,
        [("test_select_sequential_reductions", (60,)), ("test_select_sequential_reductions", (20,))]),
    "sequential select returns pool positions": (
        "select_sequential", _sequential_pool_local,
        [("test_select_sequential_reductions", (33,)), ("test_select_sequential_reductions", (60,))]),
    "schedule prunes to the next stage's budget": (
        "schedule_forward",
        _source_with(_ORIG_SCHEDULE,
                     "k_next = min(budgets[stage] if stage + 1 < len(stage_ends) else after_last, Nc)",
                     "k_next = min(budgets[stage + 1] if stage + 1 < len(stage_ends) else after_last, Nc)"),
        ["test_schedule_without_skipping_is_the_dense_stack_and_sets_nest"]),
    "schedule prunes without keeping the probe tail": (
        "schedule_forward",
        _source_with(_ORIG_SCHEDULE, "kept, _ = select_topk(f, k_next, cfg.P)", "kept, _ = select_topk(f, k_next, 0)"),
        ["test_schedule_without_skipping_is_the_dense_stack_and_sets_nest"]),
    "schedule skips before the first skipping layer": (
        "schedule_forward",
        _source_with(_ORIG_SCHEDULE, "skip = l >= first_skip and", "skip = l >= 0 and"),
        ["test_schedule_without_skipping_is_the_dense_stack_and_sets_nest"]),
    "schedule keeps skipping after the last stage": (
        "schedule_forward",
        _source_with(_ORIG_SCHEDULE, "k = min(budgets[stage], Nc) if skip else Nc",
                     "k = min(budgets[min(stage, len(budgets) - 1)], Nc) if l >= first_skip else Nc"),
        ["test_schedule_without_skipping_is_the_dense_stack_and_sets_nest"]),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    fn, mutant, pins = MUTANTS[name]
    # the pins draw from their module's generator: start it afresh so that a
    # mutant meets the same inputs whatever ran before
    monkeypatch.setattr(PINS, "rng", np.random.default_rng(12345))
    monkeypatch.setattr(OS, fn, mutant)
    monkeypatch.setattr(O, fn, mutant)
    caught = []
    for pin in pins:
        test, args = (pin, ()) if isinstance(pin, str) else pin
        try:
            getattr(PINS, test)(*args)
        except (AssertionError, ValueError, FloatingPointError, pytest.fail.Exception):
            caught.append(test)
    assert caught, f"no pin caught the mutant: {name}"
