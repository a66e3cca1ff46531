"""Host-side pieces of bench.py checked on CPU: the algorithmic work it
divides by (brute-force pair counts), and the ncu traffic figure it reports
only while the captured kernel source is unchanged."""

import os
import types

import numpy as np

import bench


def _wl(kv_active=False):
    return types.SimpleNamespace(D=64, Hq=4, Hkv=2, d=16, F=96, r=8, ltp_dout=0, kv_active=kv_active)


def _visible_pairs(q_rows, key_rows, pos):
    # causal by original position: query row i sees key row j iff pos[j] <= pos[i]
    return sum(1 for i in q_rows for j in key_rows if pos[j] <= pos[i])


def test_attention_and_probe_flops_are_the_visible_pair_counts():
    rng = np.random.default_rng(3)
    Nc, k, P = 57, 13, 5
    pos = np.sort(rng.choice(10 * Nc, Nc, replace=False))
    idx = np.sort(rng.choice(Nc, k, replace=False))
    wl = _wl()
    fl, _ = bench.layer_work(wl, Nc, k, P, idx)
    assert fl["reduced_attention"] == 4.0 * wl.Hq * wl.d * _visible_pairs(idx, range(Nc), pos)
    probe_rows = range(Nc - P, Nc)
    assert fl["probe_scores"] == 2.0 * 2.0 * wl.Hq * wl.d * _visible_pairs(probe_rows, range(Nc), pos)
    # active-row keys: the selected queries attend to the selected keys only
    wl_kv = _wl(kv_active=True)
    fl_kv, _ = bench.layer_work(wl_kv, Nc, k, P, idx)
    assert fl_kv["reduced_attention"] == 4.0 * wl.Hq * wl.d * _visible_pairs(idx, idx, pos)
    assert fl_kv["v_proj"] == 2.0 * k * wl.D * wl.Hkv * wl.d


def test_gemm_flops():
    wl = _wl()
    Nc, k, P = 40, 9, 3
    fl, _ = bench.layer_work(wl, Nc, k, P, np.arange(k))
    assert fl["gate_up_swiglu"] == 2 * (2.0 * k * wl.D * wl.F)
    assert fl["down_proj_scatter"] == 2.0 * k * wl.F * wl.D
    assert fl["q_proj_rope"] == 2.0 * k * wl.D * wl.Hq * wl.d
    assert fl["ltp_scores"] == 2.0 * Nc * (wl.D * wl.r + wl.r * wl.D)


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    """A tree whose kernel source matches the summary's recorded hash gets
    the summary's DRAM figure; one byte of difference gives None."""
    import hashlib
    src_dir = tmp_path / "token_skipping_sparse_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    text = "// a kernel source\n"
    (src_dir / "attn.cu").write_text(text)
    sha = hashlib.sha256(text.encode()).hexdigest()[:16]
    (tmp_path / "profiles" / "attention_bf16_layer_32k.md").write_text(
        f"Source: attn.cu sha256 prefix `{sha}`.\n\n| DRAM read / write per launch | 215.8 MB / 59.9 MB |\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.captured_traffic("layer_32k", "reduced_attention") == round(275.7e6)
    assert bench.captured_traffic("layer_128k", "reduced_attention") is None      # no capture
    assert bench.captured_traffic("layer_32k", "gate_up_swiglu") is None          # no summary kind
    (src_dir / "attn.cu").write_text(text + "\n")
    assert bench.captured_traffic("layer_32k", "reduced_attention") is None


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one
    JSON line with the contract's keys, on a small workload."""
    import json
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "layer_small", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=300, check=True).stdout
    lines = [ln for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"]
    assert d["metric"] == bench.METRIC and d["config"]["workload"] == "layer_small"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # the GPU arm's config object, key for key
    from synthetic import WORKLOADS
    wl = WORKLOADS["layer_small"]
    assert d["config"] == bench.layer_config(wl, wl.k, 1)
    assert "scaled" in cb["sample"] and "not scaled" in cb["sample"]


def test_cpu_baseline_times_one_whole_layer():
    from synthetic import WORKLOADS
    wl = WORKLOADS["layer_small"]
    cb = bench.cpu_baseline(wl)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1
    assert abs(cb["value"] * cb["seconds"] - wl.N) <= 0.05 * wl.N   # seconds is rounded to 1 ms
    assert "unavailable" in bench.cpu_baseline(WORKLOADS["layer_small_kv"])


def test_topk_path_label_matches_the_library_threshold():
    import re
    src = open(os.path.join(bench.ROOT, "token_skipping_sparse_b200", "csrc", "topk.cu")).read()
    m = re.search(r"#define TK_GRID_MIN (\d+)", src)
    assert m and int(m.group(1)) == bench.TOPK_GRID_MIN
