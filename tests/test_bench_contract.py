"""The benchmark's JSON line contract, exercised on the CPU through the reference
arm (the float64 oracle on a bounded sample), and the AR cache budget."""
import json
import math
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("pass_", ["fwd", "bwd", "sics"])
def test_reference_arm_prints_one_contract_line(pass_):
    d = run_bench("--impl", "reference", "--workload", "sta_tiny", "--steps", "1", "--warmup",
                  "0", "--pass", pass_)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup",
                "higher_is_better", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["unit"] == ("GB/s" if pass_ == "sics" else "TFLOP/s")
    assert d["config"]["workload"] == "sta_tiny"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


@pytest.mark.parametrize("workload", ["nabla_480p", "ar_decode", "spade_480p"])
def test_reference_arm_on_dynamic_masks(workload):
    # the oracle builds its own NABLA / autoregressive mask (untimed) and is timed
    # on sampled query blocks (two heads keep the CPU run short)
    d = run_bench("--impl", "reference", "--workload", workload, "--heads", "2", "--steps", "1",
                  "--warmup", "0", "--cpu-budget", "1")
    assert d["config"]["workload"] == workload and d["value"] > 0
    assert "oracle's own mask" in d["cpu_baseline"]["sample"]


def test_peak_choice_follows_the_run():
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}
    capped = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0}
    assert bench.choose_tensor_peak(peaks, at_max, 10.0)[:2] == (1600.0, "burst")
    assert bench.choose_tensor_peak(peaks, at_max, 1.0)[:2] == (1600.0, "burst")
    assert bench.choose_tensor_peak(peaks, capped, 1.0)[:2] == (1400.0, "sustained")
    assert bench.choose_tensor_peak(peaks, capped, 10.0)[:2] == (1400.0, "sustained")
    assert bench.choose_tensor_peak(peaks, {"sm_mhz": None}, 10.0)[:2] == (1600.0, "burst")
    r = bench.tensor_roofline(700.0, 20.0, peaks, "measured", capped, 10.0, attn_ms=20.0)
    assert r["frac"] == 0.5 and r["frac_of_burst"] == 700.0 / 1600.0
    assert r["kernel_ms_x_sm_mhz"] == 20.0 * 1500.0 and r["attn_ms"] == 20.0


def test_ar_budget_keeps_the_target_fraction():
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_tokens_b200 import configs
    w = configs.get("ar_decode")
    budget = bench.ar_budget(w)
    n_pages = math.ceil(w.n_tokens / 128)
    anchor = math.ceil(w.anchor_frames * w.tokens_per_frame / 128)
    recent = n_pages - (w.n_tokens - w.recent_frames * w.tokens_per_frame) // 128
    kept = (anchor + recent + budget) / n_pages
    assert abs(kept - bench.AR_KEEP_FRACTION) < 1.0 / n_pages


def test_roofline_reports_the_fraction_of_nominal_for_both_bounds():
    sys.path.insert(0, ROOT)
    import bench
    t = bench.with_nominal({"bound": "tensor", "achieved": 1125.0, "unit": "TFLOP/s"})
    h = bench.with_nominal({"bound": "hbm", "achieved": 3850.0, "unit": "GB/s"})
    assert t["frac_of_nominal"] == 0.5 and h["frac_of_nominal"] == 0.5


def test_mask_stats_of_the_forward_line():
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_tokens_b200 import configs
    w = configs.get("sta_720p")
    # the 720p window keeps 9,152 of 90,000 tile pairs, all tiles full
    flops = 4.0 * w.head_dim * 9152 * 384 * 384 * w.batch * w.heads
    st = bench.mask_stats(flops, w, w.nq, w.nk, [3.0, 1.0, 2.0, 5.0, 4.0], near=None)
    assert abs(st["kept_pair_fraction"] - 9152 / 90000) < 1e-12
    assert (st["attn_ms_p10"], st["attn_ms_median"], st["attn_ms_p90"]) == (1.0, 3.0, 5.0)
    assert "near_threshold_rows" not in st
    assert bench.mask_stats(flops, w, w.nq, w.nk, [1.0], near=7)["near_threshold_rows"] == 7


def test_paged_pass_refuses_a_workload_without_ar_decoding():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--pass", "ar_paged", "--workload", "sta_tiny", "--steps", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 2 and "autoregressive" in out.stderr


def test_permute_bandwidth_counts_the_algorithmic_bytes():
    from types import SimpleNamespace
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_tokens_b200 import configs
    w = configs.get("sta_720p")
    plan = SimpleNamespace(permuted=True, n_pad=115200)
    row = 24 * 128 * 2
    got = bench.permute_bandwidth(w, plan, {"permute": 0.714, "untile": 0.235}, 6543.4)
    assert got["permute"]["bytes"] == 3 * 2 * 115200 * row       # Q, K, V read + written
    assert got["untile"]["bytes"] == 2 * 115200 * row             # O read + written
    assert abs(got["permute"]["gb_s"] - 3 * 2 * 115200 * row / 0.714e-3 / 1e9) < 1e-6
    assert 0.9 < got["permute"]["frac_of_hbm"] < 0.92
    assert bench.permute_bandwidth(w, SimpleNamespace(permuted=False), {}, 6543.4) is None


def test_committed_profiles_describe_the_current_kernel_sources():
    # every ncu summary bench.py reads its DRAM traffic from was captured on the
    # kernel sources as they are now (the summary's source hash matches), so the
    # bench line's roofline carries that traffic instead of null
    sys.path.insert(0, ROOT)
    import bench
    for workload, kind in (("radial_long", "attn_fwd"), ("sta_720p", "attn_fwd"),
                           ("nabla_480p", "attn_fwd"), ("sta_720p", "attn_bwd"),
                           ("nabla_480p", "sics")):
        assert bench.profiled_traffic(workload, kind) is not None, (workload, kind)
