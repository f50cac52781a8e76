"""Host-side checks of bench.py: the algorithmic byte counts behind every
roofline fraction, the reference arm's JSON line, and the helpers that read
the committed ncu traffic and the measured peaks.  No test here needs a GPU.

The byte counts follow the layer's inputs and outputs (chatgpz.de explainer,
section "Von Residualverbindungen zu Hyperverbindungen", update equation;
reportify.cn mHC summary [12], [16]-[21]): per token the stream buffer x is
n x C, the layer input h_in and the function output f_out are C wide, and the
maps are H_pre (n), H_post (n) and H_res (n x n).  Activations are bf16 and
the maps fp32.
"""
import json
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BF16, F32 = 2, 4


def shape_bytes(n, C):
    """Bytes per token of each call, counted from the tensors it reads and
    writes once, written out tensor by tensor."""
    x, row = n * C * BF16, C * BF16                      # x or a gradient of it; h_in / f_out
    H_pre, H_post, H_res = n * F32, n * F32, n * n * F32
    return {
        # x in; h_in and the three maps out
        "pre": x + row + H_pre + H_post + H_res,
        # x, f_out, H_post, H_res in; x_next out
        "post": x + row + H_post + H_res + x,
        # x, H_pre in; h_in out
        "layer_input": x + H_pre + row,
        # one pass of the backward: x, grad_x_next, grad_h_in, f_out in;
        # grad_x and grad_f_out out
        "bwd_min": x + x + row + row + x + row,
    }


@pytest.mark.parametrize("n", [4, 8, 16])
def test_per_token_bytes_match_the_tensor_shapes(n):
    got = bench.per_token_bytes(n, 7168)
    for call, want in shape_bytes(n, 7168).items():
        assert got[call] == want, call


def test_layer_step_bytes_at_the_benchmark_shape():
    # n = 4, C = 7168: 71,776 (pre) + 129,104 (post) + 215,040 (one-pass
    # backward) = 415,920 bytes per token
    tb = bench.per_token_bytes(4, 7168)
    assert (tb["pre"], tb["post"], tb["bwd_min"]) == (71776, 129104, 215040)
    assert tb["pre"] + tb["post"] + tb["bwd_min"] == 415920
    # the apply as built re-reads x, grad_x_next and grad_h_in next to the
    # mapping's 52-float coefficient record: 200,912 bytes per token
    assert tb["bwd_apply"] == 200912


def test_phi_bytes_per_call():
    # phi is nC x (n^2 + 2n) fp32: 2.75 MB at n = 4, C = 7168; the apply reads
    # it and writes grad_phi
    pb = bench.per_call_param_bytes(4, 7168)
    assert pb["pre"] == 4 * 7168 * 24 * 4 == 2752512
    assert pb["bwd_apply"] == 2 * pb["pre"]
    assert pb["post"] == pb["layer_input"] == 0


def test_layer_metric_names_the_stream_count():
    assert bench.layer_metric(4) == bench.METRIC
    assert "n=8" in bench.layer_metric(8) and "n=4" not in bench.layer_metric(8)
    assert "n=16" in bench.layer_metric(16)


def test_step_stats():
    s = bench.step_stats([5.0, 1.0, 3.0, 2.0, 4.0])
    assert (s["median"], s["min"], s["max"], s["n"]) == (3.0, 1.0, 5.0, 5)
    assert s["p10"] <= s["median"] <= s["p90"]
    assert bench.step_stats([]) is None


def test_peaks_fall_back_without_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 7012.5}))
    assert bench.load_peaks() == (7012.5, "measured")


def test_ncu_traffic_is_tied_to_the_kernel_sources(monkeypatch):
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
        table = json.load(f)
    keys = [k for k in table if not k.startswith("_")]
    assert keys
    for k in keys:
        assert k in bench.CALL_SOURCES, k
        v = bench.ncu_traffic(k)
        assert v is None or v > 0
    # a figure taken on other sources is never reported
    monkeypatch.setattr(bench, "kernel_source_sha", lambda files: "0" * 16)
    assert all(bench.ncu_traffic(k) is None for k in keys)
    assert bench.ncu_traffic("no_such_call") is None


def _reference_line(*args, env=None):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--steps", "3", "--warmup", "1", "--reference-seconds", "2", *args]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    return lines


@pytest.mark.parametrize("workload,extra,metric,unit", [
    ("layer", [], bench.METRIC, "tokens/s"),
    ("layer", ["--streams", "8"], bench.layer_metric(8), "tokens/s"),
    ("sinkhorn", [], bench.SINKHORN_METRIC, "matrices/s"),
    ("depth", [], bench.DEPTH_METRIC, "tokens/s"),
])
def test_reference_arm_line(oracle_mod, workload, extra, metric, unit):
    lines = _reference_line("--workload", workload, *extra)
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert (d["metric"], d["unit"]) == (metric, unit)
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["n_gpus"] == 1 and d["steps"] == 3
    assert d["warmup"] == 3                     # the parser's floor of three warm-up steps
    assert d["dtype"] == "f64" and d["data"] == "synthetic" and d["vs_baseline"] is None
    assert d["value"] > 0 and d["ms_per_step"] > 0
    cfg = d["config"]
    assert isinstance(cfg["workload"], str) and cfg["parallelism"] == "host cores (oracle)"
    # the value is the units of one step's sample over its measured time
    per_step = cfg.get("tokens_per_step", cfg.get("matrices_per_step"))
    assert per_step >= 1
    assert d["value"] == pytest.approx(per_step / (d["ms_per_step"] / 1000.0), rel=1e-9)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["unit"] == unit
    assert 1 <= cb["cores"] <= oracle_mod.num_threads()
    assert d["e2e"] == {"value": d["value"], "unit": unit, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_prints_nothing_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    assert _reference_line(env=env) == []
