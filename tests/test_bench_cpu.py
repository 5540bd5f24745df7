"""The benchmark's reference arm (the fp64 oracle timed on the host cores)
runs without a GPU.  This checks that its JSON line keeps the contract the
driver reads: the same metric, unit and direction as the GPU arm, a bounded
sample stated in `cpu_baseline`, and an `e2e` object with no host<->device
bytes (the oracle never touches a device)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _reference_line(*extra):
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "0", *extra], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_arm_json_contract():
    """The default workload: the 64-layer hidden-5120 decoder."""
    import bench
    d = _reference_line()
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["higher_is_better"] is True and d["n_gpus"] == 1 and d["steps"] == 1
    assert d["warmup"] >= 3                          # warm-up is never below three steps
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "dense64L-h5120-ffn25600-q4"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "layer 0" in cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


@pytest.mark.parametrize("workload", ["dense16L-h2048-ffn8192-q4", "dense16L-h2048-ffn8192-q3",
                                      "dense16L-h2048-ffn8192-q2"])
def test_reference_arm_other_formats(workload):
    d = _reference_line("--workload", workload)
    assert d["config"]["workload"] == workload and d["value"] > 0


def test_reference_arm_shrinks_its_step_to_the_time_budget():
    """Steps + warm-up of whole layers that would overrun the budget make each
    step a share of every matrix's rows instead; the line says which share."""
    d = _reference_line("--steps", "400", "--ref-budget-s", "2", "--workload",
                        "dense16L-h2048-ffn8192-q4")
    assert d["steps"] == 400 and d["value"] > 0
    assert d["config"]["sample"] == "a share of one layer per step"
    assert "of the rows of every matrix of layer 0" in d["cpu_baseline"]["sample"]
    share = d["config"]["rows_share"]
    assert 0 < share < 1
    # ms_per_step is a whole layer's time; the share of it timed per step fits
    # the 2 s budget (with slack for a loaded host)
    assert d["ms_per_step"] * share * 403 < 30e3
    # the rate is the same whether the layer or its share is counted
    layer_mb = 34.3
    assert abs(layer_mb * 1e6 / (d["ms_per_step"] / 1e3) / 1e9 - d["value"]) < 0.2 * d["value"]


def test_default_workload_is_the_largest_single_gpu_decoder():
    import bench
    src = open(os.path.join(ROOT, "bench.py")).read()
    assert 'default=synth.DENSE_H5120.name' in src
    wl = bench.WORKLOADS["dense64L-h5120-ffn25600-q4"]
    assert wl.layers == 64 and wl.B == 1



def test_reference_arm_attention_workload():
    """The oracle arm on a decode-attention workload: layer 0's attention over
    the Q8 cache (the same seeded keys, values, queries and lengths)."""
    d = _reference_line("--workload", "attn16L-kv4-g4-t8192-b8-mixed", "--steps", "1")
    assert d["config"]["workload"] == "attn16L-kv4-g4-t8192-b8-mixed" and d["value"] > 0
    assert "layer 0" in d["cpu_baseline"]["sample"]


def test_profile_traffic_markers_match_the_current_sources():
    """Each `bench-traffic` marker under profiles/ (the DRAM bytes a bench line
    reports as `roofline.traffic`) names a benchmark workload, the graph
    engine, a positive byte count, and the hash of the kernel sources it was
    captured on; every marker is for the current sources (a summary of an
    earlier revision carries none), and the default workload has one."""
    import glob
    import re
    import bench
    found = {}
    for p in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for line in open(p):
            m = re.search(r"bench-traffic:(.*?)-->", line)
            if not m:
                continue
            kv = dict(t.split("=", 1) for t in m.group(1).split() if "=" in t)
            wl = kv["workload"]
            assert wl in bench.WORKLOADS, (p, wl)
            assert kv["engine"] == "graph", p
            assert int(kv["bytes_per_launch"]) > 0, p
            unit = ("attention.cu" if wl.startswith("attn") else
                    "verify_gemm.cu" if wl.startswith("verify") else "stream_gemv.cu")
            assert kv["source_sha256"] == bench.kernel_source_hash(unit), \
                f"{os.path.basename(p)}: {unit} changed since this traffic was captured"
            assert bench.profiled_traffic(wl, "graph", unit) == int(kv["bytes_per_launch"])
            found[wl] = int(kv["bytes_per_launch"])
    assert "dense64L-h5120-ffn25600-q4" in found


@pytest.mark.parametrize("workload", ["moe48L-e128-top8-h2048-b1", "moe48L-e128-top8-h2048-b8"])
def test_reference_arm_routed_experts(workload):
    """The oracle arm on the routed-expert workload: layer 0's routed experts
    (gate|up with SwiGLU, then down combined in slot order) per step."""
    d = _reference_line("--workload", workload)
    assert d["config"]["workload"] == workload and d["value"] > 0
    assert d["config"]["sample"] == "one layer per step"
    assert "layer 0" in d["cpu_baseline"]["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0
