"""The benchmark's JSON line on the host: the reference arm (the oracle,
timed on the CPU) carries every key the driver reads, with the types and
the fixed values the contract gives it."""

import json
import os
import subprocess
import sys

import pytest

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def line():
    env = dict(os.environ, OMP_NUM_THREADS="1")
    env.pop("RANK", None)
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, os.path.join(REPO, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_f32", "--steps", "2", "--warmup", "1"], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_reference_line_has_every_contract_key(line):
    for key, typ in [("metric", str), ("value", float), ("unit", str), ("n_gpus", int), ("steps", int),
                     ("warmup", int), ("ms_per_step", float), ("higher_is_better", bool), ("scaling", str),
                     ("dtype", str), ("data", str), ("config", dict), ("impl", str), ("cpu_baseline", dict),
                     ("e2e", dict)]:
        assert isinstance(line[key], typ), key
    assert "vs_baseline" in line
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["steps"] == 2 and line["warmup"] == 1
    assert line["higher_is_better"] is False and line["scaling"] in ("weak", "strong")
    assert abs(line["ms_per_step"] * 1e3 - line["value"]) <= 1e-6 * line["value"]


def test_reference_line_baseline_and_e2e(line):
    cb, e2e = line["cpu_baseline"], line["e2e"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["unit"] == line["unit"]
    assert isinstance(cb["sample"], str) and cb["sample"]
    assert e2e == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_line_config_names_the_workload(line):
    cfg = line["config"]
    assert cfg["workload"] == "tiny_f32"
    assert "model" not in cfg
    assert "fit in L2" in cfg["l2"]        # 4 MB of inputs: said plainly, not claimed to exceed L2


def test_launch_plan_matches_the_counted_graph_nodes():
    # The launch counts the benchmark's plan gives where the captured step graph cannot be
    # queried; the kernel nodes counted on a B200 were 3 (c1, c2, c0), 4 (c3, c4 N16-N64) and
    # 5 (c4 N128: a 128-row and a 64-row attention launch).
    sys.path.insert(0, REPO)
    import bench
    from synth import workloads as W
    for name, n in [("vicuna7b_bs1_L1024", 3), ("vicuna7b_bs1_L4096_typical", 3), ("tiny_f32", 3),
                    ("vicuna13b_bs8_ragged", 4), ("vicuna33b_bs4_L8192_N16", 4), ("vicuna33b_bs4_L8192_N64", 4),
                    ("vicuna33b_bs4_L8192_N128", 5)]:
        w = W.get(name)
        assert bench.expected_launches(w, w.T) == n, name
    w = W.shrink(W.get("vicuna13b_bs8_ragged"), name="b17", B=17)
    assert bench.expected_launches(w, w.T) == 2 * 2 + 1 + 1   # two tensor-core passes


def test_kernel_short_name():
    sys.path.insert(0, REPO)
    import bench
    assert bench._kernel_short_name("_ZN6medusa12_GLOBAL__N_115heads_tc_kernelILi1ELi16EEEvNS0_4ArgsE") == \
        "heads_tc_kernel"
    assert bench._kernel_short_name("_ZN6medusa16posterior_kernelILi0EEEvNS_8PostArgsE") == "posterior_kernel"
    assert bench._kernel_short_name("plain_name") == "plain_name"
