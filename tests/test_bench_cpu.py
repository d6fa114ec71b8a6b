"""Host-side checks of bench.py that need no GPU: the reference arm prints one JSON line with
the keys of the benchmark contract, and the DRAM-traffic figure is taken from a committed ncu
summary only while that summary's kernel source is the one in the tree."""
import importlib.util
import json
import os
import subprocess
import sys

import synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench_module():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1",
                        "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_profiled_traffic_follows_the_kernel_source():
    b = _bench_module()
    fwd = S.WORKLOADS["720p_top64"]
    pairs = fwd.batch * fwd.heads * fwd.num_tiles * fwd.topk
    got = b.profiled_traffic("fwd", fwd, pairs)
    assert got is not None and got > 32768 * pairs * 0.1  # the committed summary matches the tree
    train = S.WORKLOADS["480p_train_top64"]
    assert b.profiled_traffic("bwd", train, train.batch * train.heads * train.num_tiles * train.topk) is not None
    # another workload shape, or a summary whose recorded source is not this kernel's: no figure
    assert b.profiled_traffic("fwd", S.WORKLOADS["480p_top64"], pairs) is None
    name, _, grid = b.TRAFFIC_PROFILES["fwd"]
    b.TRAFFIC_PROFILES["fwd"] = (name, "router.cu", grid)
    assert b.profiled_traffic("fwd", fwd, pairs) is None
