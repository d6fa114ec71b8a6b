"""Host-side checks of bench.py that need no GPU: the reference arm prints one JSON line with
the keys of the benchmark contract, and the DRAM-traffic figure is taken from a committed ncu
summary only while that summary's kernel source is the one in the tree."""
import hashlib
import importlib.util
import json
import os
import re
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


def _fake_tree(tmp_path, kind, kernel_text, per_pair, recorded_text):
    b = _bench_module()
    name, src_name, _ = b.TRAFFIC_PROFILES[kind]
    (tmp_path / "profiles").mkdir(exist_ok=True)
    csrc = tmp_path / "trainable_block_sparse_fine_b200" / "csrc"
    csrc.mkdir(parents=True, exist_ok=True)
    (csrc / src_name).write_bytes(kernel_text)
    sha = hashlib.sha1(recorded_text).hexdigest()
    (tmp_path / "profiles" / name).write_text(f"dram_bytes_per_pair: {per_pair}\nsource_sha1: {sha}\n")
    return b


def test_profiled_traffic_follows_the_kernel_source(tmp_path):
    fwd = S.WORKLOADS["720p_top64"]
    pairs = fwd.batch * fwd.heads * fwd.num_tiles * fwd.topk
    b = _fake_tree(tmp_path, "fwd", b"kernel v1", 1234, b"kernel v1")
    assert b.profiled_traffic("fwd", fwd, pairs, root=str(tmp_path)) == 1234 * pairs
    # another workload shape: no figure
    assert b.profiled_traffic("fwd", S.WORKLOADS["480p_top64"], pairs, root=str(tmp_path)) is None
    # the kernel source changed since the counters were taken: no figure
    b = _fake_tree(tmp_path, "fwd", b"kernel v2", 1234, b"kernel v1")
    assert b.profiled_traffic("fwd", fwd, pairs, root=str(tmp_path)) is None
    train = S.WORKLOADS["480p_train_top64"]
    b = _fake_tree(tmp_path, "bwd", b"bwd", 99, b"bwd")
    assert b.profiled_traffic("bwd", train, 10, root=str(tmp_path)) == 990


def test_committed_summaries_name_a_source_and_a_figure():
    b = _bench_module()
    for name, src, _ in b.TRAFFIC_PROFILES.values():
        txt = open(os.path.join(ROOT, "profiles", name)).read()
        assert re.search(r"dram_bytes_per_pair:\s*\d+", txt) and re.search(r"source_sha1:\s*[0-9a-f]{40}", txt)
        assert os.path.exists(os.path.join(ROOT, "trainable_block_sparse_fine_b200", "csrc", src))
