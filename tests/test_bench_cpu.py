"""The benchmark's CPU legs (no GPU): the workload table, the oracle reference arm's JSON
line and the CPU baseline, on the small configurations."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


@pytest.mark.parametrize("cfg", list(range(1, 14)))
def test_workloads_are_complete(cfg):
    w = bench.workload(cfg)
    for key in ("kind", "B", "H", "D", "n", "plen", "cap", "name"):
        assert key in w, (cfg, key)
    assert len(w["plen"]) == w["B"] and w["H"] == 16 and w["D"] == 128


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    return out


@pytest.mark.parametrize("cfg", [1, 9])
def test_reference_arm_json_line(cfg):
    out = _run("--impl", "reference", "--config", str(cfg), "--steps", "2", "--warmup", "3")
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["metric"] == bench.METRIC
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["config_index"] == cfg


def test_warmup_below_three_is_refused():
    out = _run("--impl", "reference", "--config", "1", "--steps", "1", "--warmup", "2")
    assert out.returncode != 0 and "warmup" in out.stderr


def test_cpu_baseline_reports_threads_and_a_one_thread_figure():
    r = bench.cpu_baseline(bench.workload(1), budget_s=0.5, budget_1thread_s=0.3)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["value_1thread"] > 0
    assert r["cores"] >= 1 and r["host_cpus"] >= 1 and r["cpu_model"]


def test_traffic_records_follow_the_kernel_source():
    # a committed DRAM-traffic record is reported only while the kernel source it was captured on
    # is unchanged (comments and blank lines aside); every record names a known workload key
    kinds = {"rswa_decode": "dense", "srswa_decode": "sparse", "srswa_step_decode": "sparse",
             "rswa_prefill": "prefill", "srswa_prefill": "srswa_prefill", "rope": "rope"}
    lines = [ln.split() for ln in open(os.path.join(ROOT, "profiles", "ncu_traffic.txt"))
             if ln.strip() and not ln.startswith("#")]
    assert lines
    for parts in lines:
        key, src_hash, nbytes = parts[0], parts[1], float(parts[2])
        kind = kinds[key.rsplit("_config", 1)[0]]
        assert nbytes > 0
        assert bench.committed_traffic(key, src_hash) == nbytes
        assert bench.committed_traffic(key, "0" * 16) is None           # another source: no record
        assert len(bench.kernel_source_hash(kind)) == 16


def test_kernel_source_hash_ignores_comments(tmp_path, monkeypatch):
    # the hash strips comments and blank lines: a comment edit keeps a traffic record valid,
    # a code edit does not
    csrc = tmp_path / "long_context_decode_swa_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("rope.cu", "common.cuh"):
        (csrc / name).write_text(open(os.path.join(ROOT, "long_context_decode_swa_b200", "csrc", name)).read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash("rope")
    (csrc / "rope.cu").write_text((csrc / "rope.cu").read_text() + "\n// a note\n\n/* another */\n")
    assert bench.kernel_source_hash("rope") == h0
    (csrc / "rope.cu").write_text((csrc / "rope.cu").read_text() + "\nstatic int extra_symbol;\n")
    assert bench.kernel_source_hash("rope") != h0
