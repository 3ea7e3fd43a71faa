"""bench.py's reference arm (the fp64 oracle on the host cores) runs on the CPU
and prints the one JSON line the benchmark contract asks for."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("workload", ["tiny3d", "table_il", "ucpe"])
def test_reference_arm_json_line(workload):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", workload, "--steps", "3", "--warmup", "3",
                        "--cpu-seconds", "0.2"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3
    assert d["unit"] == "tokens/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == workload and d["n_gpus"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_kernel_hash_ignores_comments(tmp_path, monkeypatch):
    """The traffic key changes with the kernels' code, not with their comments."""
    sys.path.insert(0, ROOT)
    import bench

    csrc = os.path.join(ROOT, "qk_rmsnorm_rope_qknr_b200", "csrc")
    fake_pkg = tmp_path / "qk_rmsnorm_rope_qknr_b200" / "csrc"
    fake_pkg.mkdir(parents=True)
    for f in os.listdir(csrc):
        (fake_pkg / f).write_bytes(open(os.path.join(csrc, f), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash("3d")
    p = fake_pkg / "rope3d.cu"
    p.write_text("// a new comment\n/* and a block\n comment */\n" + p.read_text() + "\n\n")
    assert bench.kernel_source_hash("3d") == h0
    p.write_text(p.read_text().replace("kMaxGroups = 15", "kMaxGroups = 14"))
    assert bench.kernel_source_hash("3d") != h0


def test_one_core_figure_restores_threads():
    """The single-thread oracle figure beside the all-core one: positive, and
    the oracle's thread count is as before afterwards."""
    sys.path.insert(0, ROOT)
    import bench
    import oracle as O
    import workloads as W

    before = O.threads()
    for name, chunk in (("tiny3d", 16), ("table_il", 16)):
        w = W.WORKLOADS[name]
        inp = W.make_inputs(w, device="cpu", tokens=64 if name == "table_il" else None)
        if name == "table_il":
            import dataclasses
            w = dataclasses.replace(w, tokens=64)
        assert bench.one_core(w, inp, 0.05, chunk) > 0
        assert O.threads() == before


def test_host_cost_program_builds():
    """The C host-cost program (tests/host_cost.c) compiles and links against
    libqknr.so; running it needs a GPU."""
    import bench

    exe = bench.host_cost_exe()
    assert os.path.exists(exe) and os.access(exe, os.X_OK)
