"""bench.py's output contract, checked on the CPU through the reference arm
(the oracle timed on the host), and the byte accounting both arms share."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_reference_arm_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "GB/s"
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["steps"] == 1 and d["warmup"] == 3
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    import bench
    assert d["config"] == bench.run_config(1)  # the kernel arm's config
    assert d["metric"] == bench.METRIC


def test_warmup_below_three_is_rejected():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "2"], capture_output=True, text=True,
                         timeout=300, cwd=ROOT)
    assert out.returncode != 0


def test_algorithmic_bytes():
    import bench
    # lm_head, M = 1, bf16 out: codes + d/m + x + y
    assert bench.gemv_bytes(151936, 2560, 1) == 151936 * 1280 + 151936 * 10 * 4 + 2560 * 2 + \
        151936 * 2 == 200864512
    # keep-quant: int8 activations plus fp32 scales and int32 sums per 32-block
    assert bench.w4a8_gemv_bytes(2560, 4096, 4) == 2560 * 2048 + 2560 * 16 * 4 + 4 * 4096 + \
        4 * 128 * 8 + 4 * 2560 * 2
    assert bench.mmq_ops(2048, 19456, 2560) == 2 * 2048 * 19456 * 2560
    # the five decode shapes stream 253 MB per step, 2.078 GB per chain token
    step = sum(bench.gemv_bytes(n, k, 1) for n, k in bench.SHAPES)
    assert 250e6 < step < 256e6


def test_traffic_is_used_only_for_the_source_it_was_taken_on(tmp_path, monkeypatch):
    import bench
    kernel = "w4_quant_matmul_b200/csrc/gemv.cu"
    (tmp_path / "profiles").mkdir()
    entry = {"dram_bytes_per_launch": 123, "capture": "ncu --set full, kernel k, one launch"}

    def write(h):
        with open(tmp_path / "profiles" / "traffic.json", "w") as f:
            json.dump({"k": dict(entry, source_hash=h)}, f)

    # the hash is read from the real kernel source; the table from tmp_path
    current = bench.source_hash(kernel)
    monkeypatch.setattr(bench, "source_hash", lambda f: current if f == kernel else "")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    write(current)
    assert bench.load_traffic(kernel, "k") == (123, "ncu --set full, kernel k, one launch")
    write("0" * 16)
    value, why = bench.load_traffic(kernel, "k")
    assert value is None and current in why and "0" * 16 in why
    assert bench.load_traffic(kernel, "other")[0] is None
