"""bench.py on the CPU: the reference arm (the oracle on bounded samples) runs
and prints one well-formed JSON line; the host helpers give the documented
work counts."""
import json
import os
import subprocess
import sys

import bench
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_cca_fp32",
                          "--steps", "2", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"] == "tiny_cca_fp32"


def test_algorithmic_work_of_the_headline_workload():
    w = bench.algorithmic_work(workloads.WORKLOADS["ccgqa_16k_bf16"])
    assert w["attention_flops"] == 2.0 * 4 * 16384 ** 2 * 128          # 274.9 GFLOP, causal half
    assert w["down_proj_flops"] == 2.0 * 16384 * 2048 * 1024           # 68.7 GFLOP
    assert w["out_proj_flops"] == 2.0 * 16384 * 512 * 2048             # 34.4 GFLOP
    # the roofline's bytes: 67.1 MB of latents in and q / K / V cache out
    assert w["preproc_bytes"] == 16384 * (1024 + 512 + 512) * 2.0
    # moved by this design: plus fp16 attention copies of k and v (16.8 MB) and the fp16 W_o (4.2 MB)
    assert w["preproc_bytes_moved"] == w["preproc_bytes"] + 2 * 16384 * 256 * 2 + 2 * 2048 * 512 * 2


def test_backward_flops_of_the_headline_workload():
    w = bench.algorithmic_work(workloads.WORKLOADS["ccgqa_16k_bf16"])
    f = bench.backward_flops(workloads.WORKLOADS["ccgqa_16k_bf16"])
    # five products of the forward attention's QK^T size (2.5 x its two), two GEMMs per projection
    assert f["attention_backward"] == 2.5 * w["attention_flops"]
    assert f["projections_backward"] == 2 * (w["down_proj_flops"] + w["out_proj_flops"])
    assert f["total"] == f["forward"] + f["attention_backward"] + f["projections_backward"]


def test_warmup_floor():
    r = subprocess.run([sys.executable, "bench.py", "--warmup", "2"], cwd=ROOT, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode != 0


def test_clock_samples_directory(monkeypatch, tmp_path):
    """The raw nvidia-smi samples go to $CCA_BENCH_CLOCKS_DIR when set, else the temp directory."""
    import tempfile
    import bench
    monkeypatch.setenv("CCA_BENCH_CLOCKS_DIR", str(tmp_path))
    assert bench.ClockSampler(1).path == str(tmp_path / "cca_bench_clocks_rank1.csv")
    monkeypatch.delenv("CCA_BENCH_CLOCKS_DIR")
    assert bench.ClockSampler(0).path.startswith(tempfile.gettempdir())


def test_traffic_record_only_for_its_workload_and_source():
    """The committed DRAM traffic of the attention kernel is reported only for the workload it was
    captured on, and only while the kernel source hashes as it did then."""
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    current = rec["source_sha"] == bench.file_sha(bench.ATTN_KERNEL_SRC)
    got = bench.traffic_record(rec["workload"])
    assert (got is not None) == current
    for name in workloads.WORKLOADS:
        if name != rec["workload"]:
            assert bench.traffic_record(name) is None
