"""Host logic of bench.py on CPU: the algorithmic work per call, the roofline
choice, the ncu traffic record, and the oracle reference arm."""
import json
import os
import subprocess
import sys

import pytest

import bench
from adaptive_vector_quantized_avq_b200 import synthetic as syn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_work_of_the_headline_workload():
    """max-64k: K+V and Q+O are 2 x 1M rows x 64 x 2 bytes; the cost model
    counts M0 + C distances per key and M0 + P*C logits (twice: logits and
    weighted values) per query."""
    wl = syn.WORKLOADS["max-64k"]
    alg = bench.algorithmic(wl, 16)
    R = 1 * 16 * 65536
    assert alg["precompute"]["bytes"] == 2 * R * 64 * 2 == 268435456
    assert alg["attention"]["bytes"] == 268435456
    assert alg["precompute"]["flops"] == 2 * R * (128 + 8) * 64
    assert alg["attention"]["flops"] == 4 * R * (128 + 16 * 8) * 64 == 68719476736


def test_roofline_takes_the_slower_bound():
    peaks = {"hbm_gbs": 6552.3, "bf16_tflops": 1659.5, "bf16_tflops_sustained": 1401.0}
    wl = syn.WORKLOADS["max-64k"]
    alg = bench.algorithmic(wl, 16)
    pre = bench.roofline_for("precompute", alg["precompute"], 0.2, peaks, True)
    att = bench.roofline_for("attention", alg["attention"], 0.25, peaks, True)
    assert pre["bound"] == "hbm" and pre["unit"] == "GB/s"
    assert abs(pre["achieved"] - 268435456 / 0.2e-3 / 1e9) < 1e-6
    assert abs(pre["roofline_us"] - 268435456 / 6552.3e9 * 1e6) < 1e-6
    assert att["bound"] == "tensor" and att["peak"] == 1401.0
    assert abs(att["frac"] - 68719476736 / 0.25e-3 / 1e12 / 1401.0) < 1e-12
    burst = bench.roofline_for("attention", alg["attention"], 0.25, peaks, False)
    assert burst["peak"] == 1659.5


def test_ingest_records_traffic_per_launch(tmp_path, monkeypatch):
    csv_path = tmp_path / "traffic.csv"
    head = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",'
            '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n')
    rows = []
    for i, (name, rd, wr) in enumerate([("void avq::precompute_tc_kernel<64, 8, 4>(x)", "200.0", "4.0"),
                                        ("void avq::attention_tree_kernel<64, 8, 2, true>(x)", "100.0", "50.0"),
                                        ("void avq::precompute_tc_kernel<64, 8, 4>(x)", "202.0", "4.0")]):
        for metric, unit, val in (("dram__bytes_read.sum", "Mbyte", rd), ("dram__bytes_write.sum", "Mbyte", wr)):
            rows.append(f'"{i}","1","python","h","{name}","1","7","(1,1,1)","(1,1,1)","0","10.0",'
                        f'"Command line profiler metrics","{metric}","{unit}","{val}"\n')
    csv_path.write_text("==PROF== noise\n" + head + "".join(rows))
    out = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(out))
    bench.ingest_ncu(str(csv_path), "max-64k", 16)
    rec = json.loads(out.read_text())
    pre, att = rec["precompute/max-64k/P16"], rec["attention/max-64k/P16"]
    assert pre["launches"] == 2 and abs(pre["bytes_per_launch"] - 205e6) < 1
    assert att["launches"] == 1 and abs(att["bytes_per_launch"] - 150e6) < 1
    assert pre["source_hash"] == bench.kernel_source_hash("precompute")


def test_reference_arm_prints_its_line_on_cpu():
    """The reference arm is the oracle on the host's cores; it needs no GPU."""
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny-fp32",
                        "--steps", "1", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "queries/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["workload"] == "tiny-fp32"


def test_oracle_sample_is_bounded():
    """A small budget on the headline workload samples whole tiles of one
    sequence rather than the whole job."""
    smp = bench.OracleSampler(syn.WORKLOADS["max-64k"], 16)
    smp.plan(0.05)
    assert smp.n_heads == 1 and 1 <= smp.n_tiles < smp.ntiles
    rows, dt = smp.run()
    assert rows == smp.n_tiles * 128 and dt > 0
    assert "tiles of 128" in smp.describe()


def test_warmup_below_three_is_refused():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_traffic_hash_follows_each_path_sources(tmp_path, monkeypatch):
    """A stored traffic figure is tied to the sources its kernels are built
    from: editing the depth-L kernels leaves the tree path's figure valid and
    the reverse."""
    import shutil
    csrc = os.path.join(ROOT, "adaptive_vector_quantized_avq_b200", "csrc")
    fake = tmp_path / "repo"
    shutil.copytree(csrc, fake / "adaptive_vector_quantized_avq_b200" / "csrc")
    monkeypatch.setattr(bench, "ROOT", str(fake))
    tree0, deep0 = bench.kernel_source_hash("attention"), bench.kernel_source_hash("attention", True)
    assert tree0 != deep0
    with open(fake / "adaptive_vector_quantized_avq_b200" / "csrc" / "avq_deep.cu", "a") as f:
        f.write("\n// edit\n")
    assert bench.kernel_source_hash("attention") == tree0
    deep1 = bench.kernel_source_hash("attention", True)
    assert deep1 != deep0
    with open(fake / "adaptive_vector_quantized_avq_b200" / "csrc" / "avq_attention_tree.cu", "a") as f:
        f.write("\n// edit\n")
    assert bench.kernel_source_hash("attention") != tree0
    assert bench.kernel_source_hash("attention", True) == deep1


def test_kernel_names_are_kernels_of_the_sources():
    """Every name the ncu ingest matches is a kernel the sources define (a
    renamed kernel would otherwise drop out of the traffic record)."""
    import glob
    import re
    src = "".join(open(f).read() for f in glob.glob(os.path.join(bench.ROOT, "adaptive_vector_quantized_avq_b200",
                                                                  "csrc", "*.cu")))
    defined = set(re.findall(r"__global__[^;{]*?\b([a-z_0-9]+_kernel)\s*\(", src, flags=re.S))
    for kind, names in bench.KERNEL_NAMES.items():
        for n in names:
            assert n in defined, (kind, n, sorted(defined))
