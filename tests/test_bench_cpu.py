"""Host-side checks of bench.py: the CPU reference arm prints one well-formed JSON line."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.slow
def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "3", "--workload", "decode_128k", "--batch", "1"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "us/token" and d["higher_is_better"] is False
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_bench_help():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"], capture_output=True, text=True,
                       timeout=120, cwd=ROOT)
    assert r.returncode == 0 and "--impl" in r.stdout


@pytest.mark.slow
def test_reference_arm_prefill_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "3", "--workload", "prefill_32k"],
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "ms/chunk" and d["value"] > 0
    assert "prefill_32k" in d["config"]["workload"]


def test_local_pairs_matches_brute_force():
    # the local-head flop count of the prefill roofline: sum over chunk rows of |J_i|
    sys.path.insert(0, ROOT)
    import bench
    import synth

    for prefix, chunk, W, S in [(0, 300, 96, 4), (1000, 200, 128, 4), (400, 140, 1, 0), (400, 140, 64, 70),
                                (0, 50, 100000, 4)]:
        s = synth.spec("prefill_32k", prefix=prefix, chunk=chunk, window=W, n_sink=S)
        brute = 0
        for i in range(prefix, prefix + chunk):
            brute += sum(1 for j in range(i + 1) if i - j < W or j < S)
        assert bench._local_pairs(s) == brute


def test_profile_traffic_follows_the_kernel_source(tmp_path):
    # the committed ncu summary gives the select kernel's DRAM bytes only while the kernel
    # source still hashes to the value recorded beside them
    sys.path.insert(0, ROOT)
    import bench

    src = os.path.join(ROOT, "long_context_sparse_idx16_b200", "csrc", "decode_select.cu")
    text = open(os.path.join(ROOT, "profiles", "decode_select_128k.md")).read()
    rec = [ln for ln in text.splitlines() if ln.startswith("- dram bytes per launch")]
    assert len(rec) == 1
    want = float(rec[0].rsplit(":", 1)[1].split()[0])
    got = bench._profile_traffic(src)
    changed = tmp_path / "decode_select.cu"
    changed.write_bytes(open(src, "rb").read() + b"\n")
    assert bench._profile_traffic(str(changed)) is None
    import hashlib
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if ("- source sha256[:16]: " + h) in text:
        assert got == want
    else:
        assert got is None


def test_prefill_rooflines_per_kernel():
    sys.path.insert(0, ROOT)
    import bench

    flops = {"local_attention": 3.0e12, "retrieval_attention": 6.0e9, "index_scores": 2.0e9,
             "index_scores_flops": 6.4e10}
    kern = {"prefill_select": {"ms_per_launch": 10.0}, "prefill_attn": {"ms_per_launch": 5.0},
            "prefill_local": {"ms_per_launch": 6.0}, "q_prep": {"ms_per_launch": 99.0}}
    exp_peak = {"per_clk_per_sm": 16.0, "sms": 148, "sm_mhz": 1965.0}
    r = bench._prefill_rooflines(kern, flops, 2.0e9, exp_peak, 2000.0, 1650.0, "measured")
    # the selection: one exp per causal pair against the probe's rate at the sampled clock
    sel = r["prefill_select"]
    assert sel["bound"] == "alu" and sel["unit"] == "Gexp/s"
    assert abs(sel["achieved"] - 2.0e9 / 10e-3 / 1e9) < 1e-9
    assert abs(sel["peak"] - 16 * 148 * 2000.0e6 / 1e9) < 1e-9
    assert abs(sel["frac"] - sel["achieved"] / sel["peak"]) < 1e-12
    # the attention kernels: tensor rooflines with their algorithmic flops
    assert r["prefill_local"]["bound"] == "tensor" and r["prefill_local"]["peak"] == 1650.0
    assert abs(r["prefill_local"]["achieved"] - 3.0e12 / 6e-3 / 1e12) < 1e-9
    assert abs(r["prefill_attn"]["achieved"] - 6.0e9 / 5e-3 / 1e12) < 1e-9
    # the retrieval heads' two kernels together against the tensor peak
    agg = r["index_plus_sparse_attention"]
    assert abs(agg["achieved"] - (6.4e10 + 6.0e9) / 15e-3 / 1e12) < 1e-9
    # without a sampled clock the probe's own clock is used
    r = bench._prefill_rooflines(kern, flops, 2.0e9, exp_peak, None, 1650.0, "measured")
    assert abs(r["prefill_select"]["peak"] - 16 * 148 * 1965.0e6 / 1e9) < 1e-9


def test_prefill_traffic_only_for_the_captured_kernel_and_chunk():
    sys.path.insert(0, ROOT)
    import bench

    # the figures of the committed summary, or None once the kernel sources change
    t = bench._prefill_traffic("prefill_select", "prefill_32k")
    assert t is None or t == 623752704.0
    t = bench._prefill_traffic("prefill_attn", "prefill_32k")
    assert t is None or t == 245485056.0
    t = bench._prefill_traffic("prefill_select", "prefill_1m")
    assert t is None or t == 61888269824.0
    assert bench._prefill_traffic("prefill_select", "decode_1m") is None
    assert bench._prefill_traffic("prefill_local", "prefill_32k") is None
