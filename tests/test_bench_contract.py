"""bench.py on the CPU: the algorithmic-byte count behind the roofline line, and
the reference arm's JSON line (the fp64 oracle timed on the host cores)."""
import json
import os
import subprocess
import sys

import numpy as np

import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def test_algorithmic_bytes_of_the_decode_workload():
    """Each distinct adapter once (r (d_in + d_out) bf16 values), X in bf16, Y
    fp32 read and written: 16 distinct rank-16 adapters and 64 tokens at d = 4096."""
    bench = _bench()
    wl = W.decode_q_proj_7b()
    distinct = len(set(int(i) for i in wl.ids if i >= 0))
    assert distinct == 16
    assert bench.algorithmic_bytes(wl) == distinct * 16 * (4096 + 4096) * 2 + 64 * (4096 * 2 + 4096 * 4 * 2)
    assert bench.algorithmic_bytes(wl) == 6_815_744


def test_algorithmic_bytes_skip_tokens_without_an_adapter():
    bench = _bench()
    wl = W.random_small(seed=5, T=40, d_in=64, d_out=32, S=6, ranks=(4, 8), p_none=0.3, p_empty=0.4)
    rk = wl.ranks()
    ok = [int(i) for i in wl.ids if 0 <= i < wl.S and rk[i] > 0]
    want = sum(2 * int(rk[i]) * (64 + 32) for i in set(ok)) + len(ok) * (2 * 64 + 8 * 32)
    assert bench.algorithmic_bytes(wl) == want
    assert bench.algorithmic_flops(wl) == sum(2 * int(rk[i]) * (64 + 32) for i in ok)


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "1"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == "LoRA-branch tokens/s per layer" and line["unit"] == "tokens/s"
    assert line["value"] > 0 and line["higher_is_better"] is True and line["steps"] == 2
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    bench = _bench()
    wl, desc = bench.workload_spec("sweep_8b_distinct_T1024")
    assert line["config"] == bench.bench_config(wl, desc)      # the GPU arm prints the same object
    assert line["config"]["workload"].startswith("8B sweep distinct")


def test_source_digest_ignores_comments(tmp_path):
    """A profile's traffic stays valid across comment-only edits of the kernel source
    and is dropped when the code changes."""
    bench = _bench()
    a, b, c = tmp_path / "a.cu", tmp_path / "b.cu", tmp_path / "c.cu"
    a.write_text("// head\nint f(int x) {  // tail\n  return x + 1;\n}\n")
    b.write_text("/* another\n   block */\nint f(int x) {\n\n  return x + 1;   \n}\n")
    c.write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.source_digest(str(a)) == bench.source_digest(str(b)) != bench.source_digest(str(c))


def test_profiled_traffic_matches_only_the_captured_code():
    bench = _bench()
    for wl_name, prof in bench.PROFILE_FOR.items():
        f = bench.profile_fields(prof)
        assert f["source"].endswith(".cu") and len(f["source_digest"]) == 64 and int(f["traffic_bytes_per_launch"]) > 0
        same = bench.source_digest(os.path.join(ROOT, f["source"])) == f["source_digest"]
        assert (bench.profiled_traffic(wl_name) is not None) == same
