"""The bench's oracle timing and its reference arm, on the host (no GPU).

`bench.py --impl reference` times the fp64 oracle on the host cores and prints
the same JSON line as the device arm; the default bench line carries the same
timing as `cpu_baseline`. The rate is the per-token slope of two oracle calls;
where the per-call fixed cost swamps the per-token one (a small vocabulary, a
cold first call) the two times may not order, and the rate must then fall back
to a whole-call time rather than divide by a clamped difference.
"""
import json
import math
import os
import subprocess
import sys
from types import SimpleNamespace

import bench
from chunked_kl_loss_logits_b200.workloads import small_case

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_oracle_rate_is_positive_and_finite_without_warmup():
    x = small_case(256, 32, 500, 8, seed=3, dtype="bf16")
    rates, fixed, rows, cores = bench.oracle_rate(x, SimpleNamespace(T=256), steps=2, warmup=0)
    assert rows == bench.ORACLE_ROWS and cores >= 1 and len(rates) == len(fixed) == 2
    # a token's fwd+bwd over V = 500, d = 32 is a few hundred kFLOP: far below 1e7 tokens/s
    assert all(0.0 < r < 1e7 and math.isfinite(r) for r in rates)


def test_sample_text_names_whole_call_steps():
    text = bench.oracle_sample_text((64, 192), 2, [0.1, float("nan")])
    assert "fixed cost 0.10 s excluded" in text and "1 step(s)" in text and "whole time" in text
    assert "excluded" not in bench.oracle_sample_text((64, 192), 1, [float("nan")])


def test_reference_arm_json_line():
    out = subprocess.run(
        [sys.executable, "bench.py", "--impl", "reference", "--workload", "bf16_4k", "--steps", "1",
         "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["dtype"] == "f64"
    assert 0.0 < d["value"] < 1e6 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "bf16_4k" and d["n_gpus"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_kernel_hash_ignores_comments_and_layout():
    # the recorded DRAM traffic is keyed to the kernels' code, not to their comments
    assert bench.code_text("int a; // note\n/* block\n comment */  int  b;\n") == "int a; int b;"
    assert bench.code_text('asm("ex2.approx.f32 %0, %1;");') == 'asm("ex2.approx.f32 %0, %1;");'
