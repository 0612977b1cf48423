"""bench.py on the host: the reference arm (the fp64 oracle timed on the host
cores) prints one JSON line with the keys the harness reads, the warm-up
floor is enforced, and the per-step work accounting equals the FLOP counts
of the pages' formulas ("Tensor Parallelism in Large Language Models":
2 M K N per GEMM; causal attention 4 S^2 d per (sequence, head), halved)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from tensor_transformer_layer_linear_b200 import synth  # noqa: E402


def _run(*args):
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                          text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run("--impl", "reference", "--workload", "mlp_32x1024_f4096_n2", "--steps", "1",
             "--warmup", "3")
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "mlp_32x1024_f4096_n2"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]


def test_warmup_below_three_is_refused():
    r = _run("--impl", "reference", "--workload", "mlp_32x1024_f4096_n2", "--steps", "1",
             "--warmup", "2")
    assert r.returncode != 0
    assert not [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_layer_work_is_the_pages_flop_count():
    cfg = synth.config("layer_2x2048_h4096_32x128_f16384_n8")
    w = bench.work(cfg)
    b, s, h, F, heads = 2, 2048, 4096, 16384, 32
    M, d = b * s, h // heads
    qkv = 2 * M * h * (3 * h)
    up = 2 * M * h * F
    wo = 2 * M * h * h
    down = 2 * M * F * h
    attn = b * heads * 4 * s * s * d // 2
    assert w["flops"]["gemm_column_parallel"] == qkv + up
    assert w["flops"]["gemm_row_parallel"] == wo + down
    assert w["flops"]["attention"] == attn
    # the two reductions (the first fused with LN2) read the N fp32 partials
    n = 8
    assert w["bytes"]["reduce_partials"] == n * M * h * 4 + 2 * M * h * 2 + h * 2
    assert w["bytes"]["reduce_partials_layernorm"] == n * M * h * 4 + 3 * M * h * 2 + 3 * h * 2
    assert w["bytes"]["layernorm"] == 2 * M * h * 2 + 2 * h * 2            # LN1
    assert w["total_flops"] == qkv + up + wo + down + attn
    assert w["total_flops"] / 1e9 == pytest.approx(1717.99, abs=0.01)


def test_mlp_work_and_reduction_bytes():
    cfg = synth.config("mlp_8192x1024_f4096_n4")
    w = bench.work(cfg)
    M, h, F, n = 8192, 1024, 4096, 4
    assert w["total_flops"] == 2 * (2 * M * h * F)
    # the reduction reads N fp32 partials, the residual and the bias, writes Y
    expect = n * M * h * 4 + M * h * 2 + h * 2 + M * h * 2
    assert w["bytes"]["reduce_partials"] == expect


def test_layer_backward_counts_both_ln_backward_reductions():
    """The layer backward runs one LN-backward reduction per block (through
    LN2 for the MLP, through LN1 for attention): the per-step bytes are two
    launches' worth, each reading the N fp32 partials, the LN input and the
    residual gradient and writing the input gradient."""
    cfg = dict(synth.config("layer_2x2048_h4096_32x128_f16384_n8"), backward=True)
    w = bench.work(cfg)
    M, h, n = 2 * 2048, 4096, 8
    one = n * M * h * 4 + 3 * M * h * 2 + h * 2
    assert w["launch_bytes"]["reduce_partials_layernorm_backward"] == one
    assert w["bytes"]["reduce_partials_layernorm_backward"] == 2 * one
