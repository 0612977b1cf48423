"""Gated MLP (SwiGLU) on a B200 against the fp64 oracle: the fused gate/up
packing, the column-parallel GEMM with SiLU(gate) * up in its epilogue, and
tp_mlp_forward_swiglu ("Tensor Parallelism in Large Language Models",
"Partitioning the Multi-Layer Perceptron (MLP) Block", gated architectures).
"""
import numpy as np
import pytest

from oracle import tp_oracle as O
from tensor_transformer_layer_linear_b200 import synth

from helpers import assert_parity, f64, from_dev_bf16, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tp():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tensor_transformer_layer_linear_b200 import tp as _tp
    return _tp


def _bits(rng, shape, std=1.0):
    return synth.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))


def _pack(tp, Wg, Wu, n):
    h, F = Wg.shape
    W = np.ascontiguousarray(np.concatenate([Wg, Wu], axis=1))
    out = torch.empty(2 * h * F, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(to_dev(W), h, 2 * F, n, tp.TP_SPLIT_GATE_UP, 0, out)
    return out


@pytest.mark.parametrize("n", [1, 2, 4])
def test_gate_up_packing_bit_exact(tp, n):
    rng = np.random.default_rng(1000 + n)
    h, F = 200, n * 256
    Wg, Wu = _bits(rng, (h, F)), _bits(rng, (h, F))
    got = _pack(tp, Wg, Wu, n).cpu().numpy().view(np.uint16)
    assert np.array_equal(got.reshape(n, 2 * F // n, h), O.packed_gate_up(Wg, Wu, n))


@pytest.mark.parametrize("M", [64, 300])
@pytest.mark.parametrize("n", [1, 2, 4])
def test_column_swiglu(tp, n, M):
    rng = np.random.default_rng(1100 + n + M)
    h, F = 192, n * 384       # 3 gate/up blocks per shard
    X = _bits(rng, (M, h))
    Wg, Wu = _bits(rng, (h, F), 0.1), _bits(rng, (h, F), 0.1)
    Y = torch.empty((n, M, F // n), dtype=torch.int16, device="cuda")
    tp.tp_column_linear(to_dev(X), M, h, _pack(tp, Wg, Wu, n), None, 2 * F, n,
                        tp.TP_ACT_SWIGLU, Y)
    G = O.column_parallel_linear(f64(X), f64(Wg), None, n)
    U = O.column_parallel_linear(f64(X), f64(Wu), None, n)
    got = from_dev_bf16(Y)
    for i in range(n):
        assert_parity(got[i], O.silu(G[i]) * U[i], f"shard {i}")


def _run(tp, inp, cfg, n):
    M, h, F = cfg["batch"] * cfg["seq"], cfg["h"], cfg["ffn"]
    dev = {k: to_dev(v) for k, v in inp.items()}
    GU = _pack(tp, inp["Wg"], inp["Wu"], n)
    B_s = torch.empty(F * h, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(dev["B"], F, h, n, tp.TP_SPLIT_ROW, 0, B_s)
    nb = tp.tp_workspace_bytes(tp.TP_WS_MLP, M, h, F, n)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    Y = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_mlp_forward_swiglu(dev["X"], M, h, F, n, GU, B_s, dev["b2"],
                             dev["X"] if cfg.get("residual") else None, ws, nb, Y)
    assert tp.tp_get_last_error() == tp.TP_OK
    return from_dev_bf16(Y)


@pytest.mark.parametrize("n", [1, 2, 4])
def test_swiglu_mlp_small_all_elements(tp, n):
    cfg = dict(kind="swiglu", batch=2, seq=96, h=256, ffn=1024, x_std=1.0, w_std=0.05,
               b_std=0.05, residual=True)
    inp = synth.make_inputs(cfg, seed=5)
    ref = O.swiglu_mlp(f64(inp["X"]), f64(inp["Wg"]), f64(inp["Wu"]), f64(inp["B"]),
                       f64(inp["b2"]), f64(inp["X"]))
    assert_parity(_run(tp, inp, cfg, n), ref)


def test_swiglu_workload_sampled_rows(tp):
    cfg = synth.config("swiglu_8192x1024_f4096_n4")
    inp = synth.make_inputs(cfg)
    Y = _run(tp, inp, cfg, cfg["n_shards"])
    rows = synth.sample_rows(cfg["batch"], cfg["seq"])
    x = f64(inp["X"])
    ref = O.swiglu_mlp(x[rows], f64(inp["Wg"]), f64(inp["Wu"]), f64(inp["B"]), f64(inp["b2"]),
                       x[rows])
    assert_parity(Y[rows], ref)


def test_swiglu_rejects_unaligned_ffn(tp):
    X = torch.zeros(64 * 256, dtype=torch.int16, device="cuda")
    with pytest.raises(tp.TPError) as e:
        tp.tp_mlp_forward_swiglu(X, 64, 256, 4 * 96, 4, X, X, None, None, X, 1 << 20, X)
    assert e.value.status == tp.TP_ERR_SHAPE
