"""Block-level parity on a B200: tp_mlp_forward, tp_attn_forward and
tp_layer_forward against the fp64 oracle of the UNSHARDED blocks.

Small cases are compared element by element on every output; the five
workloads are run at full size in the same launch configuration the
benchmark uses and compared on a deterministic sample of token rows (every
64th row of each sequence plus its first and last). The output must not
depend on the shard count N beyond the tolerance.
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


def _shard(tp, W_bits_dev, h_in, h_out, kind, n, head_dim=0):
    out = torch.empty(h_in * h_out, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(W_bits_dev, h_in, h_out, n, kind, head_dim, out)
    return out


def _ws(tp, kind, M, h, F, n):
    nbytes = tp.tp_workspace_bytes(kind, M, h, F, n)
    return torch.empty(nbytes, dtype=torch.uint8, device="cuda"), nbytes


def run_mlp(tp, inp, cfg, n, dev=None):
    """Run tp_mlp_forward on device copies of the inputs; returns Y (device)."""
    M, h, F = cfg["batch"] * cfg["seq"], cfg["h"], cfg["ffn"]
    dev = dev if dev is not None else {k: to_dev(v) for k, v in inp.items()}
    A_s = _shard(tp, dev["A"], h, F, 0, n)
    B_s = _shard(tp, dev["B"], F, h, 1, n)
    ws, nb = _ws(tp, tp.TP_WS_MLP, M, h, F, n)
    Y = torch.empty((M, h), dtype=torch.int16, device="cuda")
    R = dev["X"] if cfg.get("residual") else None
    tp.tp_mlp_forward(dev["X"], M, h, F, n, A_s, dev["b1"], B_s, dev["b2"], R, ws, nb, Y)
    assert tp.tp_get_last_error() == tp.TP_OK
    return Y


def mlp_ref(inp, cfg, rows=None):
    x = f64(inp["X"])
    R = x if cfg.get("residual") else None
    args = (f64(inp["A"]), f64(inp["b1"]), f64(inp["B"]), f64(inp["b2"]))
    if rows is None:
        return O.mlp(x, *args, R)
    return O.mlp_rows(x, *args, R, rows)


def run_attn(tp, inp, cfg, n):
    b, s, h, nh = cfg["batch"], cfg["seq"], cfg["h"], cfg["n_heads"]
    M = b * s
    dev = {k: to_dev(v) for k, v in inp.items()}
    Wqkv_s = _shard(tp, dev["Wqkv"], h, 3 * h, 2, n, h // nh)
    bqkv_s = _shard(tp, dev["bqkv"], 1, 3 * h, 2, n, h // nh)
    Wo_s = _shard(tp, dev["Wo"], h, h, 1, n)
    ws, nb = _ws(tp, tp.TP_WS_ATTN, M, h, 0, n)
    Y = torch.empty((M, h), dtype=torch.int16, device="cuda")
    R = dev["X"] if cfg.get("residual") else None
    tp.tp_attn_forward(dev["X"], b, s, h, nh, cfg.get("causal", True), n, Wqkv_s, bqkv_s, Wo_s,
                       dev["bo"], R, ws, nb, Y)
    assert tp.tp_get_last_error() == tp.TP_OK
    return Y


def attn_ref(inp, cfg, rows=None):
    x = f64(inp["X"])
    R = x if cfg.get("residual") else None
    a = (f64(inp["Wqkv"]), f64(inp["bqkv"]), f64(inp["Wo"]), f64(inp["bo"]), R,
         cfg["batch"], cfg["seq"], cfg["n_heads"])
    if rows is None:
        return O.self_attention(x, *a, cfg.get("causal", True))
    return O.self_attention_rows(x, *a, rows, cfg.get("causal", True))


def run_layer(tp, inp, cfg, n):
    b, s, h, nh, F = cfg["batch"], cfg["seq"], cfg["h"], cfg["n_heads"], cfg["ffn"]
    M = b * s
    d = h // nh
    dev = {k: to_dev(v) for k, v in inp.items()}
    keep = dict(
        ln1_gamma=dev["ln1_g"], ln1_beta=dev["ln1_b"],
        Wqkv_shards=_shard(tp, dev["Wqkv"], h, 3 * h, 2, n, d),
        bqkv_shards=_shard(tp, dev["bqkv"], 1, 3 * h, 2, n, d),
        Wo_shards=_shard(tp, dev["Wo"], h, h, 1, n), bo=dev["bo"],
        ln2_gamma=dev["ln2_g"], ln2_beta=dev["ln2_b"],
        A_shards=_shard(tp, dev["A"], h, F, 0, n), b1_shards=dev["b1"],
        B_shards=_shard(tp, dev["B"], F, h, 1, n), b2=dev["b2"])
    w = tp.make_layer_weights(**keep)
    ws, nb = _ws(tp, tp.TP_WS_LAYER, M, h, F, n)
    Y = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_layer_forward(dev["X"], b, s, h, nh, F, n, w, cfg.get("ln_eps", 1e-5), ws, nb, Y)
    assert tp.tp_get_last_error() == tp.TP_OK
    return Y


def layer_params(inp):
    return {k: f64(v) for k, v in inp.items() if k != "X"}


def layer_ref(inp, cfg, rows=None):
    x = f64(inp["X"])
    p = layer_params(inp)
    if rows is None:
        return O.transformer_layer(x, p, cfg["batch"], cfg["seq"], cfg["n_heads"],
                                   cfg.get("ln_eps", 1e-5))
    return O.transformer_layer_rows(x, p, cfg["batch"], cfg["seq"], cfg["n_heads"], rows,
                                    cfg.get("ln_eps", 1e-5))


# ------------------------------------------------------------------ small, every element

@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_mlp_small_all_elements(tp, n):
    cfg = dict(kind="mlp", batch=2, seq=80, h=256, ffn=1024, x_std=1.0, w_std=0.05, b_std=0.05,
               residual=True)
    inp = synth.make_inputs(cfg, seed=1)
    assert_parity(from_dev_bf16(run_mlp(tp, inp, cfg, n)), mlp_ref(inp, cfg))


@pytest.mark.parametrize("n", [1, 2, 4])
def test_attn_small_all_elements(tp, n):
    cfg = dict(kind="attn", batch=2, seq=192, h=512, n_heads=4, causal=True, x_std=1.0,
               w_std=0.05, b_std=0.05, residual=True)
    inp = synth.make_inputs(cfg, seed=2)
    assert_parity(from_dev_bf16(run_attn(tp, inp, cfg, n)), attn_ref(inp, cfg))


@pytest.mark.parametrize("n", [1, 2, 4])
def test_layer_small_all_elements(tp, n):
    cfg = dict(kind="layer", batch=2, seq=160, h=512, n_heads=4, ffn=2048, x_std=1.0,
               w_std=0.05, b_std=0.05, ln_eps=1e-5)
    inp = synth.make_inputs(cfg, seed=3)
    assert_parity(from_dev_bf16(run_layer(tp, inp, cfg, n)), layer_ref(inp, cfg))


# ------------------------------------------------------------------ the five workloads

def test_workload_mlp_32x1024_n2(tp):
    cfg = synth.config("mlp_32x1024_f4096_n2")
    inp = synth.make_inputs(cfg)
    assert_parity(from_dev_bf16(run_mlp(tp, inp, cfg, cfg["n_shards"])), mlp_ref(inp, cfg))


def test_workload_mlp_8192x1024_n4(tp):
    cfg = synth.config("mlp_8192x1024_f4096_n4")
    inp = synth.make_inputs(cfg)
    rows = synth.sample_rows(cfg["batch"], cfg["seq"])
    Y = from_dev_bf16(run_mlp(tp, inp, cfg, cfg["n_shards"]))
    assert_parity(Y[rows], mlp_ref(inp, cfg, rows))


def test_workload_attn_4x2048_n8(tp):
    cfg = synth.config("attn_4x2048_h2048_16x128_n8")
    inp = synth.make_inputs(cfg)
    rows = synth.sample_rows(cfg["batch"], cfg["seq"])
    Y = from_dev_bf16(run_attn(tp, inp, cfg, cfg["n_shards"]))
    assert_parity(Y[rows], attn_ref(inp, cfg, rows))


@pytest.fixture(scope="module")
def layer_workload():
    cfg = synth.config("layer_2x2048_h4096_32x128_f16384_n8")
    inp = synth.make_inputs(cfg)
    rows = synth.sample_rows(cfg["batch"], cfg["seq"])
    return cfg, inp, rows, layer_ref(inp, cfg, rows), {}


@pytest.mark.parametrize("n", [8, 16])
def test_workload_layer_2x2048(tp, layer_workload, n):
    """The full layer workload at its own shard count (8) and at 16 (two of
    the 32 heads per shard), on sampled rows; the two outputs agree on every
    element."""
    cfg, inp, rows, ref, outs = layer_workload
    Y = from_dev_bf16(run_layer(tp, inp, cfg, n))
    torch.cuda.empty_cache()
    assert_parity(Y[rows], ref, f"N={n}")
    outs[n] = Y
    if n != 8 and 8 in outs:
        assert_parity(Y, outs[8], f"N={n} vs N=8")


@pytest.fixture(scope="module")
def layer_sweep():
    cfg = dict(kind="layer", batch=2, seq=192, h=2048, n_heads=16, ffn=8192, x_std=1.0,
               w_std=0.02, b_std=0.01, ln_eps=1e-5)
    inp = synth.make_inputs(cfg, seed=4)
    return cfg, inp, layer_ref(inp, cfg), {}


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_layer_shard_sweep_all_elements(tp, layer_sweep, n):
    """A 16-head layer (h 2048, F 8192, 2 x 192 tokens: a ragged last query
    tile) at every shard count the heads allow up to 16, every element
    against the unsharded oracle and against the N = 1 output."""
    cfg, inp, ref, outs = layer_sweep
    Y = from_dev_bf16(run_layer(tp, inp, cfg, n))
    assert_parity(Y, ref, f"N={n}")
    outs[n] = Y
    if n != 1 and 1 in outs:
        assert_parity(Y, outs[1], f"N={n} vs N=1")


@pytest.fixture(scope="module")
def sweep():
    cfg = synth.config("mlp_2048x12288_f49152_sweep")
    inp = synth.make_inputs(cfg)
    rows = synth.sample_rows(cfg["batch"], cfg["seq"])
    return cfg, inp, rows, mlp_ref(inp, cfg, rows), {}


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_workload_mlp_sweep(tp, sweep, n):
    cfg, inp, rows, ref, outs = sweep
    dev = {k: to_dev(v) for k, v in inp.items()}
    Y = from_dev_bf16(run_mlp(tp, inp, cfg, n, dev))
    del dev
    torch.cuda.empty_cache()
    assert_parity(Y[rows], ref, f"N={n}")
    outs[n] = Y
    if n != 1 and 1 in outs:   # invariance to the shard count, on every element
        assert_parity(Y, outs[1], f"N={n} vs N=1")


# ------------------------------------------------------------------ errors on the device

def test_block_errors(tp):
    cfg = dict(kind="mlp", batch=1, seq=64, h=256, ffn=1024, x_std=1.0, w_std=0.05, b_std=0.0)
    inp = synth.make_inputs(cfg)
    dev = {k: to_dev(v) for k, v in inp.items()}
    ws, nb = _ws(tp, tp.TP_WS_MLP, 64, 256, 1024, 4)
    Y = torch.empty((64, 256), dtype=torch.int16, device="cuda")
    with pytest.raises(tp.TPError) as e:
        tp.tp_mlp_forward(dev["X"], 64, 256, 1024, 4, dev["A"], None, dev["B"], None, None, ws,
                          nb - 1, Y)
    assert e.value.status == tp.TP_ERR_WORKSPACE
    with pytest.raises(tp.TPError) as e:
        tp.tp_mlp_forward(dev["X"], 64, 256, 1000, 4, dev["A"], None, dev["B"], None, None, ws,
                          nb, Y)
    assert e.value.status == tp.TP_ERR_SHAPE
    with pytest.raises(tp.TPError) as e:
        tp.tp_attn_forward(dev["X"], 1, 64, 256, 4, 1, 4, dev["A"], None, dev["B"], None, None,
                           ws, nb, Y)   # head_dim 64
    assert e.value.status == tp.TP_ERR_UNSUPPORTED
    assert tp.tp_get_last_error() == tp.TP_OK
