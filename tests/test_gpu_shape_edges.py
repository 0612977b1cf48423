"""Parity at the shapes where the kernels switch variants, on a B200.

* The small layer that ``__graft_entry__.smoke()`` runs (1 x 128 tokens,
  h 256, 2 heads of 128, F 1024, N 2), once through ``smoke()`` itself and
  once stage by stage through the C ABI, each stage fed the GPU's own output
  of the stage before, so a wrong stage is named by the first failing check.
* Every GEMM variant the launcher can pick for the forward projections:
  single-CTA tiles (M <= 128) 128 or 256 columns wide, with a half-empty last
  column tile, fp32 partials stored directly (K <= 256) or through TMA
  (K > 256), and CTA pairs (M > 128). Integer-valued inputs make every
  product and sum exact in fp32, so the results are held bit for bit to the
  fp64 oracle (bf16 outputs: to its round-to-nearest-even bf16 value).
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


def _int_bits(rng, shape, lo, hi):
    return synth.f32_to_bf16_bits(rng.integers(lo, hi + 1, size=shape).astype(np.float32))


def _shard(tp, W_dev, h_in, h_out, kind, n, head_dim=0):
    out = torch.empty(h_in * h_out, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(W_dev, h_in, h_out, n, kind, head_dim, out)
    return out


def _bits(t):
    return t.cpu().numpy().view(np.uint16)


def _bf16_of(x):
    """fp64 values (exact in fp32) -> their bf16 bit patterns (RNE)."""
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


# ------------------------------------------------------------------ smoke()

def test_smoke_entry_point():
    import __graft_entry__
    __graft_entry__.smoke()


SMOKE = dict(kind="layer", batch=1, seq=128, h=256, n_heads=2, ffn=1024, x_std=1.0,
             w_std=0.05, b_std=0.05, ln_eps=1e-5)


def test_layer_stages_at_smoke_shape(tp):
    cfg, n, eps = SMOKE, 2, 1e-5
    b, s, h, nh, F = cfg["batch"], cfg["seq"], cfg["h"], cfg["n_heads"], cfg["ffn"]
    M, d, hs = b * s, h // nh, h // n
    inp = synth.make_inputs(cfg, seed=7)
    dev = {k: to_dev(v) for k, v in inp.items()}
    p = {k: f64(v) for k, v in inp.items()}
    Wqkv_s = _shard(tp, dev["Wqkv"], h, 3 * h, tp.TP_SPLIT_QKV_HEADS, n, d)
    bqkv_s = _shard(tp, dev["bqkv"], 1, 3 * h, tp.TP_SPLIT_QKV_HEADS, n, d)
    Wo_s = _shard(tp, dev["Wo"], h, h, tp.TP_SPLIT_ROW, n)
    A_s = _shard(tp, dev["A"], h, F, tp.TP_SPLIT_COLUMN, n)
    B_s = _shard(tp, dev["B"], F, h, tp.TP_SPLIT_ROW, n)

    # LN1
    x1 = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_layernorm(dev["X"], M, h, dev["ln1_g"], dev["ln1_b"], eps, x1)
    x1_g = from_dev_bf16(x1)
    assert_parity(x1_g, O.layernorm(p["X"], p["ln1_g"], p["ln1_b"], eps), "LN1")
    # QKV column GEMM (384 columns per shard: one full and one half 256-wide tile)
    qkv = torch.empty((n, M, 3 * hs), dtype=torch.int16, device="cuda")
    tp.tp_column_linear(x1, M, h, Wqkv_s, bqkv_s, 3 * h, n, tp.TP_ACT_NONE, qkv)
    qkv_g = from_dev_bf16(qkv)
    ref = O.column_parallel_linear(x1_g, p["Wqkv"], p["bqkv"], n, kind=O.SPLIT_QKV_HEADS,
                                   head_dim=d)
    for i in range(n):
        assert_parity(qkv_g[i], ref[i], f"QKV shard {i}")
    # attention (one 128-query tile per sequence)
    o = torch.empty((n, M, hs), dtype=torch.int16, device="cuda")
    tp.tp_attention(qkv, b, s, h, nh, 1, n, o)
    o_g = from_dev_bf16(o)
    for i in range(n):
        q = qkv_g[i]
        ref = O.attention_heads(q[:, :hs], q[:, hs:2 * hs], q[:, 2 * hs:], b, s, nh // n, True)
        assert_parity(o_g[i], ref, f"attention shard {i}")
    # W_O row GEMM (K = h / N = 128: fp32 partials stored directly)
    part = torch.empty((n, M, h), dtype=torch.float32, device="cuda")
    tp.tp_row_linear(o, M, h, Wo_s, h, n, part)
    part_g = part.cpu().numpy().astype(np.float64)
    ref = O.row_parallel_linear(list(o_g), p["Wo"], n)
    for i in range(n):
        assert_parity(part_g[i], ref[i], f"W_O partial {i}")
    # sum of the partials + b_O + X, then LN2
    h1 = torch.empty((M, h), dtype=torch.int16, device="cuda")
    x2 = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_reduce_partials_layernorm(part, n, M, h, dev["bo"], dev["X"], dev["ln2_g"],
                                    dev["ln2_b"], eps, h1, x2)
    h1_g, x2_g = from_dev_bf16(h1), from_dev_bf16(x2)
    assert_parity(h1_g, O.reduce_partials(list(part_g), p["bo"], p["X"]), "h1")
    assert_parity(x2_g, O.layernorm(h1_g, p["ln2_g"], p["ln2_b"], eps), "LN2")
    # MLP column GEMM + bias + GeLU (512 columns per shard)
    a = torch.empty((n, M, F // n), dtype=torch.int16, device="cuda")
    tp.tp_column_linear(x2, M, h, A_s, dev["b1"], F, n, tp.TP_ACT_GELU_ERF, a)
    a_g = from_dev_bf16(a)
    ref = O.column_parallel_linear(x2_g, p["A"], p["b1"], n, act=O.gelu)
    for i in range(n):
        assert_parity(a_g[i], ref[i], f"GeLU(x2 A_i + b1_i) shard {i}")
    # MLP row GEMM (K = 512: fp32 partials through TMA stores)
    tp.tp_row_linear(a, M, F, B_s, h, n, part)
    part_g = part.cpu().numpy().astype(np.float64)
    ref = O.row_parallel_linear(list(a_g), p["B"], n)
    for i in range(n):
        assert_parity(part_g[i], ref[i], f"B partial {i}")
    # final sum + b2 + h1
    Y = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_reduce_partials(part, n, M, h, dev["b2"], h1, Y)
    Y_g = from_dev_bf16(Y)
    assert_parity(Y_g, O.reduce_partials(list(part_g), p["b2"], h1_g), "Y")
    # and the chain as a whole against the unsharded layer
    ref = O.transformer_layer(p["X"], p, b, s, nh, eps)
    assert_parity(Y_g, ref, "layer")
    assert tp.tp_get_last_error() == tp.TP_OK


@pytest.mark.parametrize("n", [1, 2])
def test_layer_and_mlp_at_smoke_shape(tp, n):
    """tp_layer_forward and tp_mlp_forward, whole, at the smoke shape."""
    from test_gpu_blocks import layer_ref, mlp_ref, run_layer, run_mlp
    inp = synth.make_inputs(SMOKE, seed=7)
    assert_parity(from_dev_bf16(run_layer(tp, inp, SMOKE, n)), layer_ref(inp, SMOKE), "layer")
    cfg = dict(kind="mlp", batch=1, seq=128, h=256, ffn=1024, x_std=1.0, w_std=0.05,
               b_std=0.05, residual=True)
    inp = synth.make_inputs(cfg, seed=8)
    assert_parity(from_dev_bf16(run_mlp(tp, inp, cfg, n)), mlp_ref(inp, cfg), "mlp")


# ------------------------------------------------------------------ every GEMM variant

@pytest.mark.parametrize("M", [1, 32, 64, 128, 129, 256])
@pytest.mark.parametrize("K", [64, 128, 256, 512])
@pytest.mark.parametrize("nc", [128, 256, 384])
def test_column_linear_variants_bit_exact(tp, M, K, nc):
    n = 2
    rng = np.random.default_rng(1000 + M + 7 * K + nc)
    X = _int_bits(rng, (M, K), -1, 1)
    W = _int_bits(rng, (K, n * nc), -1, 1)
    bias = _int_bits(rng, (n * nc,), -2, 2)
    Y = torch.empty((n, M, nc), dtype=torch.int16, device="cuda")
    tp.tp_column_linear(to_dev(X), M, K, _shard(tp, to_dev(W), K, n * nc, 0, n), to_dev(bias),
                        n * nc, n, tp.TP_ACT_NONE, Y)
    ref = O.column_parallel_linear(f64(X), f64(W), f64(bias), n)
    got = _bits(Y)
    for i in range(n):
        assert np.array_equal(got[i], _bf16_of(ref[i])), f"shard {i}"


@pytest.mark.parametrize("M", [1, 32, 64, 128, 129, 256])
@pytest.mark.parametrize("k_loc", [64, 128, 256, 512])
@pytest.mark.parametrize("h_out", [128, 256, 384])
def test_row_linear_variants_bit_exact(tp, M, k_loc, h_out):
    n = 2
    rng = np.random.default_rng(2000 + M + 7 * k_loc + h_out)
    X = _int_bits(rng, (M, n * k_loc), -8, 8)
    W = _int_bits(rng, (n * k_loc, h_out), -8, 8)
    Xs = np.ascontiguousarray(np.stack(O.split_columns(X, n)))
    P = torch.empty((n, M, h_out), dtype=torch.float32, device="cuda")
    tp.tp_row_linear(to_dev(Xs), M, n * k_loc, _shard(tp, to_dev(W), n * k_loc, h_out, 1, n),
                     h_out, n, P)
    ref = O.row_parallel_linear(O.split_columns(f64(X), n), f64(W), n)
    got = P.cpu().numpy().astype(np.float64)
    for i in range(n):
        assert np.array_equal(got[i], ref[i]), f"shard {i}"


@pytest.mark.parametrize("M", [64, 128])
def test_column_linear_gelu_small_m_random(tp, M):
    """Random values through the bias + GeLU epilogue of the single-CTA,
    256-wide tiles, with a half-empty last tile (384 columns per shard)."""
    n, K, nc = 2, 256, 384
    rng = np.random.default_rng(3000 + M)
    X = synth.f32_to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32))
    W = synth.f32_to_bf16_bits(rng.standard_normal((K, n * nc), dtype=np.float32) * 0.05)
    bias = synth.f32_to_bf16_bits(rng.standard_normal(n * nc, dtype=np.float32) * 0.1)
    Y = torch.empty((n, M, nc), dtype=torch.int16, device="cuda")
    tp.tp_column_linear(to_dev(X), M, K, _shard(tp, to_dev(W), K, n * nc, 0, n), to_dev(bias),
                        n * nc, n, tp.TP_ACT_GELU_ERF, Y)
    ref = O.column_parallel_linear(f64(X), f64(W), f64(bias), n, act=O.gelu)
    got = from_dev_bf16(Y)
    for i in range(n):
        assert_parity(got[i], ref[i], f"shard {i}")
