"""Sequence parallelism on a B200: reduce-scatter of the partials, all-gather
along the sequence, and the sequence-parallel layer, against the fp64 oracle
("Tensor Parallelism in Large Language Models", "Sequence Parallelism").
"""
import numpy as np
import pytest

from oracle import tp_oracle as O
from tensor_transformer_layer_linear_b200 import synth

from helpers import assert_parity, f64, from_dev_bf16, to_dev
from test_gpu_blocks import _shard, _ws, layer_params

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tp():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tensor_transformer_layer_linear_b200 import tp as _tp
    return _tp


def _bits(rng, shape, std=1.0):
    return synth.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))


def _to_slices(bits, batch, seq, n):
    """token-ordered rows -> stacked sequence slices [N][b][S/N][h] (bits)."""
    h = bits.shape[-1]
    return np.ascontiguousarray(
        np.stack(O.sequence_shard(bits.reshape(batch * seq, h), batch, seq, n)))


@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_reduce_scatter_partials(tp, n):
    rng = np.random.default_rng(900 + n)
    batch, seq, h = 3, 64, 264
    M = batch * seq
    P = rng.standard_normal((n, M, h)).astype(np.float32)
    b = _bits(rng, (h,), 0.5)
    R = _bits(rng, (M, h))
    Rs = _to_slices(R, batch, seq, n)
    Y = torch.empty((n, batch, seq // n, h), dtype=torch.int16, device="cuda")
    tp.tp_reduce_scatter_partials(torch.from_numpy(P).cuda(), n, batch, seq, h, to_dev(b),
                                  to_dev(Rs), Y)
    ref = O.reduce_scatter_partials(list(P.astype(np.float64)), batch, seq, n, f64(b),
                                    [f64(r) for r in Rs])
    got = from_dev_bf16(Y)
    for i in range(n):
        assert_parity(got[i], ref[i], f"slice {i}")
    # integer partials: exact, and the all-gather of the slices is the all-reduce
    Pi = rng.integers(-16, 17, size=(n, M, h)).astype(np.float32)
    Yi = torch.empty((n, batch, seq // n, h), dtype=torch.int16, device="cuda")
    tp.tp_reduce_scatter_partials(torch.from_numpy(Pi).cuda(), n, batch, seq, h, None, None, Yi)
    Xg = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_all_gather_sequence(Yi, n, batch, seq, h, Xg)
    assert np.array_equal(from_dev_bf16(Xg), O.reduce_partials(list(Pi.astype(np.float64))))


@pytest.mark.parametrize("n", [1, 2, 4, 16])
def test_all_gather_sequence_bit_exact(tp, n):
    rng = np.random.default_rng(950 + n)
    batch, seq, h = 2, 128, 136
    Xs = _bits(rng, (n, batch, seq // n, h))
    X = torch.empty((batch * seq, h), dtype=torch.int16, device="cuda")
    tp.tp_all_gather_sequence(to_dev(Xs), n, batch, seq, h, X)
    ref = O.all_gather_sequence(list(Xs), batch, seq)
    assert np.array_equal(X.cpu().numpy().view(np.uint16), ref)


def test_sequence_parallel_errors(tp):
    X = torch.zeros(64 * 128, dtype=torch.int16, device="cuda")
    with pytest.raises(tp.TPError) as e:
        tp.tp_all_gather_sequence(X, 3, 1, 64, 128, X)   # 64 % 3 != 0
    assert e.value.status == tp.TP_ERR_SHAPE


def _layer_weights(tp, inp, cfg, n):
    h, nh, F = cfg["h"], cfg["n_heads"], cfg["ffn"]
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
    return tp.make_layer_weights(**keep), keep, dev


def _run_both(tp, inp, cfg, n):
    b, s, h, nh, F = cfg["batch"], cfg["seq"], cfg["h"], cfg["n_heads"], cfg["ffn"]
    M = b * s
    w, keep, dev = _layer_weights(tp, inp, cfg, n)
    ws, nb = _ws(tp, tp.TP_WS_LAYER_SP, M, h, F, n)
    Xs = to_dev(_to_slices(inp["X"], b, s, n))
    Ys = torch.empty((n, b, s // n, h), dtype=torch.int16, device="cuda")
    tp.tp_layer_forward_sp(Xs, b, s, h, nh, F, n, w, cfg.get("ln_eps", 1e-5), ws, nb, Ys)
    Y = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_layer_forward(dev["X"], b, s, h, nh, F, n, w, cfg.get("ln_eps", 1e-5), ws, nb, Y)
    assert tp.tp_get_last_error() == tp.TP_OK
    return Ys, Y


@pytest.mark.parametrize("n", [1, 2, 4])
def test_sequence_parallel_layer_small(tp, n):
    cfg = dict(kind="layer", batch=2, seq=160, h=512, n_heads=4, ffn=2048, x_std=1.0,
               w_std=0.05, b_std=0.05, ln_eps=1e-5)
    inp = synth.make_inputs(cfg, seed=4)
    Ys, Y = _run_both(tp, inp, cfg, n)
    got = from_dev_bf16(Ys)
    p = layer_params(inp)
    X_sl = O.sequence_shard(f64(inp["X"]), cfg["batch"], cfg["seq"], n)
    ref = O.transformer_layer_sp(X_sl, p, cfg["batch"], cfg["seq"], cfg["n_heads"], n)
    for i in range(n):
        assert_parity(got[i], ref[i], f"slice {i}")
    # same kernels, permuted rows: bit-identical to the standard layer
    gathered = O.all_gather_sequence(list(Ys.cpu().numpy().view(np.uint16)), cfg["batch"],
                                     cfg["seq"])
    assert np.array_equal(gathered, Y.cpu().numpy().view(np.uint16))


def test_sequence_parallel_layer_workload(tp):
    cfg = synth.config("layer_2x2048_h4096_32x128_f16384_n8")
    inp = synth.make_inputs(cfg)
    n = cfg["n_shards"]
    Ys, Y = _run_both(tp, inp, cfg, n)
    gathered = O.all_gather_sequence(list(Ys.cpu().numpy().view(np.uint16)), cfg["batch"],
                                     cfg["seq"])
    assert np.array_equal(gathered, Y.cpu().numpy().view(np.uint16))
    rows = synth.sample_rows(cfg["batch"], cfg["seq"])
    ref = O.transformer_layer_rows(f64(inp["X"]), layer_params(inp), cfg["batch"], cfg["seq"],
                                   cfg["n_heads"], rows, cfg["ln_eps"])
    assert_parity(synth.bf16_bits_to_f64(gathered)[rows], ref)
