"""Layer backward on a B200 against the fp64 oracle: the LayerNorm-backward
reduction (a block's one backward all-reduce fused with the LN backward and
the residual) and the whole pre-LN layer ("Tensor Parallelism in Large
Language Models", "Communication Budget and Scaling Limits": two reductions in
the backward pass of a layer).
"""
import numpy as np
import pytest

from oracle import tp_oracle as O
from tensor_transformer_layer_linear_b200 import synth

from helpers import BWD_FRO_REL, assert_parity, f64, from_dev_bf16, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tp():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tensor_transformer_layer_linear_b200 import tp as _tp
    return _tp


def _bits(rng, shape, std=1.0, mean=0.0):
    x = rng.standard_normal(shape, dtype=np.float32) * np.float32(std) + np.float32(mean)
    return synth.f32_to_bf16_bits(x)


def _ws(tp, kind, M, h, F, n):
    nbytes = tp.tp_workspace_bytes(kind, M, h, F, n)
    assert nbytes > 0
    return torch.empty(nbytes, dtype=torch.uint8, device="cuda"), nbytes


@pytest.mark.parametrize("n,B,h", [(1, 64, 256), (2, 300, 1000), (3, 77, 512), (4, 130, 4096),
                                   (8, 257, 4096), (2, 40, 12288),
                                   # more shards than ring stages per row, many rows per CTA
                                   (16, 1000, 1024), (5, 333, 1536),
                                   # rows of two stages (the second one ragged or full)
                                   (3, 17, 4104), (2, 150, 6152), (8, 64, 8192),
                                   (1, 20, 16384)])
def test_reduce_partials_layernorm_backward(tp, n, B, h):
    rng = np.random.default_rng(1400 + n + h)
    P = rng.standard_normal((n, B, h)).astype(np.float32)
    x = _bits(rng, (B, h), 2.0, 0.5)
    gamma = _bits(rng, (h,), 0.3, 1.0)
    res = _bits(rng, (B, h))
    dX = torch.empty((B, h), dtype=torch.int16, device="cuda")
    dg = torch.empty(h, dtype=torch.float32, device="cuda")
    db = torch.empty(h, dtype=torch.float32, device="cuda")
    ws, nb = _ws(tp, tp.TP_WS_LN_BWD, B, h, 0, n)
    tp.tp_reduce_partials_layernorm_backward(torch.from_numpy(P).cuda(), n, B, h, to_dev(x),
                                             to_dev(gamma), to_dev(res), 1e-5, ws, nb, dX, dg, db)
    assert tp.tp_get_last_error() == tp.TP_OK
    g = O.reduce_partials(list(P.astype(np.float64)))
    ref_dx, ref_dg, ref_db = O.layernorm_backward(f64(x), f64(gamma), g, 1e-5)
    assert_parity(from_dev_bf16(dX), f64(res) + ref_dx, "dX")
    assert_parity(dg.cpu().numpy().astype(np.float64), ref_dg, "dgamma")
    assert_parity(db.cpu().numpy().astype(np.float64), ref_db, "dbeta")
    # without a residual gradient the row sums of dX vanish (LN is shift invariant)
    tp.tp_reduce_partials_layernorm_backward(torch.from_numpy(P).cuda(), n, B, h, to_dev(x),
                                             to_dev(gamma), None, 1e-5, ws, nb, dX, dg, db)
    d0 = from_dev_bf16(dX)
    assert np.abs(d0.sum(axis=1)).max() <= 2e-2 * np.abs(d0).sum(axis=1).max()


def test_layernorm_backward_errors(tp):
    z = torch.zeros(1 << 16, dtype=torch.int16, device="cuda")
    f = torch.zeros(1 << 16, dtype=torch.float32, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(tp.TPError) as e:
        tp.tp_reduce_partials_layernorm_backward(f, 1, 4, 12, z, z, None, 1e-5, ws, ws.numel(), z, f, f)
    assert e.value.status == tp.TP_ERR_SHAPE
    with pytest.raises(tp.TPError) as e:
        tp.tp_reduce_partials_layernorm_backward(f, 1, 4, 256, z, z, None, 1e-5, ws, 64, z, f, f)
    assert e.value.status == tp.TP_ERR_WORKSPACE
    with pytest.raises(tp.TPError) as e:
        tp.tp_reduce_partials_layernorm_backward(f, 1, 4, 256, None, z, None, 1e-5, ws, ws.numel(),
                                                 z, f, f)
    assert e.value.status == tp.TP_ERR_NULL


# ---------------------------------------------------------------- the layer

GRAD_NAMES = ("ln1_gamma", "ln1_beta", "Wqkv_shards", "bqkv_shards", "Wo_shards", "bo",
              "ln2_gamma", "ln2_beta", "A_shards", "b1_shards", "B_shards", "b2")


def _shard(tp, W_dev, h_in, h_out, kind, n, head_dim=0):
    out = torch.empty(h_in * h_out, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(W_dev, h_in, h_out, n, kind, head_dim, out)
    return out


def run_layer_backward(tp, inp, dY_bits, cfg, n):
    b, s, h, nh, F = cfg["batch"], cfg["seq"], cfg["h"], cfg["n_heads"], cfg["ffn"]
    M = b * s
    dev = {k: to_dev(v) for k, v in inp.items()}
    keep = dict(
        ln1_gamma=dev["ln1_g"], ln1_beta=dev["ln1_b"],
        Wqkv_shards=_shard(tp, dev["Wqkv"], h, 3 * h, 2, n, 128),
        bqkv_shards=_shard(tp, dev["bqkv"], 1, 3 * h, 2, n, 128),
        Wo_shards=_shard(tp, dev["Wo"], h, h, 1, n), bo=dev["bo"],
        ln2_gamma=dev["ln2_g"], ln2_beta=dev["ln2_b"],
        A_shards=_shard(tp, dev["A"], h, F, 0, n), b1_shards=dev["b1"],
        B_shards=_shard(tp, dev["B"], F, h, 1, n), b2=dev["b2"])
    w = tp.make_layer_weights(**keep)
    sizes = dict(ln1_gamma=h, ln1_beta=h, Wqkv_shards=3 * h * h, bqkv_shards=3 * h,
                 Wo_shards=h * h, bo=h, ln2_gamma=h, ln2_beta=h, A_shards=h * F, b1_shards=F,
                 B_shards=F * h, b2=h)
    gt = {k: torch.empty(v, dtype=torch.float32, device="cuda") for k, v in sizes.items()}
    g = tp.make_layer_grads(**gt)
    ws, nb = _ws(tp, tp.TP_WS_LAYER_BWD, M, h, F, n)
    dX = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_layer_backward(dev["X"], b, s, h, nh, F, n, w, cfg.get("ln_eps", 1e-5), to_dev(dY_bits),
                         ws, nb, dX, g)
    assert tp.tp_get_last_error() == tp.TP_OK
    out = {k: v.cpu().numpy().astype(np.float64) for k, v in gt.items()}
    out["dX"] = from_dev_bf16(dX)
    return out


def _packed_ref(ref, n, h, F):
    """The oracle's unsharded gradients in the packed layouts of the weights."""
    return dict(
        ln1_gamma=ref["dln1_g"], ln1_beta=ref["dln1_b"],
        Wqkv_shards=O.packed_shards(ref["dWqkv"], O.SPLIT_QKV_HEADS, n, 128).ravel(),
        bqkv_shards=O.shard_vector(ref["dbqkv"], O.SPLIT_QKV_HEADS, n, 128).ravel(),
        Wo_shards=O.packed_shards(ref["dWo"], O.SPLIT_ROW, n).ravel(), bo=ref["dbo"],
        ln2_gamma=ref["dln2_g"], ln2_beta=ref["dln2_b"],
        A_shards=O.packed_shards(ref["dA"], O.SPLIT_COLUMN, n).ravel(), b1_shards=ref["db1"],
        B_shards=O.packed_shards(ref["dB"], O.SPLIT_ROW, n).ravel(), b2=ref["db2"])


@pytest.mark.parametrize("n", [1, 2, 4])
def test_layer_backward_small(tp, n):
    cfg = dict(kind="layer", batch=2, seq=160, h=512, n_heads=4, ffn=2048, x_std=1.0,
               w_std=0.05, b_std=0.05, ln_eps=1e-5)
    inp = synth.make_inputs(cfg, seed=11)
    # LN parameters away from (1, 0) so that their gradients matter
    rng = np.random.default_rng(1500)
    for k in ("ln1_g", "ln2_g"):
        inp[k] = _bits(rng, (cfg["h"],), 0.2, 1.0)
    for k in ("ln1_b", "ln2_b"):
        inp[k] = _bits(rng, (cfg["h"],), 0.1)
    M = cfg["batch"] * cfg["seq"]
    dY = _bits(rng, (M, cfg["h"]))
    got = run_layer_backward(tp, inp, dY, cfg, n)
    p = {k: f64(v) for k, v in inp.items() if k != "X"}
    ref = O.transformer_layer_backward(f64(inp["X"]), p, f64(dY), cfg["batch"], cfg["seq"],
                                       cfg["n_heads"], n, cfg["ln_eps"])
    assert_parity(got["dX"], ref["dX"], "dX", fro_rel=BWD_FRO_REL)
    failures = []
    for k, v in _packed_ref(ref, n, cfg["h"], cfg["ffn"]).items():
        try:
            assert_parity(got[k], v, k, fro_rel=BWD_FRO_REL)
        except AssertionError as e:
            failures.append(str(e))
    assert not failures, failures


def test_layer_backward_workload(tp):
    """The 2 x 2048-token layer (h 4096, 32 heads, F 16384, 8 shards): dX of
    the first sequence against the oracle run on that sequence alone
    (sequences do not interact in a layer), and db2 as the column sum of dY."""
    cfg = synth.config("layer_2x2048_h4096_32x128_f16384_n8")
    inp = synth.make_inputs(cfg)
    b, s, h, nh, n = cfg["batch"], cfg["seq"], cfg["h"], cfg["n_heads"], cfg["n_shards"]
    dY = _bits(np.random.default_rng(1600), (b * s, h))
    got = run_layer_backward(tp, inp, dY, cfg, n)
    p = {k: f64(v) for k, v in inp.items() if k != "X"}
    ref = O.transformer_layer_backward(f64(inp["X"][:s]), p, f64(dY[:s]), 1, s, nh, n,
                                       cfg["ln_eps"])
    assert_parity(got["dX"][:s], ref["dX"], "dX of sequence 0", fro_rel=BWD_FRO_REL)
    np.testing.assert_allclose(got["b2"], f64(dY).sum(axis=0), rtol=1e-5, atol=1e-3)


# ---------------------------------------------------------------- sequence parallelism

def _slices(bits, batch, seq, n):
    h = bits.shape[-1]
    return np.ascontiguousarray(np.stack(O.sequence_shard(bits.reshape(batch * seq, h), batch, seq, n)))


# gradients that do not depend on dQ (whose fp32 accumulation order varies
# between runs) are bit-identical between the two layouts
EXACT = ("ln2_gamma", "ln2_beta", "A_shards", "b1_shards", "B_shards", "b2", "Wo_shards", "bo")


def _same_as_standard(sp, std, b, s):
    """The same kernels on permuted rows: the MLP side and W_O bit-identical,
    the rest equal up to dQ's accumulation order."""
    for k in EXACT:
        assert np.array_equal(sp[k], std[k]), k
    got = synth.bf16_bits_to_f64(O.all_gather_sequence(list(sp["dX_bits"]), b, s))
    assert_parity(got, std["dX"], "dX vs standard", max_rel=2e-3, fro_rel=1e-4)
    for k in ("Wqkv_shards", "bqkv_shards", "ln1_gamma", "ln1_beta"):
        assert_parity(sp[k], std[k], k + " vs standard", max_rel=2e-3, fro_rel=1e-4)


def run_layer_backward_sp(tp, inp, dY_bits, cfg, n):
    """tp_layer_backward_sp on the slices of X and dY; returns dX slices and
    the gradients (same packing as run_layer_backward)."""
    b, s, h, nh, F = cfg["batch"], cfg["seq"], cfg["h"], cfg["n_heads"], cfg["ffn"]
    M = b * s
    dev = {k: to_dev(v) for k, v in inp.items()}
    keep = dict(
        ln1_gamma=dev["ln1_g"], ln1_beta=dev["ln1_b"],
        Wqkv_shards=_shard(tp, dev["Wqkv"], h, 3 * h, 2, n, 128),
        bqkv_shards=_shard(tp, dev["bqkv"], 1, 3 * h, 2, n, 128),
        Wo_shards=_shard(tp, dev["Wo"], h, h, 1, n), bo=dev["bo"],
        ln2_gamma=dev["ln2_g"], ln2_beta=dev["ln2_b"],
        A_shards=_shard(tp, dev["A"], h, F, 0, n), b1_shards=dev["b1"],
        B_shards=_shard(tp, dev["B"], F, h, 1, n), b2=dev["b2"])
    w = tp.make_layer_weights(**keep)
    sizes = dict(ln1_gamma=h, ln1_beta=h, Wqkv_shards=3 * h * h, bqkv_shards=3 * h,
                 Wo_shards=h * h, bo=h, ln2_gamma=h, ln2_beta=h, A_shards=h * F, b1_shards=F,
                 B_shards=F * h, b2=h)
    gt = {k: torch.empty(v, dtype=torch.float32, device="cuda") for k, v in sizes.items()}
    g = tp.make_layer_grads(**gt)
    ws, nb = _ws(tp, tp.TP_WS_LAYER_BWD_SP, M, h, F, n)
    dXs = torch.empty((n, b, s // n, h), dtype=torch.int16, device="cuda")
    tp.tp_layer_backward_sp(to_dev(_slices(inp["X"], b, s, n)), b, s, h, nh, F, n, w,
                            cfg.get("ln_eps", 1e-5), to_dev(_slices(dY_bits, b, s, n)), ws, nb,
                            dXs, g)
    assert tp.tp_get_last_error() == tp.TP_OK
    out = {k: v.cpu().numpy().astype(np.float64) for k, v in gt.items()}
    out["dX_bits"] = dXs.cpu().numpy().view(np.uint16)
    return out


@pytest.mark.parametrize("n", [1, 2, 4])
def test_layer_backward_sp_small(tp, n):
    cfg = dict(kind="layer", batch=2, seq=160, h=512, n_heads=4, ffn=2048, x_std=1.0,
               w_std=0.05, b_std=0.05, ln_eps=1e-5)
    inp = synth.make_inputs(cfg, seed=12)
    rng = np.random.default_rng(1700)
    for k in ("ln1_g", "ln2_g"):
        inp[k] = _bits(rng, (cfg["h"],), 0.2, 1.0)
    for k in ("ln1_b", "ln2_b"):
        inp[k] = _bits(rng, (cfg["h"],), 0.1)
    b, s = cfg["batch"], cfg["seq"]
    dY = _bits(rng, (b * s, cfg["h"]))
    sp = run_layer_backward_sp(tp, inp, dY, cfg, n)
    std = run_layer_backward(tp, inp, dY, cfg, n)
    _same_as_standard(sp, std, b, s)
    # and against the oracle's sequence-parallel backward
    p = {k: f64(v) for k, v in inp.items() if k != "X"}
    ref = O.transformer_layer_sp_backward(O.sequence_shard(f64(inp["X"]), b, s, n), p,
                                          O.sequence_shard(f64(dY), b, s, n), b, s,
                                          cfg["n_heads"], n, cfg["ln_eps"])
    for i in range(n):
        assert_parity(synth.bf16_bits_to_f64(sp["dX_bits"][i]), ref["dX"][i], f"dX slice {i}",
                      fro_rel=BWD_FRO_REL)
    for k, v in _packed_ref(ref, n, cfg["h"], cfg["ffn"]).items():
        assert_parity(sp[k], v, k, fro_rel=BWD_FRO_REL)


def test_layer_backward_sp_workload(tp):
    """The layer workload under sequence parallelism: bit-identical to the
    standard layer backward up to the row permutation."""
    cfg = synth.config("layer_2x2048_h4096_32x128_f16384_n8")
    inp = synth.make_inputs(cfg)
    b, s, n = cfg["batch"], cfg["seq"], cfg["n_shards"]
    dY = _bits(np.random.default_rng(1800), (b * s, cfg["h"]))
    sp = run_layer_backward_sp(tp, inp, dY, cfg, n)
    std = run_layer_backward(tp, inp, dY, cfg, n)
    _same_as_standard(sp, std, b, s)
