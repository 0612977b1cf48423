"""MLP backward on a B200 against the fp64 oracle ("Tensor Parallelism in
Large Language Models", MLP block: one all-reduce in the backward pass, of
the input gradient across the column-parallel layer). Exercises the GEMM's
MN-major operand paths (the weight gradients and the transposed pairing)
and the GeLU-backward epilogue.
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


def _run_backward(tp, X, A, b1, B, dY, n, residual=True):
    M, h = X.shape
    F = A.shape[1]
    dev = {k: to_dev(v) for k, v in dict(X=X, A=A, b1=b1, B=B, dY=dY).items()}
    A_s = torch.empty(h * F, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(dev["A"], h, F, n, tp.TP_SPLIT_COLUMN, 0, A_s)
    B_s = torch.empty(F * h, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(dev["B"], F, h, n, tp.TP_SPLIT_ROW, 0, B_s)
    nb = tp.tp_workspace_bytes(tp.TP_WS_MLP_BWD, M, h, F, n)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    dX = torch.empty((M, h), dtype=torch.int16, device="cuda")
    dA = torch.empty((n, F // n, h), dtype=torch.float32, device="cuda")
    dB = torch.empty((n, h, F // n), dtype=torch.float32, device="cuda")
    db1 = torch.empty(F, dtype=torch.float32, device="cuda")
    db2 = torch.empty(h, dtype=torch.float32, device="cuda")
    tp.tp_mlp_backward(dev["X"], M, h, F, n, A_s, dev["b1"], B_s, dev["dY"], residual, ws, nb,
                       dX, dA, db1, dB, db2)
    assert tp.tp_get_last_error() == tp.TP_OK
    return dict(dX=from_dev_bf16(dX), dA=dA.cpu().numpy().astype(np.float64),
                dB=dB.cpu().numpy().astype(np.float64), db1=db1.cpu().numpy().astype(np.float64),
                db2=db2.cpu().numpy().astype(np.float64))


def _check(got, ref, n):
    assert_parity(got["dX"], ref["dX"], "dX")
    assert_parity(got["dA"], O.packed_shards(ref["dA"], O.SPLIT_COLUMN, n), "dA")
    assert_parity(got["dB"], O.packed_shards(ref["dB"], O.SPLIT_ROW, n), "dB")
    assert_parity(got["db1"], ref["db1"], "db1")
    assert_parity(got["db2"], ref["db2"], "db2")


def _bits(rng, shape, std):
    return synth.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))


@pytest.mark.parametrize("residual", [True, False])
@pytest.mark.parametrize("n", [1, 2, 4])
def test_mlp_backward_small(tp, n, residual):
    rng = np.random.default_rng(1400 + n)
    M, h, F = 160, 256, 1024
    X, A, B = _bits(rng, (M, h), 1.0), _bits(rng, (h, F), 0.05), _bits(rng, (F, h), 0.05)
    b1, dY = _bits(rng, (F,), 0.05), _bits(rng, (M, h), 1.0)
    got = _run_backward(tp, X, A, b1, B, dY, n, residual)
    ref = O.mlp_backward(f64(X), f64(A), f64(b1), f64(B), f64(dY), residual)
    _check(got, ref, n)


def test_mlp_backward_ragged_tokens(tp):
    """Token count (the K of the weight-gradient GEMMs) not a multiple of 64."""
    rng = np.random.default_rng(1450)
    M, h, F, n = 200, 256, 512, 2
    X, A, B = _bits(rng, (M, h), 1.0), _bits(rng, (h, F), 0.05), _bits(rng, (F, h), 0.05)
    b1, dY = _bits(rng, (F,), 0.05), _bits(rng, (M, h), 1.0)
    got = _run_backward(tp, X, A, b1, B, dY, n)
    _check(got, O.mlp_backward(f64(X), f64(A), f64(b1), f64(B), f64(dY)), n)


def test_mlp_backward_workload(tp):
    cfg = synth.config("mlp_8192x1024_f4096_n4")
    inp = synth.make_inputs(cfg)
    rng = np.random.default_rng(1500)
    dY = _bits(rng, (cfg["batch"] * cfg["seq"], cfg["h"]), 1.0)
    n = cfg["n_shards"]
    got = _run_backward(tp, inp["X"], inp["A"], inp["b1"], inp["B"], dY, n)
    ref = O.mlp_backward(f64(inp["X"]), f64(inp["A"]), f64(inp["b1"]), f64(inp["B"]), f64(dY))
    _check(got, ref, n)


def _bf16_ulp(v):
    """Spacing of bf16 values at magnitude |v| (8 significand bits)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


@pytest.mark.parametrize("n", [1, 2])
def test_backward_gelu_epilogue_pointwise(tp, n):
    """The backward recomputes H = GeLU(Z) and GeLU'(Z) in one GEMM epilogue
    with the complementary error function of Abramowitz & Stegun eq. 7.1.26
    (absolute error <= 1.5e-7 in erf, so <= 0.75e-7 in Phi). With A = I
    (h = F), b1 = 0, dY = I (tokens = h) and B all ones, every product and sum
    around that epilogue is exact: Z = X, dB_i^T[j][f] = H[j][f], and
    dX[m][j] = bf16(1 * GeLU'(Z[m][j])) (no residual). So each of the 65536
    grid values z is held to one bf16 rounding of GeLU(z) and of GeLU'(z),
    beyond the approximation's bound plus fp32 evaluation slop
    delta = 5e-7 (1 + |z|)."""
    h = F = M = 256
    grid = [0.0]
    for e in range(-24, 4):                       # every bf16 value of 2^e <= |z| < 2^(e+1)
        for m in range(128):
            v = (1.0 + m / 128.0) * 2.0 ** e
            if v <= 9.0:
                grid += [v, -v]
    rest = M * h - len(grid)
    z = np.concatenate([np.asarray(grid), np.linspace(-9.0, 9.0, rest)]).astype(np.float32)
    X = synth.f32_to_bf16_bits(z.reshape(M, h))
    A = synth.f32_to_bf16_bits(np.eye(h, F, dtype=np.float32))
    B = synth.f32_to_bf16_bits(np.ones((F, h), dtype=np.float32))
    dY = synth.f32_to_bf16_bits(np.eye(M, h, dtype=np.float32))
    b1 = np.zeros(F, dtype=np.uint16)
    got = _run_backward(tp, X, A, b1, B, dY, n, residual=False)
    zz = f64(X)
    H = np.concatenate(list(got["dB"]), axis=1)   # [tokens][F]: H = GeLU(Z)
    delta = 5e-7 * (1.0 + np.abs(zz))
    for what, g, ref in (("GeLU", H, O.gelu(zz)), ("GeLU'", got["dX"], O.gelu_grad(zz))):
        tol = _bf16_ulp(np.abs(ref) + delta) / 2 + delta
        bad = np.abs(g - ref) > tol
        assert not bad.any(), (what, zz[bad][:8], g[bad][:8], ref[bad][:8])
