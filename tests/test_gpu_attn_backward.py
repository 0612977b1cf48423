"""Attention backward on a B200 against the fp64 oracle: the per-shard
attention backward kernel (with the forward's log-sum-exp) and the attention
block's tensor-parallel backward ("Tensor Parallelism in Large Language
Models", "Local Self-Attention Computation" and "Communication Budget and
Scaling Limits": one reduction per block in the backward pass).
"""
import math

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


def _ws(tp, kind, M, h, F, n):
    nbytes = tp.tp_workspace_bytes(kind, M, h, F, n)
    assert nbytes > 0
    return torch.empty(nbytes, dtype=torch.uint8, device="cuda"), nbytes


def _core_case(tp, rng, n, batch, seq, h, causal, q_std=1.0):
    d = 128
    n_heads = h // d
    hs = h // n
    M = batch * seq
    QKV = _bits(rng, (n, M, 3 * hs), q_std)
    dO = _bits(rng, (n, M, hs))
    qkv_d, do_d = to_dev(QKV), to_dev(dO)
    O_d = torch.empty((n, M, hs), dtype=torch.int16, device="cuda")
    lse = torch.empty(n_heads * (M + 128), dtype=torch.float32, device="cuda")
    tp.tp_attention_lse(qkv_d, batch, seq, h, n_heads, causal, n, O_d, lse)
    ws, nb = _ws(tp, tp.TP_WS_ATTN_CORE_BWD, M, h, 0, n)
    dQKV = torch.empty((n, M, 3 * hs), dtype=torch.int16, device="cuda")
    tp.tp_attention_backward(qkv_d, O_d, do_d, lse, batch, seq, h, n_heads, causal, n, ws, nb, dQKV)
    assert tp.tp_get_last_error() == tp.TP_OK
    return QKV, dO, O_d, lse, dQKV


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("n,batch,seq,h", [(1, 2, 128, 256), (2, 2, 200, 512), (2, 1, 384, 256),
                                           (4, 3, 136, 512), (2, 3, 130, 256)])
def test_attention_backward_parity(tp, n, batch, seq, h, causal):
    rng = np.random.default_rng(1000 + n * 7 + seq + int(causal))
    hs = h // n
    hps = hs // 128
    QKV, dO, O_d, lse, dQKV = _core_case(tp, rng, n, batch, seq, h, causal)
    got = from_dev_bf16(dQKV)
    lse_h = lse.cpu().numpy().reshape(n * hps, batch * seq + 128)
    for i in range(n):
        q, k, v = (f64(QKV[i][:, c * hs:(c + 1) * hs]) for c in range(3))
        dq, dk, dv = O.attention_heads_backward(q, k, v, f64(dO[i]), batch, seq, hps, causal)
        assert_parity(got[i][:, :hs], dq, f"dQ shard {i}")
        assert_parity(got[i][:, hs:2 * hs], dk, f"dK shard {i}")
        assert_parity(got[i][:, 2 * hs:], dv, f"dV shard {i}")
        # the forward's log-sum-exp (base 2) against the oracle's (natural)
        for s in range(batch):
            r = slice(s * seq, (s + 1) * seq)
            for kk in range(hps):
                c = slice(kk * 128, (kk + 1) * 128)
                ref = O.attention_logsumexp(q[r, c], k[r, c], causal)
                np.testing.assert_allclose(lse_h[i * hps + kk, s * seq:(s + 1) * seq] * math.log(2.0),
                                           ref, rtol=0, atol=2e-3)


def test_attention_backward_identities(tp):
    """Per (sequence, head): sum over keys of dK is 0 and of dV is sum over
    queries of dO, up to the bf16 rounding of the outputs; the first causal
    query of every sequence has dQ = 0 (its softmax row is the constant 1),
    up to the rounding of dP - D."""
    rng = np.random.default_rng(1100)
    n, batch, seq, h = 2, 2, 256, 512
    hs, hps = h // n, h // n // 128
    QKV, dO, _, _, dQKV = _core_case(tp, rng, n, batch, seq, h, True)
    got = from_dev_bf16(dQKV)
    for i in range(n):
        for s in range(batch):
            r = slice(s * seq, (s + 1) * seq)
            assert np.abs(got[i][s * seq, :hs]).max() <= 1e-3 * np.abs(got[i][:, :hs]).max()
            for kk in range(hps):
                dk = got[i][r, hs + kk * 128:hs + (kk + 1) * 128]
                dv = got[i][r, 2 * hs + kk * 128:2 * hs + (kk + 1) * 128]
                do = f64(dO[i])[r, kk * 128:(kk + 1) * 128]
                assert np.abs(dk.sum(axis=0)).max() <= 2e-2 * np.abs(dk).sum(axis=0).max()
                np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), rtol=0,
                                           atol=2e-2 * np.abs(do).sum(axis=0).max())


def test_attention_backward_errors(tp):
    z = torch.zeros(1 << 16, dtype=torch.int16, device="cuda")
    lse = torch.zeros(1 << 12, dtype=torch.float32, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(tp.TPError) as e:      # head_dim 64
        tp.tp_attention_backward(z, z, z, lse, 1, 64, 256, 4, 1, 1, ws, ws.numel(), z)
    assert e.value.status == tp.TP_ERR_UNSUPPORTED
    with pytest.raises(tp.TPError) as e:      # 2 heads over 4 shards
        tp.tp_attention_backward(z, z, z, lse, 1, 64, 256, 2, 1, 4, ws, ws.numel(), z)
    assert e.value.status == tp.TP_ERR_SHAPE
    with pytest.raises(tp.TPError) as e:      # workspace too small
        tp.tp_attention_backward(z, z, z, lse, 1, 64, 256, 2, 1, 1, ws, 16, z)
    assert e.value.status == tp.TP_ERR_WORKSPACE
    with pytest.raises(tp.TPError) as e:
        tp.tp_attention_backward(z, None, z, lse, 1, 64, 256, 2, 1, 1, ws, ws.numel(), z)
    assert e.value.status == tp.TP_ERR_NULL


# ---------------------------------------------------------------- the attention block

def _shard(tp, W_dev, h_in, h_out, kind, n, head_dim=0):
    out = torch.empty(h_in * h_out, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(W_dev, h_in, h_out, n, kind, head_dim, out)
    return out


def run_attn_backward(tp, inp, dY_bits, batch, seq, h, n_heads, n, causal=True, residual=True):
    M = batch * seq
    hs = h // n
    dev = {k: to_dev(v) for k, v in inp.items()}
    Wqkv_s = _shard(tp, dev["Wqkv"], h, 3 * h, 2, n, 128)
    bqkv_s = _shard(tp, dev["bqkv"], 1, 3 * h, 2, n, 128)
    Wo_s = _shard(tp, dev["Wo"], h, h, 1, n)
    ws, nb = _ws(tp, tp.TP_WS_ATTN_BWD, M, h, 0, n)
    dX = torch.empty((M, h), dtype=torch.int16, device="cuda")
    dWqkv = torch.empty((n, 3 * hs, h), dtype=torch.float32, device="cuda")
    dbqkv = torch.empty((n, 3 * hs), dtype=torch.float32, device="cuda")
    dWo = torch.empty((n, h, hs), dtype=torch.float32, device="cuda")
    dbo = torch.empty(h, dtype=torch.float32, device="cuda")
    tp.tp_attn_backward(dev["X"], batch, seq, h, n_heads, causal, n, Wqkv_s, bqkv_s, Wo_s,
                        to_dev(dY_bits), residual, ws, nb, dX, dWqkv, dbqkv, dWo, dbo)
    assert tp.tp_get_last_error() == tp.TP_OK
    return dict(dX=from_dev_bf16(dX), dWqkv=dWqkv.cpu().numpy().astype(np.float64),
                dbqkv=dbqkv.cpu().numpy().astype(np.float64),
                dWo=dWo.cpu().numpy().astype(np.float64), dbo=dbo.cpu().numpy().astype(np.float64))


@pytest.mark.parametrize("n,batch,seq,h", [(1, 2, 128, 256), (2, 2, 192, 512), (4, 1, 256, 512)])
def test_attn_block_backward_small(tp, n, batch, seq, h):
    cfg = dict(kind="attn", batch=batch, seq=seq, h=h, n_heads=h // 128, x_std=1.0, w_std=0.05,
               b_std=0.05)
    inp = synth.make_inputs(cfg, seed=7 + n)
    M = batch * seq
    dY = _bits(np.random.default_rng(1200 + n), (M, h))
    got = run_attn_backward(tp, inp, dY, batch, seq, h, h // 128, n)
    ref = O.self_attention_backward_sharded(f64(inp["X"]), f64(inp["Wqkv"]), f64(inp["bqkv"]),
                                            f64(inp["Wo"]), f64(inp["bo"]), f64(dY), batch, seq,
                                            h // 128, n)
    assert_parity(got["dX"], ref["dX"], "dX")
    # weight gradients in the packed shard layouts of the weights
    assert_parity(got["dWqkv"], O.packed_shards(ref["dWqkv"], O.SPLIT_QKV_HEADS, n, 128), "dWqkv")
    assert_parity(got["dbqkv"], O.shard_vector(ref["dbqkv"], O.SPLIT_QKV_HEADS, n, 128), "dbqkv")
    assert_parity(got["dWo"], O.packed_shards(ref["dWo"], O.SPLIT_ROW, n), "dWo")
    assert_parity(got["dbo"], ref["dbo"], "dbo")


def test_attn_block_backward_workload(tp):
    """The 4 x 2048-token, 16-head, 8-shard attention workload: dX of the
    first sequence against the oracle (sequences are independent, so the
    oracle runs on that sequence alone), dbo exactly as the column sum of dY."""
    cfg = synth.config("attn_4x2048_h2048_16x128_n8")
    inp = synth.make_inputs(cfg)
    b, s, h, nh, n = cfg["batch"], cfg["seq"], cfg["h"], cfg["n_heads"], cfg["n_shards"]
    dY = _bits(np.random.default_rng(1300), (b * s, h))
    got = run_attn_backward(tp, inp, dY, b, s, h, nh, n)
    ref = O.self_attention_backward_sharded(f64(inp["X"][:s]), f64(inp["Wqkv"]), f64(inp["bqkv"]),
                                            f64(inp["Wo"]), f64(inp["bo"]), f64(dY[:s]), 1, s,
                                            nh, n)
    assert_parity(got["dX"][:s], ref["dX"], "dX of sequence 0")
    np.testing.assert_allclose(got["dbo"], f64(dY).sum(axis=0), rtol=1e-5, atol=1e-3)
