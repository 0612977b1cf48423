"""Kernel parity on a B200: every entry point of the C ABI against the fp64
oracle, at sizes that span several tiles and end in ragged tails.

Integer-valued inputs make the GEMMs and the reduction exact in fp32 (and in
bf16 where the results stay within +-256), so those checks are bit-exact;
random inputs are held to the value tolerance of tests/helpers.py.
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


def _rand_bits(rng, shape, std=1.0):
    return synth.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))


def _int_bits(rng, shape, lo, hi):
    return synth.f32_to_bf16_bits(rng.integers(lo, hi + 1, size=shape).astype(np.float32))


def _shard(tp, W_bits, kind, n, head_dim=0):
    h_in, h_out = W_bits.shape
    out = torch.empty(W_bits.size, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(to_dev(W_bits), h_in, h_out, n, kind, head_dim, out)
    return out


def _bits(t):
    return t.cpu().numpy().view(np.uint16)


# ------------------------------------------------------------------ sharding

@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("kind,h_in,h_out,hd", [
    (0, 200, 640, 0), (1, 384, 200, 0), (2, 136, 3 * 256, 16), (0, 1, 640, 0), (2, 1, 3 * 256, 16)])
def test_shard_weights_bit_exact(tp, kind, h_in, h_out, hd, n):
    rng = np.random.default_rng(100 + kind)
    W = _rand_bits(rng, (h_in, h_out))
    got = _bits(_shard(tp, W, kind, n, hd))
    ref = O.packed_shards(W, kind, n, hd)
    assert np.array_equal(got.reshape(ref.shape), ref)
    torch.cuda.synchronize()


# ------------------------------------------------------------------ GEMMs

@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_row_linear_integer_bit_exact(tp, n):
    rng = np.random.default_rng(200 + n)
    M, k_loc, h_out = 300, 200, 520            # 3 m-tiles, K tail 8, N tail 8
    h_in = n * k_loc
    X = _int_bits(rng, (M, h_in), -8, 8)
    W = _int_bits(rng, (h_in, h_out), -8, 8)
    Xs = np.ascontiguousarray(np.stack(O.split_columns(X, n)))   # [N][M][k_loc]
    P = torch.empty((n, M, h_out), dtype=torch.float32, device="cuda")
    tp.tp_row_linear(to_dev(Xs), M, h_in, _shard(tp, W, 1, n), h_out, n, P)
    ref = O.row_parallel_linear(O.split_columns(f64(X), n), f64(W), n)
    got = P.cpu().numpy().astype(np.float64)
    for i in range(n):
        assert np.array_equal(got[i], ref[i]), f"shard {i}"


@pytest.mark.parametrize("n", [1, 2, 4])
@pytest.mark.parametrize("nc", [264, 120])
def test_column_linear_integer_bit_exact(tp, n, nc):
    rng = np.random.default_rng(300 + n)
    M, h_in = 130, 136                         # ragged m, K = 2 blocks + 8
    h_out = n * nc
    X = _int_bits(rng, (M, h_in), -1, 1)
    W = _int_bits(rng, (h_in, h_out), -1, 1)
    b = _int_bits(rng, (h_out,), -2, 2)
    Y = torch.empty((n, M, nc), dtype=torch.int16, device="cuda")
    tp.tp_column_linear(to_dev(X), M, h_in, _shard(tp, W, 0, n), to_dev(b), h_out, n,
                        tp.TP_ACT_NONE, Y)
    ref = O.column_parallel_linear(f64(X), f64(W), f64(b), n)
    got = from_dev_bf16(Y)
    for i in range(n):
        assert np.array_equal(got[i], ref[i]), f"shard {i}"


@pytest.mark.parametrize("n", [1, 2, 4, 8])
@pytest.mark.parametrize("act", [0, 1])
def test_column_linear_random(tp, n, act):
    rng = np.random.default_rng(400 + n)
    M, h_in, nc = 257, 320, 136
    h_out = n * nc
    X = _rand_bits(rng, (M, h_in))
    W = _rand_bits(rng, (h_in, h_out), 0.05)
    b = _rand_bits(rng, (h_out,), 0.1)
    Y = torch.empty((n, M, nc), dtype=torch.int16, device="cuda")
    tp.tp_column_linear(to_dev(X), M, h_in, _shard(tp, W, 0, n), to_dev(b), h_out, n, act, Y)
    ref = O.column_parallel_linear(f64(X), f64(W), f64(b), n, act=O.gelu if act else None)
    got = from_dev_bf16(Y)
    for i in range(n):
        assert_parity(got[i], ref[i], f"shard {i}")
    # the gather of the column shards is the unsharded product
    full = O.linear(f64(X), f64(W), f64(b))
    assert_parity(np.concatenate(list(got), axis=1), O.gelu(full) if act else full, "gather")


def test_column_linear_gelu_pointwise(tp):
    """With an identity weight the column GEMM's epilogue applies GeLU to each
    input value exactly (the products and sums are exact), so the output can
    be held to one bf16 rounding of the true erf GeLU at 16384 points."""
    z = np.linspace(-8.0, 8.0, 256 * 64).astype(np.float32)
    z[:4] = [0.0, 1e-30, -1e-30, -0.0]
    X = synth.f32_to_bf16_bits(z).reshape(256, 64)
    W = synth.f32_to_bf16_bits(np.eye(64, dtype=np.float32))
    Y = torch.empty((1, 256, 64), dtype=torch.int16, device="cuda")
    tp.tp_column_linear(to_dev(X), 256, 64, _shard(tp, W, 0, 1), None, 64, 1, 1, Y)
    zx = f64(X)
    ref = O.gelu(zx)
    got = from_dev_bf16(Y)[0]
    # bf16 keeps 8 significant bits: one rounding is within 2^-8 relative; the
    # absolute floor covers the far negative tail where GeLU is ~1e-9
    tol = np.maximum(2.0 ** -8 * np.abs(ref), 1e-7 * np.abs(zx))
    bad = np.abs(got - ref) > tol
    assert not bad.any(), (zx[bad][:5], got[bad][:5], ref[bad][:5])


def test_column_linear_qkv_heads(tp):
    rng = np.random.default_rng(450)
    M, h, d, n = 192, 512, 128, 2
    X = _rand_bits(rng, (M, h))
    W = _rand_bits(rng, (h, 3 * h), 0.05)
    b = _rand_bits(rng, (3 * h,), 0.1)
    bs = torch.empty(3 * h, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(to_dev(b), 1, 3 * h, n, 2, d, bs)
    assert np.array_equal(_bits(bs).reshape(n, -1), O.shard_vector(b, 2, n, d))
    Y = torch.empty((n, M, 3 * h // n), dtype=torch.int16, device="cuda")
    tp.tp_column_linear(to_dev(X), M, h, _shard(tp, W, 2, n, d), bs, 3 * h, n, 0, Y)
    ref = O.column_parallel_linear(f64(X), f64(W), f64(b), n, kind=O.SPLIT_QKV_HEADS, head_dim=d)
    got = from_dev_bf16(Y)
    for i in range(n):
        assert_parity(got[i], ref[i], f"shard {i}")


# ------------------------------------------------------------------ reduction / LN

@pytest.mark.parametrize("n", [1, 2, 3, 4, 8, 16])
def test_reduce_partials(tp, n):
    rng = np.random.default_rng(500 + n)
    M, h = 77, 1032
    P = rng.standard_normal((n, M, h)).astype(np.float32)
    b = _rand_bits(rng, (h,), 0.5)
    R = _rand_bits(rng, (M, h))
    Y = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_reduce_partials(torch.from_numpy(P).cuda(), n, M, h, to_dev(b), to_dev(R), Y)
    ref = O.reduce_partials(list(P.astype(np.float64)), f64(b), f64(R))
    assert_parity(from_dev_bf16(Y), ref)
    # integer partials: the fp32 sum and the bf16 rounding are exact
    Pi = rng.integers(-16, 17, size=(n, M, h)).astype(np.float32)
    Yi = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_reduce_partials(torch.from_numpy(Pi).cuda(), n, M, h, None, None, Yi)
    ref = O.reduce_partials(list(Pi.astype(np.float64)))
    assert np.all(np.abs(ref) <= 256)
    assert np.array_equal(from_dev_bf16(Yi), ref)


@pytest.mark.parametrize("h", [1024, 4096, 12288])
def test_layernorm(tp, h):
    rng = np.random.default_rng(600)
    M = 33
    X = synth.f32_to_bf16_bits(rng.standard_normal((M, h)).astype(np.float32) * 3 + 1)
    g = _rand_bits(rng, (h,))
    be = _rand_bits(rng, (h,))
    Y = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_layernorm(to_dev(X), M, h, to_dev(g), to_dev(be), 1e-5, Y)
    assert_parity(from_dev_bf16(Y), O.layernorm(f64(X), f64(g), f64(be), 1e-5))


@pytest.mark.parametrize("n", [2, 8])
def test_reduce_partials_layernorm(tp, n):
    rng = np.random.default_rng(700 + n)
    M, h = 65, 4096
    P = (rng.standard_normal((n, M, h)) * 0.3).astype(np.float32)
    b = _rand_bits(rng, (h,), 0.1)
    R = _rand_bits(rng, (M, h))
    g = _rand_bits(rng, (h,))
    be = _rand_bits(rng, (h,))
    S = torch.empty((M, h), dtype=torch.int16, device="cuda")
    L = torch.empty((M, h), dtype=torch.int16, device="cuda")
    tp.tp_reduce_partials_layernorm(torch.from_numpy(P).cuda(), n, M, h, to_dev(b), to_dev(R),
                                    to_dev(g), to_dev(be), 1e-5, S, L)
    ref_s = O.reduce_partials(list(P.astype(np.float64)), f64(b), f64(R))
    assert_parity(from_dev_bf16(S), ref_s, "sum")
    assert_parity(from_dev_bf16(L), O.layernorm(ref_s, f64(g), f64(be), 1e-5), "ln")


# ------------------------------------------------------------------ attention

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("n", [1, 2, 4])
def test_attention(tp, n, causal):
    rng = np.random.default_rng(800 + n)
    batch, seq, n_heads, d = 2, 300, 4, 128
    h = n_heads * d
    hs = h // n
    QKV = _rand_bits(rng, (n, batch * seq, 3 * hs))
    O_ = torch.empty((n, batch * seq, hs), dtype=torch.int16, device="cuda")
    tp.tp_attention(to_dev(QKV), batch, seq, h, n_heads, causal, n, O_)
    got = from_dev_bf16(O_)
    q = f64(QKV)
    for i in range(n):
        ref = O.attention_heads(q[i][:, :hs], q[i][:, hs:2 * hs], q[i][:, 2 * hs:], batch, seq,
                                n_heads // n, causal)
        assert_parity(got[i], ref, f"shard {i}")


@pytest.mark.parametrize("causal", [True, False])
def test_attention_more_tiles_than_sms(tp, causal):
    """512 query tiles (2 shards x 2 sequences x 16 heads x 8 tiles of a
    1000-token sequence, the last ragged) over the persistent CTAs: every CTA
    walks several tiles, so the Q ring, the block numbering across tiles and
    the deferred O store of each tile are all exercised. Every output and, for
    two heads per shard, the log-sum-exp are checked."""
    rng = np.random.default_rng(870 + int(causal))
    n, batch, seq, n_heads, d = 2, 2, 1000, 32, 128
    h = n_heads * d
    hs, hps = h // n, n_heads // n
    M = batch * seq
    QKV = _rand_bits(rng, (n, M, 3 * hs))
    O_ = torch.empty((n, M, hs), dtype=torch.int16, device="cuda")
    lse = torch.empty(n * hps * (M + 128), dtype=torch.float32, device="cuda")
    tp.tp_attention_lse(to_dev(QKV), batch, seq, h, n_heads, causal, n, O_, lse)
    got = from_dev_bf16(O_)
    lse_h = lse.cpu().numpy().reshape(n * hps, M + 128)
    q = f64(QKV)
    for i in range(n):
        Q, K, V = q[i][:, :hs], q[i][:, hs:2 * hs], q[i][:, 2 * hs:]
        ref = O.attention_heads(Q, K, V, batch, seq, hps, causal)
        assert_parity(got[i], ref, f"shard {i}")
        for kk in (0, hps - 1):
            c = slice(kk * d, (kk + 1) * d)
            for s in range(batch):
                r = slice(s * seq, (s + 1) * seq)
                np.testing.assert_allclose(lse_h[i * hps + kk, r] * np.log(2.0),
                                           O.attention_logsumexp(Q[r, c], K[r, c], causal),
                                           rtol=0, atol=2e-3)


def test_attention_first_query_sees_itself(tp):
    """Causal: the first query of every sequence returns its own V row."""
    rng = np.random.default_rng(850)
    batch, seq, h = 3, 130, 128
    QKV = _rand_bits(rng, (1, batch * seq, 3 * h), 4.0)
    O_ = torch.empty((1, batch * seq, h), dtype=torch.int16, device="cuda")
    tp.tp_attention(to_dev(QKV), batch, seq, h, 1, True, 1, O_)
    got = _bits(O_)[0]
    for s in range(batch):
        assert np.array_equal(got[s * seq], QKV[0, s * seq, 2 * h:])


# ------------------------------------------------------------------ errors

def test_device_argument_errors(tp):
    X = torch.zeros(64 * 64 + 8, dtype=torch.int16, device="cuda")
    W = torch.zeros(64 * 64, dtype=torch.int16, device="cuda")
    Y = torch.zeros(64 * 64, dtype=torch.int16, device="cuda")
    with pytest.raises(tp.TPError) as e:
        tp.tp_column_linear(X.data_ptr() + 2, 64, 64, W, None, 64, 1, 0, Y)
    assert e.value.status == tp.TP_ERR_ALIGN
    assert tp.tp_get_last_error() == tp.TP_OK
