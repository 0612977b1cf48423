"""Pins for the fp64 CPU oracle: values and identities fixed by the pages and
by mathematics, independent of the oracle's own code.

Each check is chosen so that a plausible slip in the oracle (tanh-form GeLU,
a dropped bias, a transposed operand, a wrong shard index, a missing 1/sqrt(d)
or causal mask, sample instead of population variance) fails at least one of
them; ``test_planted_mistakes_are_caught`` plants several such slips in the
oracle and checks that they are.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import tp_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# Standard normal CDF at integer points, from a printed normal table.
PHI = {0: 0.5, 1: 0.8413447460685429, 2: 0.9772498680518208,
       3: 0.9986501019683699, -1: 0.15865525393145707,
       -2: 0.022750131948179195}


def _int_matrix(rng, shape, lo=-4, hi=5):
    return rng.integers(lo, hi, size=shape).astype(np.float64)


# ---------------------------------------------------------------- GeLU

def test_gelu_textbook_values():
    for z, phi in PHI.items():
        assert O.gelu(np.array([float(z)]))[0] == pytest.approx(z * phi, abs=1e-15)
    # GeLU(x) -> x for large positive x, -> 0 for large negative x
    assert O.gelu(np.array([12.0]))[0] == 12.0
    assert abs(O.gelu(np.array([-12.0]))[0]) < 1e-30
    # the erf form, not the tanh approximation (which gives 0.841191990607...)
    assert abs(O.gelu(np.array([1.0]))[0] - 0.8411919906082768) > 1e-4


def test_gelu_is_elementwise_per_slice():
    """sigma([Z_1, Z_2]) = [sigma(Z_1), sigma(Z_2)] (TP-LLM, MLP block)."""
    rng = np.random.default_rng(1)
    Z = rng.standard_normal((5, 12))
    whole = O.gelu(Z)
    for n in (1, 2, 3, 4, 6):
        parts = np.concatenate([O.gelu(z) for z in np.split(Z, n, axis=1)], axis=1)
        assert np.array_equal(parts, whole)


# ---------------------------------------------------------------- shard maps

@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_column_and_row_index_maps(n):
    h_in, h_out = 64, 128
    owner, local = O.shard_index_map(O.SPLIT_COLUMN, h_in, h_out, n)
    w = h_out // n
    for i in range(n):                      # shard i = the i-th block of columns
        for j in range(i * w, (i + 1) * w):
            assert owner[j] == i and local[j] == j - i * w
    owner, local = O.shard_index_map(O.SPLIT_ROW, h_in, h_out, n)
    w = h_in // n
    for i in range(n):
        for r in range(i * w, (i + 1) * w):
            assert owner[r] == i and local[r] == r - i * w


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_qkv_head_index_map(n):
    n_heads, d = 16, 4
    h = n_heads * d
    owner, local = O.shard_index_map(O.SPLIT_QKV_HEADS, h, 3 * h, n, d)
    hpg = n_heads // n                      # heads per shard
    for part in range(3):                   # Q, K, V
        for head in range(n_heads):
            shard = head // hpg
            for e in range(d):
                col = part * h + head * d + e
                assert owner[col] == shard
                assert local[col] == part * hpg * d + (head - shard * hpg) * d + e
    # each shard receives exactly 3 h / n columns, all locals distinct
    for i in range(n):
        assert sorted(local[owner == i].tolist()) == list(range(3 * h // n))


def test_index_map_rejects_indivisible():
    with pytest.raises(ValueError):
        O.shard_index_map(O.SPLIT_COLUMN, 8, 12, 5)
    with pytest.raises(ValueError):
        O.shard_index_map(O.SPLIT_ROW, 12, 8, 8)
    with pytest.raises(ValueError):
        O.shard_index_map(O.SPLIT_QKV_HEADS, 12, 36, 8, 4)   # 3 heads, N = 8


def test_packed_shards_are_transposed_slices():
    rng = np.random.default_rng(2)
    W = rng.standard_normal((6, 8))
    p = O.packed_shards(W, O.SPLIT_COLUMN, 2)
    assert p.shape == (2, 4, 6)
    assert np.array_equal(p[1], W[:, 4:8].T)
    p = O.packed_shards(W, O.SPLIT_ROW, 3)
    assert p.shape == (3, 8, 2)
    assert np.array_equal(p[2], W[4:6, :].T)


def test_worked_example_shapes():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_column_parallel_linear.json")))
    X = np.zeros((g["tokens"], g["in_features"]))
    W = np.zeros((g["in_features"], g["out_features"]))
    n = g["tensor_model_parallel_size"]
    shards = O.shard_matrices(W, O.SPLIT_COLUMN, n)
    assert [list(s.shape) for s in shards] == [g["shard_weight_shape"]] * n
    Y = O.column_parallel_linear(X, W, None, n)
    assert [list(y.shape) for y in Y] == [g["shard_output_shape"]] * n
    assert list(np.concatenate(Y, axis=1).shape) == g["full_output_shape"]


# ---------------------------------------------------------------- linear primitives

@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_column_parallel_concat_equals_full(n):
    """Y = [X W_1 ... X W_N] = X W, exact for integer-valued operands."""
    rng = np.random.default_rng(3)
    X, W, b = _int_matrix(rng, (7, 16)), _int_matrix(rng, (16, 32)), _int_matrix(rng, (32,))
    full = X @ W + b
    parts = O.column_parallel_linear(X, W, b, n)
    assert np.array_equal(np.concatenate(parts, axis=1), full)


@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_row_parallel_partials_sum_to_full(n):
    """Y = sum_i X_i W_i = X W, exact for integer-valued operands."""
    rng = np.random.default_rng(4)
    X, W = _int_matrix(rng, (5, 32)), _int_matrix(rng, (32, 12))
    P = O.row_parallel_linear(O.split_columns(X, n), W, n)
    assert all(p.shape == (5, 12) for p in P)
    assert np.array_equal(O.reduce_partials(P), X @ W)
    # a brute-force triple loop of the same product
    ref = np.zeros((5, 12))
    for r in range(5):
        for c in range(12):
            ref[r, c] = sum(X[r, k] * W[k, c] for k in range(32))
    assert np.array_equal(O.reduce_partials(P), ref)


def test_hand_worked_mlp():
    g = json.load(open(os.path.join(GOLDEN, "hand_mlp_2x2_tp2.json")))
    X, A, B = (np.array(g[k], dtype=np.float64) for k in ("X", "A", "B"))
    n = g["n_shards"]
    assert np.array_equal(X @ A, np.array(g["Z"], dtype=np.float64))
    A_i = O.column_parallel_linear(X, A, None, n, act=O.gelu)
    P = O.row_parallel_linear(A_i, B, n)
    np.testing.assert_allclose(P[0], g["P0"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(P[1], g["P1"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.reduce_partials(P), g["Y"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.mlp(X, A, None, B), g["Y"], rtol=0, atol=1e-12)


def test_row_first_split_needs_sync_before_gelu():
    """A row split of the first GEMM yields partial sums, and
    GeLU(sum P_i) != sum GeLU(P_i): the route the method avoids is wrong."""
    g = json.load(open(os.path.join(GOLDEN, "hand_mlp_2x2_tp2.json")))
    X, A = np.array(g["X"], float), np.array(g["A"], float)
    partial = O.row_parallel_linear(O.split_columns(X, 2), A, 2)
    right = O.gelu(O.reduce_partials(partial))
    wrong = O.reduce_partials([O.gelu(p) for p in partial])
    assert np.array_equal(right, O.gelu(X @ A))
    assert np.max(np.abs(right - wrong)) > 0.1


# ---------------------------------------------------------------- brute force

def _phi(x):
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def _brute_mlp(X, A, b1, B, b2, R):
    M, h = X.shape
    F = A.shape[1]
    Y = [[0.0] * h for _ in range(M)]
    for r in range(M):
        act = []
        for f in range(F):
            z = b1[f]
            for k in range(h):
                z += X[r][k] * A[k][f]
            act.append(z * _phi(z))
        for c in range(h):
            y = b2[c] + R[r][c]
            for f in range(F):
                y += act[f] * B[f][c]
            Y[r][c] = y
    return np.array(Y)


@pytest.mark.parametrize("n", [1, 2, 4])
def test_mlp_brute_force(n):
    rng = np.random.default_rng(5)
    M, h, F = 3, 4, 8
    X = rng.standard_normal((M, h))
    A, B = rng.standard_normal((h, F)), rng.standard_normal((F, h))
    b1, b2 = rng.standard_normal(F), rng.standard_normal(h)
    ref = _brute_mlp(X, A, b1, B, b2, X)
    np.testing.assert_allclose(O.mlp(X, A, b1, B, b2, X), ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(O.mlp_sharded(X, A, b1, B, b2, X, n), ref,
                               rtol=1e-12, atol=1e-12)


def _brute_attention(X, Wqkv, bqkv, Wo, bo, R, batch, seq, n_heads, causal):
    M, h = X.shape
    d = h // n_heads
    proj = [[bqkv[c] + sum(X[r][k] * Wqkv[k][c] for k in range(h))
             for c in range(3 * h)] for r in range(M)]
    out = [[0.0] * h for _ in range(M)]
    for s in range(batch):
        for hd in range(n_heads):
            for t in range(seq):
                qi = s * seq + t
                keys = range(t + 1) if causal else range(seq)
                scores = []
                for u in keys:
                    kj = s * seq + u
                    dot = sum(proj[qi][hd * d + e] * proj[kj][h + hd * d + e]
                              for e in range(d))
                    scores.append(dot / math.sqrt(d))
                m = max(scores)
                w = [math.exp(x - m) for x in scores]
                tot = sum(w)
                for e in range(d):
                    out[qi][hd * d + e] = sum(
                        w[j] / tot * proj[s * seq + u][2 * h + hd * d + e]
                        for j, u in enumerate(keys))
    Y = [[bo[c] + R[r][c] + sum(out[r][k] * Wo[k][c] for k in range(h))
          for c in range(h)] for r in range(M)]
    return np.array(Y)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("n", [1, 2, 4])
def test_attention_brute_force(n, causal):
    rng = np.random.default_rng(6)
    batch, seq, n_heads, d = 2, 5, 4, 2
    h = n_heads * d
    X = rng.standard_normal((batch * seq, h))
    Wqkv, bqkv = rng.standard_normal((h, 3 * h)), rng.standard_normal(3 * h)
    Wo, bo = rng.standard_normal((h, h)), rng.standard_normal(h)
    ref = _brute_attention(X, Wqkv, bqkv, Wo, bo, X, batch, seq, n_heads, causal)
    got = O.self_attention(X, Wqkv, bqkv, Wo, bo, X, batch, seq, n_heads, causal)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)
    got = O.self_attention_sharded(X, Wqkv, bqkv, Wo, bo, X, batch, seq,
                                   n_heads, n, causal)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)


def test_attention_closed_forms():
    rng = np.random.default_rng(7)
    batch, seq, n_heads, d = 2, 9, 2, 4
    h = n_heads * d
    M = batch * seq
    K, V = rng.standard_normal((M, h)), rng.standard_normal((M, h))
    # Q = 0: every visible key gets the same score, so causal output row t is
    # the mean of V rows 0..t of its sequence.
    O_ = O.attention_heads(np.zeros((M, h)), K, V, batch, seq, n_heads, True)
    for s in range(batch):
        for t in range(seq):
            rows = V[s * seq:s * seq + t + 1]
            np.testing.assert_allclose(O_[s * seq + t], rows.mean(axis=0), atol=1e-14)
    # the first query of each sequence sees only its own key: output = V row
    Q = rng.standard_normal((M, h)) * 5
    O_ = O.attention_heads(Q, K, V, batch, seq, n_heads, True)
    for s in range(batch):
        assert np.allclose(O_[s * seq], V[s * seq], atol=1e-15)
    # softmax rows sum to one, masked probabilities are exactly zero
    S = rng.standard_normal((6, 6))
    S[np.triu_indices(6, 1)] = -np.inf
    P = O.softmax_rows(S)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-15)
    assert np.all(P[np.triu_indices(6, 1)] == 0.0)
    # two keys with score gap log(3): weights 3/4 and 1/4 (scale 1/sqrt(d))
    q = np.zeros((2, 4)); q[1, 0] = 2.0 * math.log(3.0)
    k = np.zeros((2, 4)); k[0, 0] = 1.0
    v = np.array([[1.0, 0, 0, 0], [0, 1.0, 0, 0]])
    out = O.attention_head(q, k, v, causal=True)
    np.testing.assert_allclose(out[1], [0.75, 0.25, 0, 0], atol=1e-15)


# ---------------------------------------------------------------- LayerNorm

def test_layernorm_closed_forms():
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    s5 = math.sqrt(5.0)
    np.testing.assert_allclose(O.layernorm(x, 1.0, 0.0, eps=0.0),
                               [[-3 / s5, -1 / s5, 1 / s5, 3 / s5]], atol=1e-15)
    rng = np.random.default_rng(8)
    x = rng.standard_normal((4, 64)) * 3 + 2
    eps = 1e-5
    y = O.layernorm(x, np.ones(64), np.zeros(64), eps)
    var = x.var(axis=1)        # population variance (numpy's default ddof=0)
    np.testing.assert_allclose(y.mean(axis=1), 0.0, atol=1e-14)
    np.testing.assert_allclose(y.var(axis=1), var / (var + eps), rtol=1e-12)
    g, b = rng.standard_normal(64), rng.standard_normal(64)
    np.testing.assert_allclose(O.layernorm(x, g, b, eps), y * g + b, atol=1e-13)


# ---------------------------------------------------------------- blocks and rows

@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_sharded_blocks_equal_unsharded(n):
    rng = np.random.default_rng(9)
    batch, seq, n_heads, d, F = 2, 6, 8, 4, 64
    h = n_heads * d
    X = rng.standard_normal((batch * seq, h))
    Wqkv, bqkv = rng.standard_normal((h, 3 * h)) * .2, rng.standard_normal(3 * h)
    Wo, bo = rng.standard_normal((h, h)) * .2, rng.standard_normal(h)
    A, b1 = rng.standard_normal((h, F)) * .2, rng.standard_normal(F)
    B, b2 = rng.standard_normal((F, h)) * .2, rng.standard_normal(h)
    np.testing.assert_allclose(
        O.self_attention_sharded(X, Wqkv, bqkv, Wo, bo, X, batch, seq, n_heads, n),
        O.self_attention(X, Wqkv, bqkv, Wo, bo, X, batch, seq, n_heads),
        rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(O.mlp_sharded(X, A, b1, B, b2, X, n),
                               O.mlp(X, A, b1, B, b2, X), rtol=1e-12, atol=1e-12)


def _layer_params(rng, h, F):
    return dict(Wqkv=rng.standard_normal((h, 3 * h)) * .2, bqkv=rng.standard_normal(3 * h) * .1,
                Wo=rng.standard_normal((h, h)) * .2, bo=rng.standard_normal(h) * .1,
                A=rng.standard_normal((h, F)) * .2, b1=rng.standard_normal(F) * .1,
                B=rng.standard_normal((F, h)) * .2, b2=rng.standard_normal(h) * .1,
                ln1_g=rng.standard_normal(h), ln1_b=rng.standard_normal(h),
                ln2_g=rng.standard_normal(h), ln2_b=rng.standard_normal(h))


def test_layer_composition_brute_force():
    rng = np.random.default_rng(10)
    batch, seq, n_heads, d, F = 1, 4, 2, 2, 8
    h = n_heads * d
    p = _layer_params(rng, h, F)
    X = rng.standard_normal((batch * seq, h))

    def ln(x, g, b):
        out = []
        for row in x:
            mu = sum(row) / len(row)
            var = sum((v - mu) ** 2 for v in row) / len(row)
            out.append([(v - mu) / math.sqrt(var + 1e-5) * g[j] + b[j]
                        for j, v in enumerate(row)])
        return np.array(out)

    x1 = ln(X, p["ln1_g"], p["ln1_b"])
    h1 = _brute_attention(x1, p["Wqkv"], p["bqkv"], p["Wo"], p["bo"], X,
                          batch, seq, n_heads, True)
    x2 = ln(h1, p["ln2_g"], p["ln2_b"])
    ref = _brute_mlp(x2, p["A"], p["b1"], p["B"], p["b2"], h1)
    np.testing.assert_allclose(O.transformer_layer(X, p, batch, seq, n_heads), ref,
                               rtol=1e-10, atol=1e-10)


def test_row_restricted_variants_match_full():
    rng = np.random.default_rng(11)
    batch, seq, n_heads, d, F = 2, 16, 4, 4, 32
    h = n_heads * d
    p = _layer_params(rng, h, F)
    X = rng.standard_normal((batch * seq, h))
    rows = np.array([0, 3, 15, 16, 21, 31])
    np.testing.assert_allclose(
        O.mlp_rows(X, p["A"], p["b1"], p["B"], p["b2"], X, rows),
        O.mlp(X, p["A"], p["b1"], p["B"], p["b2"], X)[rows], rtol=1e-13, atol=1e-13)
    for causal in (True, False):
        np.testing.assert_allclose(
            O.self_attention_rows(X, p["Wqkv"], p["bqkv"], p["Wo"], p["bo"], X,
                                  batch, seq, n_heads, rows, causal),
            O.self_attention(X, p["Wqkv"], p["bqkv"], p["Wo"], p["bo"], X,
                             batch, seq, n_heads, causal)[rows], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(
        O.transformer_layer_rows(X, p, batch, seq, n_heads, rows),
        O.transformer_layer(X, p, batch, seq, n_heads)[rows], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- sensitivity

def test_planted_mistakes_are_caught(monkeypatch):
    """Plant typical slips in the oracle (on the CPU) and check that the pins
    above reject each of them."""
    tanh_gelu = lambda x: 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))
    with monkeypatch.context() as m:
        m.setattr(O, "gelu", tanh_gelu)
        with pytest.raises(AssertionError):
            test_gelu_textbook_values()
    with monkeypatch.context() as m:      # population -> sample variance
        m.setattr(O, "layernorm", lambda x, g, b, eps=1e-5: (x - x.mean(-1, keepdims=True))
                  / np.sqrt(x.var(-1, ddof=1, keepdims=True) + eps) * g + b)
        with pytest.raises(AssertionError):
            test_layernorm_closed_forms()
    with monkeypatch.context() as m:      # forgetting the causal mask
        orig = O.attention_head
        m.setattr(O, "attention_head", lambda q, k, v, causal: orig(q, k, v, False))
        with pytest.raises(AssertionError):
            test_attention_closed_forms()
    with monkeypatch.context() as m:      # forgetting 1/sqrt(d_k)
        def no_scale(q, k, v, causal):
            return orig(q * math.sqrt(q.shape[1]), k, v, causal)
        m.setattr(O, "attention_head", no_scale)
        with pytest.raises(AssertionError):
            test_attention_brute_force(2, True)
    with monkeypatch.context() as m:      # shard i gets the wrong (reversed) block
        orig_map = O.shard_index_map
        def rev(kind, h_in, h_out, n, hd=0):
            own, loc = orig_map(kind, h_in, h_out, n, hd)
            return n - 1 - own, loc
        m.setattr(O, "shard_index_map", rev)
        with pytest.raises(AssertionError):
            test_column_and_row_index_maps(4)
    with monkeypatch.context() as m:      # bias added once per partial
        orig_red = O.reduce_partials
        def per_partial(P, bias=None, residual=None):
            return orig_red(P, None if bias is None else bias * len(P), residual)
        m.setattr(O, "reduce_partials", per_partial)
        with pytest.raises(AssertionError):
            test_mlp_brute_force(2)


# ---------------------------------------------------------------- sequence parallelism

@pytest.mark.parametrize("n", [1, 2, 4])
def test_reduce_scatter_then_all_gather_is_all_reduce(n):
    """[TP-LLM] "Sequence Parallelism": an all-reduce is a reduce-scatter
    followed by an all-gather; exact for integer-valued partials."""
    rng = np.random.default_rng(12)
    batch, seq, h = 3, 8, 5
    P = [_int_matrix(rng, (batch * seq, h)) for _ in range(n)]
    b = _int_matrix(rng, (h,))
    rs = O.reduce_scatter_partials(P, batch, seq, n, b)
    assert all(r.shape == (batch, seq // n, h) for r in rs)
    assert np.array_equal(O.all_gather_sequence(rs, batch, seq), O.reduce_partials(P, b))
    # shard i holds positions [i S/N, (i+1) S/N) of every sequence
    full = O.reduce_partials(P, b).reshape(batch, seq, h)
    for i, r in enumerate(rs):
        for bb in range(batch):
            for s_ in range(seq // n):
                assert np.array_equal(r[bb, s_], full[bb, i * (seq // n) + s_])


@pytest.mark.parametrize("n", [1, 2, 4])
def test_sequence_parallel_layer_equals_standard_layer(n):
    """Sharding LayerNorm, dropout and the residual along the sequence does
    not change the layer's output ([TP-LLM] "Sequence Parallelism": the same
    math with reduce-scatter + all-gather in place of all-reduce)."""
    rng = np.random.default_rng(13)
    batch, seq, n_heads, d, F = 2, 8, 4, 2, 16
    h = n_heads * d
    p = _layer_params(rng, h, F)
    X = rng.standard_normal((batch * seq, h))
    ref = O.transformer_layer(X, p, batch, seq, n_heads)
    out = O.transformer_layer_sp(O.sequence_shard(X, batch, seq, n), p, batch, seq, n_heads, n)
    np.testing.assert_allclose(O.all_gather_sequence(out, batch, seq), ref, rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- SwiGLU

def test_silu_textbook_values():
    e = math.e
    for x, ref in [(0.0, 0.0), (1.0, 1.0 / (1.0 + 1.0 / e)), (-1.0, -1.0 / (1.0 + e)),
                   (2.0, 2.0 / (1.0 + e ** -2))]:
        assert O.silu(np.array([x]))[0] == pytest.approx(ref, rel=1e-15, abs=1e-300)
    # SiLU(x) -> x from below for large x (x e^{-x} ~ 2.8e-12 at x = 30)
    assert 0.0 < 30.0 - O.silu(np.array([30.0]))[0] < 1e-11
    assert O.silu(np.array([1.0]))[0] == pytest.approx(0.7310585786300049, abs=1e-15)
    assert abs(O.silu(np.array([-40.0]))[0]) < 1e-15


def _brute_swiglu(X, Wg, Wu, B, b2, R):
    M, h = X.shape
    F = Wg.shape[1]
    Y = np.zeros((M, B.shape[1]))
    for r in range(M):
        a = []
        for f in range(F):
            g = sum(X[r][k] * Wg[k][f] for k in range(h))
            u = sum(X[r][k] * Wu[k][f] for k in range(h))
            a.append(g / (1.0 + math.exp(-g)) * u)
        for c in range(B.shape[1]):
            Y[r][c] = b2[c] + R[r][c] + sum(a[f] * B[f][c] for f in range(F))
    return Y


@pytest.mark.parametrize("n", [1, 2, 4])
def test_swiglu_brute_force_and_sharded(n):
    rng = np.random.default_rng(14)
    M, h, F = 3, 4, 8
    X = rng.standard_normal((M, h))
    Wg, Wu, B = rng.standard_normal((h, F)), rng.standard_normal((h, F)), rng.standard_normal((F, h))
    b2 = rng.standard_normal(h)
    ref = _brute_swiglu(X, Wg, Wu, B, b2, X)
    np.testing.assert_allclose(O.swiglu_mlp(X, Wg, Wu, B, b2, X), ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(O.swiglu_mlp_sharded(X, Wg, Wu, B, b2, X, n), ref,
                               rtol=1e-12, atol=1e-12)


def test_packed_gate_up_layout():
    rng = np.random.default_rng(15)
    h, F, n = 3, 2 * 256, 2
    Wg, Wu = rng.standard_normal((h, F)), rng.standard_normal((h, F))
    P = O.packed_gate_up(Wg, Wu, n)
    assert P.shape == (n, 2 * F // n, h)
    b = O.GATE_UP_BLOCK
    fs = F // n
    for i in range(n):
        for k in range(fs // b):
            for j in range(b):
                f = i * fs + k * b + j              # global output feature
                assert np.array_equal(P[i, 2 * k * b + j], Wg[:, f])
                assert np.array_equal(P[i, 2 * k * b + b + j], Wu[:, f])


def test_gate_up_index_map_matches_packing():
    rng = np.random.default_rng(16)
    h, F, n = 3, 2 * 256, 2
    Wg, Wu = rng.standard_normal((h, F)), rng.standard_normal((h, F))
    W = np.concatenate([Wg, Wu], axis=1)
    assert np.array_equal(O.packed_shards(W, O.SPLIT_GATE_UP, n), O.packed_gate_up(Wg, Wu, n))
    with pytest.raises(ValueError):
        O.shard_index_map(O.SPLIT_GATE_UP, h, 2 * 192, 2)   # F/N = 96 not a block multiple



# ---------------------------------------------------------------- grouped-query attention

def _gqa_params(rng, h, n_q, n_kv, d):
    cols = (n_q + 2 * n_kv) * d
    return (rng.standard_normal((h, cols)) * .3, rng.standard_normal(cols) * .1,
            rng.standard_normal((n_q * d, h)) * .3, rng.standard_normal(h) * .1)


def test_gqa_with_all_kv_heads_is_multi_head_attention():
    rng = np.random.default_rng(17)
    batch, seq, n, d = 2, 6, 4, 3
    h = n * d
    X = rng.standard_normal((batch * seq, h))
    Wqkv, bqkv, Wo, bo = _gqa_params(rng, h, n, n, d)
    np.testing.assert_allclose(
        O.gqa_self_attention(X, Wqkv, bqkv, Wo, bo, X, batch, seq, n, n),
        O.self_attention(X, Wqkv, bqkv, Wo, bo, X, batch, seq, n), rtol=1e-12, atol=1e-12)


def test_gqa_brute_force_shared_kv():
    """Every query head of a group sees the same K, V: a brute-force loop
    that uses head j // g explicitly."""
    rng = np.random.default_rng(18)
    batch, seq, n_q, n_kv, d = 1, 5, 4, 2, 2
    Q = rng.standard_normal((seq, n_q * d))
    K = rng.standard_normal((seq, n_kv * d))
    V = rng.standard_normal((seq, n_kv * d))
    out = O.gqa_attention_heads(Q, K, V, batch, seq, n_q, n_kv, True)
    for j in range(n_q):
        kv = j // (n_q // n_kv)
        for t in range(seq):
            sc = [sum(Q[t, j * d + e] * K[u, kv * d + e] for e in range(d)) / math.sqrt(d)
                  for u in range(t + 1)]
            m = max(sc)
            w = [math.exp(x - m) for x in sc]
            for e in range(d):
                ref = sum(w[u] * V[u, kv * d + e] for u in range(t + 1)) / sum(w)
                assert abs(out[t, j * d + e] - ref) < 1e-12


@pytest.mark.parametrize("n_q,n_kv,n", [(8, 2, 1), (8, 2, 2), (8, 4, 4), (8, 2, 4), (8, 1, 8),
                                        (8, 2, 8)])
def test_gqa_sharded_equals_unsharded(n_q, n_kv, n):
    """Including N > n_kv, where kv heads are duplicated across shards."""
    rng = np.random.default_rng(19)
    batch, seq, d = 2, 5, 2
    h = n_q * d
    X = rng.standard_normal((batch * seq, h))
    Wqkv, bqkv, Wo, bo = _gqa_params(rng, h, n_q, n_kv, d)
    np.testing.assert_allclose(
        O.gqa_self_attention_sharded(X, Wqkv, bqkv, Wo, bo, X, batch, seq, n_q, n_kv, n),
        O.gqa_self_attention(X, Wqkv, bqkv, Wo, bo, X, batch, seq, n_q, n_kv),
        rtol=1e-12, atol=1e-12)


def test_gqa_shard_columns_and_constraints():
    cols = O.gqa_shard_columns(8, 2, 1, 4)      # N = 4 > n_kv = 2: duplication
    # shard 0, 1 use kv head 0; shards 2, 3 kv head 1 (K at 8 + kv, V at 10 + kv)
    assert [c.tolist() for c in cols] == [[0, 1, 8, 10], [2, 3, 8, 10], [4, 5, 9, 11],
                                         [6, 7, 9, 11]]
    with pytest.raises(ValueError):
        O.gqa_shard_columns(8, 4, 1, 3)          # 8 % 3
    with pytest.raises(ValueError):
        O.gqa_kv_local(4, 6)                     # N = 6 neither divides nor is divided by 4



# ---------------------------------------------------------------- MLP backward

def test_gelu_grad_values_and_finite_difference():
    assert O.gelu_grad(np.array([0.0]))[0] == pytest.approx(0.5, abs=1e-15)
    # Phi(1) + phi(1) = 0.8413447460685429 + 0.24197072451914337 (normal table values)
    assert O.gelu_grad(np.array([1.0]))[0] == pytest.approx(0.8413447460685429 + 0.24197072451914337,
                                                            abs=1e-14)
    assert O.gelu_grad(np.array([12.0]))[0] == pytest.approx(1.0, abs=1e-12)
    assert abs(O.gelu_grad(np.array([-12.0]))[0]) < 1e-20
    z = np.linspace(-4, 4, 41)
    eps = 1e-6
    fd = (O.gelu(z + eps) - O.gelu(z - eps)) / (2 * eps)
    np.testing.assert_allclose(O.gelu_grad(z), fd, atol=1e-8)


def _mlp_loss(X, A, b1, B, b2, dY):
    return float(np.sum(O.mlp(X, A, b1, B, b2, X) * dY))


def test_mlp_backward_matches_finite_differences():
    """Every gradient against central differences of <Y, dY> (an independent
    check of the chain rule, the transposes and the residual term)."""
    rng = np.random.default_rng(20)
    M, h, F = 3, 4, 6
    X, A, B = rng.standard_normal((M, h)), rng.standard_normal((h, F)) * .5, rng.standard_normal((F, h)) * .5
    b1, b2 = rng.standard_normal(F) * .1, rng.standard_normal(h) * .1
    dY = rng.standard_normal((M, h))
    g = O.mlp_backward(X, A, b1, B, dY)
    eps = 1e-6
    for name, arr in (("dX", X), ("dA", A), ("db1", b1), ("dB", B), ("db2", b2)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + eps
            up = _mlp_loss(X, A, b1, B, b2, dY)
            arr[idx] = orig - eps
            dn = _mlp_loss(X, A, b1, B, b2, dY)
            arr[idx] = orig
            num[idx] = (up - dn) / (2 * eps)
        np.testing.assert_allclose(g[name], num, rtol=1e-6, atol=1e-7, err_msg=name)


@pytest.mark.parametrize("n", [1, 2, 3, 6])
def test_mlp_backward_sharded_equals_unsharded(n):
    rng = np.random.default_rng(21)
    M, h, F = 5, 4, 12
    X, A, B = rng.standard_normal((M, h)), rng.standard_normal((h, F)), rng.standard_normal((F, h))
    b1, dY = rng.standard_normal(F), rng.standard_normal((M, h))
    ref = O.mlp_backward(X, A, b1, B, dY)
    got = O.mlp_backward_sharded(X, A, b1, B, dY, n)
    for k in ("dX", "dA", "db1", "dB", "db2"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-12, atol=1e-12, err_msg=k)
    assert len(got["dX_partials"]) == n and all(p.shape == (M, h) for p in got["dX_partials"])


# ---------------------------------------------------------------- attention and layer backward

def _num_grad(loss, arr, eps=1e-6):
    """Central differences of loss() with respect to every element of arr."""
    num = np.zeros_like(arr)
    for idx in np.ndindex(arr.shape):
        orig = arr[idx]
        arr[idx] = orig + eps
        up = loss()
        arr[idx] = orig - eps
        dn = loss()
        arr[idx] = orig
        num[idx] = (up - dn) / (2 * eps)
    return num


@pytest.mark.parametrize("causal", [True, False])
def test_attention_head_backward_matches_finite_differences(causal):
    rng = np.random.default_rng(30)
    T, d = 5, 4
    Q, K, V = (rng.standard_normal((T, d)) for _ in range(3))
    dO = rng.standard_normal((T, d))
    dQ, dK, dV = O.attention_head_backward(Q, K, V, dO, causal)
    loss = lambda: float(np.sum(O.attention_head(Q, K, V, causal) * dO))  # noqa: E731
    for name, g, arr in (("dQ", dQ, Q), ("dK", dK, K), ("dV", dV, V)):
        np.testing.assert_allclose(g, _num_grad(loss, arr), rtol=1e-6, atol=1e-8, err_msg=name)


@pytest.mark.parametrize("causal", [True, False])
def test_attention_head_backward_closed_forms(causal):
    """Exact identities of the softmax attention gradient: every softmax row
    sums to 1, so sum_j dV_j = sum_i dO_i; adding one vector to every key
    leaves each softmax row unchanged, so sum_j dK_j = 0; the first causal
    query attends to one key with weight 1, so its dQ row is 0."""
    rng = np.random.default_rng(31)
    T, d = 7, 4
    Q, K, V, dO = (rng.standard_normal((T, d)) for _ in range(4))
    dQ, dK, dV = O.attention_head_backward(Q, K, V, dO, causal)
    np.testing.assert_allclose(dV.sum(axis=0), dO.sum(axis=0), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dK.sum(axis=0), np.zeros(d), rtol=0, atol=1e-12)
    if causal:
        assert np.all(dQ[0] == 0.0)
        # the last key is seen by the last query only: dV_last = P[last, last] dO_last
        S = Q[-1] @ K.T / math.sqrt(d)
        p_last = math.exp(S[-1] - S.max()) / np.exp(S - S.max()).sum()
        np.testing.assert_allclose(dV[-1], p_last * dO[-1], rtol=1e-12, atol=1e-14)


def test_self_attention_backward_matches_finite_differences():
    rng = np.random.default_rng(32)
    b, s, h, nh = 2, 3, 4, 2
    X = rng.standard_normal((b * s, h))
    Wqkv, Wo = rng.standard_normal((h, 3 * h)) * .4, rng.standard_normal((h, h)) * .4
    bqkv, bo = rng.standard_normal(3 * h) * .1, rng.standard_normal(h) * .1
    dY = rng.standard_normal((b * s, h))
    g = O.self_attention_backward(X, Wqkv, bqkv, Wo, bo, dY, b, s, nh)
    loss = lambda: float(np.sum(O.self_attention(X, Wqkv, bqkv, Wo, bo, X, b, s, nh) * dY))  # noqa: E731
    for name, arr in (("dX", X), ("dWqkv", Wqkv), ("dbqkv", bqkv), ("dWo", Wo), ("dbo", bo)):
        np.testing.assert_allclose(g[name], _num_grad(loss, arr), rtol=1e-6, atol=1e-8,
                                   err_msg=name)


@pytest.mark.parametrize("n", [1, 2, 4])
def test_self_attention_backward_sharded_equals_unsharded(n):
    rng = np.random.default_rng(33)
    b, s, h, nh = 2, 5, 16, 4
    X = rng.standard_normal((b * s, h))
    Wqkv, Wo = rng.standard_normal((h, 3 * h)) * .3, rng.standard_normal((h, h)) * .3
    bqkv, bo = rng.standard_normal(3 * h) * .1, rng.standard_normal(h) * .1
    dY = rng.standard_normal((b * s, h))
    ref = O.self_attention_backward(X, Wqkv, bqkv, Wo, bo, dY, b, s, nh)
    got = O.self_attention_backward_sharded(X, Wqkv, bqkv, Wo, bo, dY, b, s, nh, n)
    for k in ("dX", "dWqkv", "dbqkv", "dWo", "dbo"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-12, atol=1e-12, err_msg=k)
    assert len(got["dX_partials"]) == n
    # the one reduction: the partials sum to dX - dY
    np.testing.assert_allclose(sum(got["dX_partials"]), ref["dX"] - dY, rtol=1e-12, atol=1e-12)


def test_layernorm_backward_matches_finite_differences_and_identities():
    rng = np.random.default_rng(34)
    x = rng.standard_normal((3, 6)) * 2 + 1
    gamma, beta = rng.standard_normal(6), rng.standard_normal(6)
    dy = rng.standard_normal((3, 6))
    dx, dg, db = O.layernorm_backward(x, gamma, dy, 1e-5)
    loss = lambda: float(np.sum(O.layernorm(x, gamma, beta, 1e-5) * dy))  # noqa: E731
    np.testing.assert_allclose(dx, _num_grad(loss, x), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dg, _num_grad(loss, gamma), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(db, _num_grad(loss, beta), rtol=1e-6, atol=1e-8)
    # LN is invariant to shifting a row and (with eps = 0) to scaling it, so
    # each row of dx is orthogonal to the ones vector and to the row itself
    dx0, _, _ = O.layernorm_backward(x, gamma, dy, 0.0)
    np.testing.assert_allclose(dx0.sum(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose((dx0 * x).sum(axis=1), 0.0, atol=1e-11)


def test_transformer_layer_backward_matches_finite_differences():
    """The tensor-parallel layer backward (N = 2) against central differences
    of <Y, dY> through the unsharded layer definition."""
    rng = np.random.default_rng(35)
    b, s, h, nh, F, n = 1, 3, 4, 2, 8, 2
    X = rng.standard_normal((b * s, h))
    p = dict(Wqkv=rng.standard_normal((h, 3 * h)) * .4, bqkv=rng.standard_normal(3 * h) * .1,
             Wo=rng.standard_normal((h, h)) * .4, bo=rng.standard_normal(h) * .1,
             A=rng.standard_normal((h, F)) * .4, b1=rng.standard_normal(F) * .1,
             B=rng.standard_normal((F, h)) * .4, b2=rng.standard_normal(h) * .1,
             ln1_g=1 + rng.standard_normal(h) * .1, ln1_b=rng.standard_normal(h) * .1,
             ln2_g=1 + rng.standard_normal(h) * .1, ln2_b=rng.standard_normal(h) * .1)
    dY = rng.standard_normal((b * s, h))
    g = O.transformer_layer_backward(X, p, dY, b, s, nh, n)
    loss = lambda: float(np.sum(O.transformer_layer(X, p, b, s, nh) * dY))  # noqa: E731
    np.testing.assert_allclose(g["dX"], _num_grad(loss, X), rtol=1e-5, atol=1e-7, err_msg="dX")
    for key, name in (("Wqkv", "dWqkv"), ("bqkv", "dbqkv"), ("Wo", "dWo"), ("bo", "dbo"),
                      ("A", "dA"), ("b1", "db1"), ("B", "dB"), ("b2", "db2"),
                      ("ln1_g", "dln1_g"), ("ln1_b", "dln1_b"), ("ln2_g", "dln2_g"),
                      ("ln2_b", "dln2_b")):
        np.testing.assert_allclose(g[name], _num_grad(loss, p[key]), rtol=1e-5, atol=1e-7,
                                   err_msg=name)


def test_attention_logsumexp_closed_forms():
    """Q = 0 makes every score 0, so causal row t sums t + 1 ones (ln(t + 1))
    and a full row sums T ones; one key scored log 3 above the other gives
    ln(e^a + 3 e^a)."""
    T, d = 6, 4
    K = np.random.default_rng(36).standard_normal((T, d))
    np.testing.assert_allclose(O.attention_logsumexp(np.zeros((T, d)), K, True),
                               np.log(np.arange(1, T + 1)), rtol=0, atol=1e-15)
    np.testing.assert_allclose(O.attention_logsumexp(np.zeros((T, d)), K, False),
                               np.full(T, math.log(T)), rtol=0, atol=1e-15)
    q = np.array([[2.0, 0.0]])                     # d = 2: scores k . q / sqrt 2
    k = np.array([[0.0, 0.0], [math.log(3) * math.sqrt(2) / 2, 0.0]])
    assert O.attention_logsumexp(q, k, False)[0] == pytest.approx(math.log(4.0), abs=1e-14)


def test_gqa_attention_backward_matches_finite_differences():
    rng = np.random.default_rng(37)
    b, s, d, nq, nkv = 1, 4, 2, 4, 2
    h = nq * d
    X = rng.standard_normal((b * s, h))
    Wqkv = rng.standard_normal((h, (nq + 2 * nkv) * d)) * .4
    bqkv = rng.standard_normal((nq + 2 * nkv) * d) * .1
    Wo, bo = rng.standard_normal((h, h)) * .4, rng.standard_normal(h) * .1
    dY = rng.standard_normal((b * s, h))
    g = O.gqa_self_attention_backward(X, Wqkv, bqkv, Wo, bo, dY, b, s, nq, nkv)
    loss = lambda: float(np.sum(O.gqa_self_attention(X, Wqkv, bqkv, Wo, bo, X, b, s, nq, nkv) * dY))  # noqa: E731
    for name, arr in (("dX", X), ("dWqkv", Wqkv), ("dbqkv", bqkv), ("dWo", Wo), ("dbo", bo)):
        np.testing.assert_allclose(g[name], _num_grad(loss, arr), rtol=1e-6, atol=1e-8,
                                   err_msg=name)


@pytest.mark.parametrize("n,nkv", [(1, 2), (2, 2), (4, 2), (8, 2), (4, 4), (2, 8)])
def test_gqa_attention_backward_sharded_equals_unsharded(n, nkv):
    """Whole groups per shard (N <= n_kv) and duplicated kv heads (N > n_kv):
    the replicas' weight gradients sum to the logical ones."""
    rng = np.random.default_rng(38 + n)
    b, s, d, nq = 2, 5, 2, 8
    h = nq * d
    X = rng.standard_normal((b * s, h))
    Wqkv = rng.standard_normal((h, (nq + 2 * nkv) * d)) * .3
    bqkv = rng.standard_normal((nq + 2 * nkv) * d) * .1
    Wo, bo = rng.standard_normal((h, h)) * .3, rng.standard_normal(h) * .1
    dY = rng.standard_normal((b * s, h))
    ref = O.gqa_self_attention_backward(X, Wqkv, bqkv, Wo, bo, dY, b, s, nq, nkv)
    got = O.gqa_self_attention_backward_sharded(X, Wqkv, bqkv, Wo, bo, dY, b, s, nq, nkv, n)
    for k in ("dX", "dWqkv", "dbqkv", "dWo", "dbo"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-11, atol=1e-11, err_msg=k)
    # with n_kv = n_q GQA is multi-head attention
    if nkv == nq:
        mha = O.self_attention_backward(X, Wqkv, bqkv, Wo, bo, dY, b, s, nq)
        np.testing.assert_allclose(ref["dX"], mha["dX"], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n", [1, 2, 4])
def test_transformer_layer_sp_backward_is_the_sharded_layer_backward(n):
    """Sequence parallelism only moves rows: the SP backward's dX slices are
    the slices of the standard layer backward's dX and every parameter
    gradient is the same (up to summation order)."""
    rng = np.random.default_rng(39 + n)
    b, s, h, nh, F = 2, 8, 8, 4, 16
    X = rng.standard_normal((b * s, h))
    p = dict(Wqkv=rng.standard_normal((h, 3 * h)) * .4, bqkv=rng.standard_normal(3 * h) * .1,
             Wo=rng.standard_normal((h, h)) * .4, bo=rng.standard_normal(h) * .1,
             A=rng.standard_normal((h, F)) * .4, b1=rng.standard_normal(F) * .1,
             B=rng.standard_normal((F, h)) * .4, b2=rng.standard_normal(h) * .1,
             ln1_g=1 + rng.standard_normal(h) * .1, ln1_b=rng.standard_normal(h) * .1,
             ln2_g=1 + rng.standard_normal(h) * .1, ln2_b=rng.standard_normal(h) * .1)
    dY = rng.standard_normal((b * s, h))
    ref = O.transformer_layer_backward(X, p, dY, b, s, nh, n)
    got = O.transformer_layer_sp_backward(O.sequence_shard(X, b, s, n), p,
                                          O.sequence_shard(dY, b, s, n), b, s, nh, n)
    np.testing.assert_allclose(O.all_gather_sequence(got["dX"], b, s), ref["dX"], rtol=1e-12,
                               atol=1e-12)
    for k in ("dWqkv", "dbqkv", "dWo", "dbo", "dA", "db1", "dB", "db2", "dln1_g", "dln1_b",
              "dln2_g", "dln2_b"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-12, atol=1e-12, err_msg=k)
    # and the SP forward's h1 is the standard layer's h1, sliced
    h1 = O.transformer_layer_sp_block_out(O.sequence_shard(X, b, s, n), p, b, s, nh, n)
    x1 = O.layernorm(X, p["ln1_g"], p["ln1_b"])
    ref_h1 = O.self_attention(x1, p["Wqkv"], p["bqkv"], p["Wo"], p["bo"], X, b, s, nh)
    np.testing.assert_allclose(O.all_gather_sequence(h1, b, s), ref_h1, rtol=1e-12, atol=1e-12)
