"""CPU oracle for the Megatron-LM tensor-parallel Transformer layer (fp64).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or run
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code with the CUDA library and imports nothing from it; it receives plain
numpy arrays (bf16 inputs widened exactly to float64) and computes in float64
with no intermediate rounding.

Sources (web pages on Megatron-LM tensor parallelism), cited by title and
section:
  [TP-LLM]  "Tensor Parallelism in Large Language Models: How Megatron-LM
            Partitions Multi-Layer Perceptrons and Attention Heads"
            (llms.blog), sections "The Core Primitives", "Partitioning the
            Multi-Layer Perceptron (MLP) Block", "Partitioning Multi-Head and
            Grouped-Query Attention", "Sequence Parallelism".
  [M-LM]    "Megatron-LM" (ai360xpert.com), section "How It Works".
  [INTRO]   "Introduction to Megatron-LM" (apxml.com course chapter),
            "Core Contributions" and its ColumnParallelLinear example.
  [FANOUT]  "Megatron-LM: Training Multi-Billion Parameter Language Models
            Using Model Parallelism" (fanout.sh), "What you will learn".

Readings where the pages are silent (each is listed with its reason in the
design notes of the repository):
  * GeLU is the erf form 0.5 x (1 + erf(x / sqrt 2)).
  * The column-parallel bias is sliced with the columns and added before the
    activation; the row-parallel bias is added once, after the sum.
  * The residual is added once, after the sum.
  * Causal attention: query t of a sequence sees keys 0..t of the same
    sequence; attention never crosses sequences.
  * LayerNorm uses the population variance and eps = 1e-5 unless given.
  * The layer is pre-LN: h1 = X + Attn(LN1(X)); Y = h1 + MLP(LN2(h1)).
  * Dropout is the identity (forward pass).

Every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, brute-force scalar loops, textbook values and the identities
the pages state.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

SPLIT_COLUMN = 0
SPLIT_ROW = 1
SPLIT_QKV_HEADS = 2
SPLIT_GATE_UP = 3

# gate / up columns are packed in blocks of this many output features
GATE_UP_BLOCK = 128


# --------------------------------------------------------------------------
# elementwise pieces
# --------------------------------------------------------------------------

def gelu(x: np.ndarray) -> np.ndarray:
    """GeLU(x) = x * Phi(x), Phi the standard normal CDF, in its erf form.

    The pages name "GeLU" only ([M-LM] "How It Works", [TP-LLM] MLP block);
    the erf form is the plainest reading.
    """
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def layernorm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray,
              eps: float = 1e-5) -> np.ndarray:
    """Per-token LayerNorm over the hidden dimension, population variance.

    [TP-LLM] "Sequence Parallelism": LayerNorm is replicated on every
    tensor-parallel rank and acts along h independently for every token.
    """
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * gamma + beta


def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row softmax, max-subtracted; -inf entries get probability exactly 0."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# the shard index maps ([TP-LLM] "The Core Primitives"; attention section)
# --------------------------------------------------------------------------

def _check_div(what: str, value: int, n: int) -> None:
    if n <= 0 or value % n != 0:
        raise ValueError(f"{what}={value} is not divisible by N={n}")


def shard_index_map(kind: int, h_in: int, h_out: int, n_shards: int,
                    head_dim: int = 0):
    """Which shard owns each split index, and its position inside the shard.

    * column split: W = [W_1 ... W_N] along H_out, each W_i of width
      H_out / N ([TP-LLM] "Column-Parallel Linear Layer"); index = column.
    * row split: W = [W_1; ...; W_N] along H_in, each of height H_in / N
      ([TP-LLM] "Row-Parallel Linear Layer"); index = row.
    * QKV head split: W_QKV = [W_Q | W_K | W_V] (each h x h, h = h_out / 3);
      shard i owns heads [i n_h/N, (i+1) n_h/N) of each projection, head k
      being columns [k d, (k+1) d) ([TP-LLM] "Partitioning Multi-Head ...
      Attention", Q, K, V projections). Inside a shard the local columns are
      ordered [Q_i | K_i | V_i]. index = column of W_QKV.

    Returns (owner, local) int64 arrays over the split index.
    """
    if kind == SPLIT_COLUMN:
        _check_div("h_out", h_out, n_shards)
        w = h_out // n_shards
        j = np.arange(h_out, dtype=np.int64)
        return j // w, j % w
    if kind == SPLIT_ROW:
        _check_div("h_in", h_in, n_shards)
        w = h_in // n_shards
        r = np.arange(h_in, dtype=np.int64)
        return r // w, r % w
    if kind == SPLIT_QKV_HEADS:
        if h_out % 3 != 0:
            raise ValueError("QKV weight must have 3h columns")
        h = h_out // 3
        if head_dim <= 0 or h % head_dim != 0:
            raise ValueError("h must be a multiple of head_dim")
        n_heads = h // head_dim
        _check_div("n_heads", n_heads, n_shards)
        hs = h // n_shards                 # columns of one projection per shard
        j = np.arange(h_out, dtype=np.int64)
        part, within_part = j // h, j % h  # part 0 = Q, 1 = K, 2 = V
        head = within_part // head_dim
        owner = head // (n_heads // n_shards)
        local = part * hs + (within_part - owner * hs)
        return owner, local
    if kind == SPLIT_GATE_UP:
        # W = [W_gate | W_up] (h_out = 2F): both column-parallel; a shard's
        # columns alternate GATE_UP_BLOCK gate features and the same up ones
        if h_out % 2 != 0:
            raise ValueError("gate/up weight must have 2F columns")
        F = h_out // 2
        _check_div("F", F, n_shards)
        fs = F // n_shards
        if fs % GATE_UP_BLOCK != 0:
            raise ValueError("F/N must be a multiple of the gate/up block")
        j = np.arange(h_out, dtype=np.int64)
        part, f = j // F, j % F                # part 0 = gate, 1 = up
        owner = f // fs
        within = f % fs
        local = (within // GATE_UP_BLOCK) * 2 * GATE_UP_BLOCK + part * GATE_UP_BLOCK + \
            within % GATE_UP_BLOCK
        return owner, local
    raise ValueError(f"unknown split kind {kind}")


def shard_matrices(W: np.ndarray, kind: int, n_shards: int,
                   head_dim: int = 0) -> list:
    """The N logical shards W_i (H_in x H_out/N, or H_in/N x H_out, or the
    head-sliced [Q_i | K_i | V_i] of width 3h/N), built from the index map."""
    h_in, h_out = W.shape
    owner, local = shard_index_map(kind, h_in, h_out, n_shards, head_dim)
    shards = []
    for i in range(n_shards):
        sel = np.nonzero(owner == i)[0]
        order = sel[np.argsort(local[sel], kind="stable")]
        shards.append(W[order, :] if kind == SPLIT_ROW else W[:, order])
    return shards


def packed_shards(W: np.ndarray, kind: int, n_shards: int,
                  head_dim: int = 0) -> np.ndarray:
    """Byte layout the GPU consumes: shard i stored transposed (K-major),
    i.e. out[i] = W_i^T, shape [N, cols_per_shard, rows_per_shard]."""
    return np.stack([np.ascontiguousarray(s.T)
                     for s in shard_matrices(W, kind, n_shards, head_dim)])


def shard_vector(b: np.ndarray, kind: int, n_shards: int,
                 head_dim: int = 0) -> np.ndarray:
    """A column bias sliced like the columns it belongs to: [N, H_out/N]."""
    return packed_shards(np.asarray(b).reshape(1, -1), kind, n_shards,
                         head_dim)[:, :, 0]


# --------------------------------------------------------------------------
# the parallel linear primitives ([TP-LLM] "The Core Primitives")
# --------------------------------------------------------------------------

def linear(X: np.ndarray, W: np.ndarray, b=None) -> np.ndarray:
    """Y = X W (+ b), X in R^{B x H_in}, W in R^{H_in x H_out}."""
    Y = np.asarray(X, dtype=np.float64) @ np.asarray(W, dtype=np.float64)
    if b is not None:
        Y = Y + b
    return Y


def column_parallel_linear(X, W, b, n_shards: int, act=None,
                           kind: int = SPLIT_COLUMN, head_dim: int = 0) -> list:
    """Y_i = act(X W_i + b_i) on every shard; X is replicated, no exchange.

    [TP-LLM] "Column-Parallel Linear Layer" (Y_i = X W_i) and its note that an
    element-wise function can be applied to the local slice; [M-LM] step 1
    (GeLU(X A_i) per GPU).
    """
    Ws = shard_matrices(W, kind, n_shards, head_dim)
    bs = (shard_matrices(np.asarray(b).reshape(1, -1), kind, n_shards,
                         head_dim) if b is not None else [None] * n_shards)
    out = []
    for Wi, bi in zip(Ws, bs):
        Yi = linear(X, Wi, None if bi is None else bi[0])
        out.append(act(Yi) if act is not None else Yi)
    return out


def row_parallel_linear(X_shards: list, W: np.ndarray, n_shards: int) -> list:
    """Partial products Y_i = X_i W_i, each full size B x H_out.

    [TP-LLM] "Row-Parallel Linear Layer" (Y_i = X_i W_i); [M-LM] step 2.
    """
    Ws = shard_matrices(W, SPLIT_ROW, n_shards)
    return [linear(Xi, Wi) for Xi, Wi in zip(X_shards, Ws)]


def reduce_partials(partials: list, bias=None, residual=None) -> np.ndarray:
    """Y = sum_i Y_i (+ b) (+ R): the all-reduce sum of the row-parallel
    partials ([TP-LLM] "Row-Parallel Linear Layer", Y = sum_i Y_i = XW;
    [M-LM] step 3), with the output bias and the residual added once."""
    Y = np.zeros_like(partials[0])
    for P in partials:
        Y = Y + P
    if bias is not None:
        Y = Y + bias
    if residual is not None:
        Y = Y + residual
    return Y


def split_columns(X: np.ndarray, n_shards: int) -> list:
    """X = [X_1 ... X_N] along its channel dimension ([TP-LLM] row-parallel
    input)."""
    _check_div("channels", X.shape[1], n_shards)
    w = X.shape[1] // n_shards
    return [X[:, i * w:(i + 1) * w] for i in range(n_shards)]


# --------------------------------------------------------------------------
# blocks, unsharded (the definition) and sharded (the method)
# --------------------------------------------------------------------------

def mlp(X, A, b1, B, b2=None, residual=None) -> np.ndarray:
    """MLP(X) = GeLU(X A + b1) B + b2 (+ R), unsharded.

    [M-LM] "How It Works" (Y = GeLU(X A) B); [TP-LLM] MLP block
    (sigma(X W_in) W_out, W_in h x 4h, W_out 4h x h).
    """
    return reduce_partials([linear(gelu(linear(X, A, b1)), B)], b2, residual)


def mlp_sharded(X, A, b1, B, b2, residual, n_shards: int) -> np.ndarray:
    """The tensor-parallel route: column-parallel A with per-shard bias+GeLU,
    row-parallel B, one sum of the N partials ([TP-LLM] "Partitioning the
    Multi-Layer Perceptron (MLP) Block" steps 1-4)."""
    A_i = column_parallel_linear(X, A, b1, n_shards, act=gelu)
    P_i = row_parallel_linear(A_i, B, n_shards)
    return reduce_partials(P_i, b2, residual)


def attention_head(Q: np.ndarray, K: np.ndarray, V: np.ndarray,
                   causal: bool) -> np.ndarray:
    """softmax(Q K^T / sqrt(d_k)) V for one head of one sequence
    ([TP-LLM] "Local Self-Attention Computation"); with ``causal`` query t
    sees keys 0..t only."""
    d = Q.shape[1]
    S = (Q @ K.T) / math.sqrt(d)
    if causal:
        t = np.arange(Q.shape[0])[:, None]
        s = np.arange(K.shape[0])[None, :]
        S = np.where(s <= t, S, -np.inf)
    return softmax_rows(S) @ V


def attention_heads(Q, K, V, batch: int, seq: int, n_heads: int,
                    causal: bool) -> np.ndarray:
    """Every (sequence, head) pair independently; head k is columns
    [k d, (k+1) d); the head outputs are concatenated in head order."""
    M, h = Q.shape
    d = h // n_heads
    O = np.zeros((M, h))
    for s in range(batch):
        r = slice(s * seq, (s + 1) * seq)
        for k in range(n_heads):
            c = slice(k * d, (k + 1) * d)
            O[r, c] = attention_head(Q[r, c], K[r, c], V[r, c], causal)
    return O


def self_attention(X, Wqkv, bqkv, Wo, bo, residual, batch: int, seq: int,
                   n_heads: int, causal: bool = True) -> np.ndarray:
    """Multi-head self-attention block, unsharded:
    [Q|K|V] = X [W_Q|W_K|W_V] + b_QKV; O = concat_k head_k; Y = O W_O + b_O
    (+ R). [TP-LLM] "Partitioning Multi-Head and Grouped-Query Attention"
    (d_k = h / h_heads)."""
    h = X.shape[1]
    QKV = linear(X, Wqkv, bqkv)
    O = attention_heads(QKV[:, :h], QKV[:, h:2 * h], QKV[:, 2 * h:],
                        batch, seq, n_heads, causal)
    return reduce_partials([linear(O, Wo)], bo, residual)


def self_attention_sharded(X, Wqkv, bqkv, Wo, bo, residual, batch: int,
                           seq: int, n_heads: int, n_shards: int,
                           causal: bool = True) -> np.ndarray:
    """The tensor-parallel route: QKV column-parallel by whole heads, local
    attention for the shard's heads, heads concatenated locally, W_O
    row-parallel, one sum of the partials ([TP-LLM] attention steps 1-4)."""
    h = X.shape[1]
    d = h // n_heads
    hs = h // n_shards
    QKV_i = column_parallel_linear(X, Wqkv, bqkv, n_shards,
                                   kind=SPLIT_QKV_HEADS, head_dim=d)
    O_i = [attention_heads(q[:, :hs], q[:, hs:2 * hs], q[:, 2 * hs:],
                           batch, seq, n_heads // n_shards, causal)
           for q in QKV_i]
    P_i = row_parallel_linear(O_i, Wo, n_shards)
    return reduce_partials(P_i, bo, residual)


def transformer_layer(X, p: dict, batch: int, seq: int, n_heads: int,
                      eps: float = 1e-5, causal: bool = True) -> np.ndarray:
    """Pre-LN layer: h1 = X + Attn(LN1(X)); Y = h1 + MLP(LN2(h1)).

    LayerNorm, dropout (identity here) and the residual adds are replicated
    around the two tensor-parallel blocks ([TP-LLM] "Sequence Parallelism",
    standard formulation).
    """
    x1 = layernorm(X, p["ln1_g"], p["ln1_b"], eps)
    h1 = self_attention(x1, p["Wqkv"], p["bqkv"], p["Wo"], p["bo"], X,
                        batch, seq, n_heads, causal)
    x2 = layernorm(h1, p["ln2_g"], p["ln2_b"], eps)
    return mlp(x2, p["A"], p["b1"], p["B"], p["b2"], h1)


# --------------------------------------------------------------------------
# gated MLP (SwiGLU) ([TP-LLM] MLP block, gated architectures)
# --------------------------------------------------------------------------

def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x * sigmoid(x) = x / (1 + exp(-x))."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def swiglu_mlp(X, W_gate, W_up, B, b2=None, residual=None) -> np.ndarray:
    """(SiLU(X W_gate) * (X W_up)) B + b2 (+ R), unsharded. [TP-LLM] "For
    gated architectures like SwiGLU ... SiLU(X W_gate,i) (.) (X W_up,i)"."""
    return reduce_partials([linear(silu(linear(X, W_gate)) * linear(X, W_up), B)],
                           b2, residual)


def swiglu_mlp_sharded(X, W_gate, W_up, B, b2, residual, n_shards: int) -> np.ndarray:
    """Gate and up both column-parallel, the gated product local to each
    shard, B row-parallel, one sum of the partials."""
    G_i = column_parallel_linear(X, W_gate, None, n_shards)
    U_i = column_parallel_linear(X, W_up, None, n_shards)
    A_i = [silu(g) * u for g, u in zip(G_i, U_i)]
    return reduce_partials(row_parallel_linear(A_i, B, n_shards), b2, residual)


def packed_gate_up(W_gate: np.ndarray, W_up: np.ndarray, n_shards: int) -> np.ndarray:
    """Byte layout of the fused gate/up column-parallel weights: for shard i
    the column shards W_gate,i and W_up,i (F/N columns each), interleaved in
    blocks of GATE_UP_BLOCK output features - block k holds gate features
    [k b, (k+1) b) then the same up features - and stored transposed:
    shape [N, 2 F/N, h]."""
    G = shard_matrices(W_gate, SPLIT_COLUMN, n_shards)
    U = shard_matrices(W_up, SPLIT_COLUMN, n_shards)
    fs = G[0].shape[1]
    if fs % GATE_UP_BLOCK:
        raise ValueError("F/N must be a multiple of the gate/up block")
    out = []
    for g, u in zip(G, U):
        cols = []
        for k in range(fs // GATE_UP_BLOCK):
            sl = slice(k * GATE_UP_BLOCK, (k + 1) * GATE_UP_BLOCK)
            cols += [g[:, sl], u[:, sl]]
        out.append(np.ascontiguousarray(np.concatenate(cols, axis=1).T))
    return np.stack(out)


# --------------------------------------------------------------------------
# MLP backward ([TP-LLM] MLP block: "exactly one All-Reduce in the backward
# pass (to synchronize input gradients across the column-parallel layer)")
# --------------------------------------------------------------------------

def gelu_grad(z: np.ndarray) -> np.ndarray:
    """d GeLU / dz = Phi(z) + z phi(z), phi the standard normal density."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * (1.0 + _erf(z / math.sqrt(2.0))) + z * np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)


def mlp_backward(X, A, b1, B, dY, residual: bool = True) -> dict:
    """Gradients of Y = GeLU(X A + b1) B + b2 (+ X) given dY = dL/dY:
    dX, dA, db1, dB, db2 (unsharded)."""
    Z = linear(X, A, b1)
    H = gelu(Z)
    dH = dY @ B.T
    dZ = dH * gelu_grad(Z)
    dX = dZ @ A.T
    if residual:
        dX = dX + dY
    return dict(dX=dX, dA=X.T @ dZ, db1=dZ.sum(axis=0), dB=H.T @ dY, db2=dY.sum(axis=0))


def mlp_backward_sharded(X, A, b1, B, dY, n_shards: int, residual: bool = True) -> dict:
    """The tensor-parallel backward: dY reaches every shard whole (the
    row-parallel layer's backward needs no exchange); each shard forms
    dH_i = dY B_i^T, dZ_i = dH_i GeLU'(Z_i), its weight gradients dB_i, dA_i,
    db1_i locally, and a full-size partial dX_i = dZ_i A_i^T; the one
    reduction is dX = sum_i dX_i (+ dY for the residual)."""
    A_i = shard_matrices(A, SPLIT_COLUMN, n_shards)
    b_i = shard_matrices(np.asarray(b1).reshape(1, -1), SPLIT_COLUMN, n_shards)
    B_i = shard_matrices(B, SPLIT_ROW, n_shards)
    parts, dA, db1, dB = [], [], [], []
    for Ai, bi, Bi in zip(A_i, b_i, B_i):
        Z = linear(X, Ai, bi[0])
        dZ = (dY @ Bi.T) * gelu_grad(Z)
        parts.append(dZ @ Ai.T)
        dA.append(X.T @ dZ)
        db1.append(dZ.sum(axis=0))
        dB.append(gelu(Z).T @ dY)
    dX = reduce_partials(parts, None, dY if residual else None)
    return dict(dX=dX, dA=np.concatenate(dA, axis=1), db1=np.concatenate(db1),
                dB=np.concatenate(dB, axis=0), db2=dY.sum(axis=0), dX_partials=parts)


# --------------------------------------------------------------------------
# attention-block and layer backward ([TP-LLM] "Communication Budget and
# Scaling Limits": two all-reduces in the forward pass and two in the
# backward pass of every layer, one per block)
# --------------------------------------------------------------------------

def attention_head_backward(Q, K, V, dO, causal: bool) -> tuple:
    """Gradients of O = softmax(Q K^T / sqrt d) V for one head of one
    sequence, given dO = dL/dO: (dQ, dK, dV). The chain rule through the
    three steps S = Q K^T / sqrt d, P = softmax_rows(S), O = P V:
    dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dP * P)) (the softmax
    Jacobian applied row by row), dQ = dS K / sqrt d, dK = dS^T Q / sqrt d.
    Masked (causal) entries have P = 0 and receive no gradient."""
    d = Q.shape[1]
    S = (Q @ K.T) / math.sqrt(d)
    if causal:
        t = np.arange(Q.shape[0])[:, None]
        s = np.arange(K.shape[0])[None, :]
        S = np.where(s <= t, S, -np.inf)
    P = softmax_rows(S)
    dV = P.T @ dO
    dP = dO @ V.T
    dS = P * (dP - np.sum(dP * P, axis=1, keepdims=True))
    return dS @ K / math.sqrt(d), dS.T @ Q / math.sqrt(d), dV


def attention_logsumexp(Q, K, causal: bool) -> np.ndarray:
    """Per query row: ln sum_s exp(q . k_s / sqrt d) over the keys the query
    sees (the normaliser of its softmax row), for one head of one
    sequence."""
    d = Q.shape[1]
    S = (Q @ K.T) / math.sqrt(d)
    if causal:
        t = np.arange(Q.shape[0])[:, None]
        s = np.arange(K.shape[0])[None, :]
        S = np.where(s <= t, S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    return (m + np.log(np.exp(S - m).sum(axis=1, keepdims=True)))[:, 0]


def attention_heads_backward(Q, K, V, dO, batch: int, seq: int, n_heads: int,
                             causal: bool) -> tuple:
    """attention_head_backward for every (sequence, head) pair; head k is
    columns [k d, (k+1) d) of Q, K, V, dO. Returns (dQ, dK, dV) [M][h]."""
    M, h = Q.shape
    d = h // n_heads
    dQ, dK, dV = np.zeros((M, h)), np.zeros((M, h)), np.zeros((M, h))
    for s in range(batch):
        r = slice(s * seq, (s + 1) * seq)
        for k in range(n_heads):
            c = slice(k * d, (k + 1) * d)
            dQ[r, c], dK[r, c], dV[r, c] = attention_head_backward(
                Q[r, c], K[r, c], V[r, c], dO[r, c], causal)
    return dQ, dK, dV


def self_attention_backward(X, Wqkv, bqkv, Wo, bo, dY, batch: int, seq: int,
                            n_heads: int, causal: bool = True,
                            residual: bool = True) -> dict:
    """Gradients of Y = concat_heads(attention) W_O + b_O (+ X) given dY
    (unsharded): dX, dWqkv, dbqkv, dWo, dbo."""
    h = X.shape[1]
    QKV = linear(X, Wqkv, bqkv)
    Q, K, V = QKV[:, :h], QKV[:, h:2 * h], QKV[:, 2 * h:]
    O = attention_heads(Q, K, V, batch, seq, n_heads, causal)
    dO = dY @ Wo.T
    dQ, dK, dV = attention_heads_backward(Q, K, V, dO, batch, seq, n_heads, causal)
    dQKV = np.concatenate([dQ, dK, dV], axis=1)
    dX = dQKV @ Wqkv.T
    if residual:
        dX = dX + dY
    return dict(dX=dX, dWqkv=X.T @ dQKV, dbqkv=dQKV.sum(axis=0), dWo=O.T @ dY,
                dbo=dY.sum(axis=0))


def self_attention_backward_sharded(X, Wqkv, bqkv, Wo, bo, dY, batch: int,
                                    seq: int, n_heads: int, n_shards: int,
                                    causal: bool = True,
                                    residual: bool = True) -> dict:
    """The tensor-parallel backward of the attention block: dY reaches every
    shard whole (the backward of the row-parallel W_O needs no exchange);
    shard i forms dO_i = dY W_O,i^T, the attention backward of its own heads,
    dQKV_i = [dQ_i | dK_i | dV_i], its weight gradients dW_QKV,i = X^T dQKV_i,
    db_QKV,i, dW_O,i = O_i^T dY locally, and a full-size partial
    dX_i = dQKV_i W_QKV,i^T; the one reduction is dX = sum_i dX_i (+ dY).
    The gradients of the sharded weights are returned in the unsharded
    orientation (the shards' pieces put back in place)."""
    h = X.shape[1]
    d = h // n_heads
    hs = h // n_shards
    hps = n_heads // n_shards
    owner, local = shard_index_map(SPLIT_QKV_HEADS, h, 3 * h, n_shards, d)
    Wqkv_i = shard_matrices(Wqkv, SPLIT_QKV_HEADS, n_shards, d)
    bqkv_i = shard_matrices(np.asarray(bqkv).reshape(1, -1), SPLIT_QKV_HEADS, n_shards, d)
    Wo_i = shard_matrices(Wo, SPLIT_ROW, n_shards)
    parts, dqkv_shards = [], []
    dWqkv, dbqkv = np.zeros((h, 3 * h)), np.zeros(3 * h)
    dWo = np.zeros((h, h))
    for i in range(n_shards):
        QKV = linear(X, Wqkv_i[i], bqkv_i[i][0])
        Q, K, V = QKV[:, :hs], QKV[:, hs:2 * hs], QKV[:, 2 * hs:]
        O = attention_heads(Q, K, V, batch, seq, hps, causal)
        dO = dY @ Wo_i[i].T
        dQ, dK, dV = attention_heads_backward(Q, K, V, dO, batch, seq, hps, causal)
        dQKV = np.concatenate([dQ, dK, dV], axis=1)
        dqkv_shards.append(dQKV)
        parts.append(dQKV @ Wqkv_i[i].T)
        mine = owner == i                      # W_QKV columns of shard i
        dWqkv[:, mine] = (X.T @ dQKV)[:, local[mine]]
        dbqkv[mine] = dQKV.sum(axis=0)[local[mine]]
        dWo[i * hs:(i + 1) * hs, :] = O.T @ dY
    dX = reduce_partials(parts, None, dY if residual else None)
    return dict(dX=dX, dWqkv=dWqkv, dbqkv=dbqkv, dWo=dWo, dbo=dY.sum(axis=0),
                dX_partials=parts, dQKV_shards=dqkv_shards)


def layernorm_backward(x, gamma, dy, eps: float = 1e-5) -> tuple:
    """Gradients of y = gamma * (x - mu) / sqrt(var + eps) + beta per row
    (population variance) given dy: (dx, dgamma, dbeta). With x_hat the
    normalised row and g = dy * gamma, the row's dx is
    (g - mean(g) - x_hat * mean(g * x_hat)) / sqrt(var + eps)."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xh = (x - mu) * rstd
    g = dy * gamma
    dx = rstd * (g - g.mean(axis=1, keepdims=True) - xh * (g * xh).mean(axis=1, keepdims=True))
    return dx, (dy * xh).sum(axis=0), dy.sum(axis=0)


def transformer_layer_backward(X, p: dict, dY, batch: int, seq: int,
                               n_heads: int, n_shards: int, eps: float = 1e-5,
                               causal: bool = True) -> dict:
    """Gradients of the pre-LN layer Y = h1 + MLP(LN2(h1)),
    h1 = X + Attn(LN1(X)), by the tensor-parallel route: the MLP block's
    backward (one reduction, of its input gradient) and the attention
    block's backward (one reduction) with the LayerNorm backward and the
    residual paths between them. Returns dX and every parameter gradient
    (LN gammas and betas included)."""
    x1 = layernorm(X, p["ln1_g"], p["ln1_b"], eps)
    h1 = self_attention_sharded(x1, p["Wqkv"], p["bqkv"], p["Wo"], p["bo"], X,
                                batch, seq, n_heads, n_shards, causal)
    x2 = layernorm(h1, p["ln2_g"], p["ln2_b"], eps)
    gm = mlp_backward_sharded(x2, p["A"], p["b1"], p["B"], dY, n_shards, residual=False)
    dx2 = gm["dX"]
    dln2, dg2, db2n = layernorm_backward(h1, p["ln2_g"], dx2, eps)
    dh1 = dY + dln2
    ga = self_attention_backward_sharded(x1, p["Wqkv"], p["bqkv"], p["Wo"], p["bo"], dh1,
                                         batch, seq, n_heads, n_shards, causal, residual=False)
    dln1, dg1, db1n = layernorm_backward(X, p["ln1_g"], ga["dX"], eps)
    return dict(dX=dh1 + dln1, dh1=dh1,
                dWqkv=ga["dWqkv"], dbqkv=ga["dbqkv"], dWo=ga["dWo"], dbo=ga["dbo"],
                dA=gm["dA"], db1=gm["db1"], dB=gm["dB"], db2=gm["db2"],
                dln1_g=dg1, dln1_b=db1n, dln2_g=dg2, dln2_b=db2n)


# --------------------------------------------------------------------------
# grouped-query attention ([TP-LLM] "Grouped-Query Attention (GQA)
# Constraints")
# --------------------------------------------------------------------------
#
# W_QKV = [W_Q | W_K | W_V] with n_q query heads and n_kv key/value heads of
# dimension d (W_Q: h x n_q d, W_K, W_V: h x n_kv d); query head j uses
# key/value head j // (n_q / n_kv). Sharding keeps whole groups local: with
# n_kv % N == 0 shard i owns query heads [i n_q/N, (i+1) n_q/N) and kv heads
# [i n_kv/N, (i+1) n_kv/N); with N > n_kv (N % n_kv == 0) each shard owns
# n_q/N query heads, all in one group, and a copy of that group's kv head
# (the duplication the page allows). Shard i's columns: [Q_i | K_i | V_i].

def gqa_kv_local(n_kv: int, n_shards: int) -> int:
    if n_shards <= n_kv:
        _check_div("n_kv", n_kv, n_shards)
        return n_kv // n_shards
    _check_div("N", n_shards, n_kv)
    return 1


def gqa_shard_columns(n_q: int, n_kv: int, d: int, n_shards: int) -> list:
    """For each shard, the W_QKV column indices of [Q_i | K_i | V_i]."""
    _check_div("n_q", n_q, n_shards)
    if n_q % n_kv:
        raise ValueError("n_q must be a multiple of n_kv")
    qs, kvl = n_q // n_shards, gqa_kv_local(n_kv, n_shards)
    kv0 = n_q * d                      # first K column
    v0 = kv0 + n_kv * d                # first V column
    out = []
    for i in range(n_shards):
        q_heads = range(i * qs, (i + 1) * qs)
        first_kv = (i * qs) // (n_q // n_kv)
        kv_heads = range(first_kv, first_kv + kvl)
        cols = [k * d + e for k in q_heads for e in range(d)]
        cols += [kv0 + k * d + e for k in kv_heads for e in range(d)]
        cols += [v0 + k * d + e for k in kv_heads for e in range(d)]
        out.append(np.asarray(cols, dtype=np.int64))
    return out


def packed_gqa_shards(Wqkv: np.ndarray, n_q: int, n_kv: int, d: int,
                      n_shards: int) -> np.ndarray:
    """Byte layout of GQA QKV shards: [N, (n_q/N + 2 kv_local) d, h_in]."""
    return np.stack([np.ascontiguousarray(Wqkv[:, c].T)
                     for c in gqa_shard_columns(n_q, n_kv, d, n_shards)])


def gqa_attention_heads(Q, K, V, batch: int, seq: int, n_q: int, n_kv: int,
                        causal: bool) -> np.ndarray:
    """Query head j attends with key/value head j // (n_q / n_kv)."""
    d = Q.shape[1] // n_q
    g = n_q // n_kv
    O = np.zeros((Q.shape[0], n_q * d))
    for s in range(batch):
        r = slice(s * seq, (s + 1) * seq)
        for j in range(n_q):
            c = slice(j * d, (j + 1) * d)
            kc = slice((j // g) * d, (j // g + 1) * d)
            O[r, c] = attention_head(Q[r, c], K[r, kc], V[r, kc], causal)
    return O


def gqa_self_attention(X, Wqkv, bqkv, Wo, bo, residual, batch: int, seq: int,
                       n_q: int, n_kv: int, causal: bool = True) -> np.ndarray:
    """Unsharded GQA block: Y = concat_j head_j W_O + b_O (+ R)."""
    d = Wo.shape[0] // n_q
    QKV = linear(X, Wqkv, bqkv)
    Q = QKV[:, :n_q * d]
    K = QKV[:, n_q * d:(n_q + n_kv) * d]
    V = QKV[:, (n_q + n_kv) * d:]
    O = gqa_attention_heads(Q, K, V, batch, seq, n_q, n_kv, causal)
    return reduce_partials([linear(O, Wo)], bo, residual)


def gqa_self_attention_sharded(X, Wqkv, bqkv, Wo, bo, residual, batch: int,
                               seq: int, n_q: int, n_kv: int, n_shards: int,
                               causal: bool = True) -> np.ndarray:
    """The tensor-parallel route for GQA: each shard projects its query heads
    and its (possibly duplicated) kv heads, attends locally, and W_O is
    row-parallel over the query heads; one sum of the partials."""
    d = Wo.shape[0] // n_q
    qs, kvl = n_q // n_shards, gqa_kv_local(n_kv, n_shards)
    O_i = []
    for cols in gqa_shard_columns(n_q, n_kv, d, n_shards):
        q = linear(X, Wqkv[:, cols], None if bqkv is None else bqkv[cols])
        O_i.append(gqa_attention_heads(q[:, :qs * d], q[:, qs * d:(qs + kvl) * d],
                                       q[:, (qs + kvl) * d:], batch, seq, qs, kvl, causal))
    return reduce_partials(row_parallel_linear(O_i, Wo, n_shards), bo, residual)


def gqa_attention_heads_backward(Q, K, V, dO, batch: int, seq: int, n_q: int,
                                 n_kv: int, causal: bool) -> tuple:
    """attention_head_backward for every (sequence, query head); query head j
    uses key/value head j // (n_q / n_kv), so a key/value head's gradient is
    the sum over the query heads of its group. Returns (dQ, dK, dV)."""
    d = Q.shape[1] // n_q
    g = n_q // n_kv
    dQ, dK, dV = np.zeros_like(Q, dtype=np.float64), np.zeros_like(K, dtype=np.float64), \
        np.zeros_like(V, dtype=np.float64)
    for s in range(batch):
        r = slice(s * seq, (s + 1) * seq)
        for j in range(n_q):
            c = slice(j * d, (j + 1) * d)
            kc = slice((j // g) * d, (j // g + 1) * d)
            dq, dk, dv = attention_head_backward(Q[r, c], K[r, kc], V[r, kc], dO[r, c], causal)
            dQ[r, c] = dq
            dK[r, kc] += dk
            dV[r, kc] += dv
    return dQ, dK, dV


def gqa_self_attention_backward(X, Wqkv, bqkv, Wo, bo, dY, batch: int, seq: int,
                                n_q: int, n_kv: int, causal: bool = True,
                                residual: bool = True) -> dict:
    """Gradients of the unsharded GQA block given dY: dX, dWqkv, dbqkv, dWo, dbo."""
    d = Wo.shape[0] // n_q
    QKV = linear(X, Wqkv, bqkv)
    Q = QKV[:, :n_q * d]
    K = QKV[:, n_q * d:(n_q + n_kv) * d]
    V = QKV[:, (n_q + n_kv) * d:]
    O = gqa_attention_heads(Q, K, V, batch, seq, n_q, n_kv, causal)
    dO = dY @ Wo.T
    dQ, dK, dV = gqa_attention_heads_backward(Q, K, V, dO, batch, seq, n_q, n_kv, causal)
    dQKV = np.concatenate([dQ, dK, dV], axis=1)
    dX = dQKV @ Wqkv.T
    if residual:
        dX = dX + dY
    return dict(dX=dX, dWqkv=X.T @ dQKV, dbqkv=dQKV.sum(axis=0), dWo=O.T @ dY,
                dbo=dY.sum(axis=0))


def gqa_self_attention_backward_sharded(X, Wqkv, bqkv, Wo, bo, dY, batch: int,
                                        seq: int, n_q: int, n_kv: int,
                                        n_shards: int, causal: bool = True,
                                        residual: bool = True) -> dict:
    """The tensor-parallel GQA backward: as self_attention_backward_sharded,
    with each shard's key/value heads (duplicated when N > n_kv) receiving the
    gradient of its own query heads. A duplicated head's weight gradient is the
    sum over its replicas (the gradient of a replicated parameter); the
    per-shard gradients, packed like the shards, are returned as well."""
    d = Wo.shape[0] // n_q
    qs, kvl = n_q // n_shards, gqa_kv_local(n_kv, n_shards)
    hs = qs * d
    Wo_i = shard_matrices(Wo, SPLIT_ROW, n_shards)
    parts, dqkv_shards, dW_shards, db_shards = [], [], [], []
    dWqkv, dbqkv = np.zeros(Wqkv.shape), np.zeros(Wqkv.shape[1])
    dWo = np.zeros(Wo.shape)
    for i, cols in enumerate(gqa_shard_columns(n_q, n_kv, d, n_shards)):
        W = Wqkv[:, cols]
        q = linear(X, W, None if bqkv is None else bqkv[cols])
        Q, K, V = q[:, :hs], q[:, hs:hs + kvl * d], q[:, hs + kvl * d:]
        O = gqa_attention_heads(Q, K, V, batch, seq, qs, kvl, causal)
        dO = dY @ Wo_i[i].T
        dQ, dK, dV = gqa_attention_heads_backward(Q, K, V, dO, batch, seq, qs, kvl, causal)
        dQKV = np.concatenate([dQ, dK, dV], axis=1)
        dqkv_shards.append(dQKV)
        parts.append(dQKV @ W.T)
        dW_shards.append((X.T @ dQKV).T)       # packed like the shard: [cols][h_in]
        db_shards.append(dQKV.sum(axis=0))
        np.add.at(dWqkv.T, cols, (X.T @ dQKV).T)
        np.add.at(dbqkv, cols, dQKV.sum(axis=0))
        dWo[i * hs:(i + 1) * hs, :] = O.T @ dY
    dX = reduce_partials(parts, None, dY if residual else None)
    return dict(dX=dX, dWqkv=dWqkv, dbqkv=dbqkv, dWo=dWo, dbo=dY.sum(axis=0),
                dX_partials=parts, dQKV_shards=dqkv_shards,
                dWqkv_packed=np.stack(dW_shards), dbqkv_packed=np.stack(db_shards))


# --------------------------------------------------------------------------
# sequence parallelism ([TP-LLM] "Sequence Parallelism")
# --------------------------------------------------------------------------
#
# Activations outside the blocks are split along the sequence: shard i owns
# positions [i S/N, (i+1) S/N) of every sequence of the batch. A shard's
# slice is stored [batch][S/N][h]; the N slices stacked make [N][b][S/N][h].

def sequence_shard(X: np.ndarray, batch: int, seq: int, n_shards: int) -> list:
    """Split token rows (batch-major [b*S, h]) into the N sequence slices,
    each [b, S/N, h]."""
    _check_div("seq", seq, n_shards)
    ss = seq // n_shards
    X3 = X.reshape(batch, seq, -1)
    return [X3[:, i * ss:(i + 1) * ss, :] for i in range(n_shards)]


def all_gather_sequence(slices: list, batch: int, seq: int) -> np.ndarray:
    """The all-gather before a column-parallel layer: the N sequence slices
    concatenated along the sequence, back to [b*S, h] token rows."""
    return np.concatenate(slices, axis=1).reshape(batch * seq, -1)


def reduce_scatter_partials(partials: list, batch: int, seq: int, n_shards: int,
                            bias=None, residual_slices=None) -> list:
    """The reduce-scatter after a row-parallel layer: the sum of the N
    partials, scattered along the sequence (shard i keeps its slice), with the
    output bias and that shard's residual slice added once."""
    Y = reduce_partials(partials, bias)
    out = sequence_shard(Y, batch, seq, n_shards)
    if residual_slices is not None:
        out = [o + r for o, r in zip(out, residual_slices)]
    return out


def transformer_layer_sp(X_slices: list, p: dict, batch: int, seq: int,
                         n_heads: int, n_shards: int, eps: float = 1e-5,
                         causal: bool = True) -> list:
    """Pre-LN layer with sequence parallelism: LayerNorm on each shard's
    slice, all-gather before each column-parallel layer, reduce-scatter
    after each row-parallel layer, residual adds on the slices.
    Returns the N output slices [b, S/N, h]."""
    h = X_slices[0].shape[-1]
    d = h // n_heads
    hs = h // n_shards
    x1 = [layernorm(x, p["ln1_g"], p["ln1_b"], eps) for x in X_slices]
    X1 = all_gather_sequence(x1, batch, seq)
    QKV_i = column_parallel_linear(X1, p["Wqkv"], p["bqkv"], n_shards,
                                   kind=SPLIT_QKV_HEADS, head_dim=d)
    O_i = [attention_heads(q[:, :hs], q[:, hs:2 * hs], q[:, 2 * hs:],
                           batch, seq, n_heads // n_shards, causal)
           for q in QKV_i]
    P_i = row_parallel_linear(O_i, p["Wo"], n_shards)
    h1 = reduce_scatter_partials(P_i, batch, seq, n_shards, p["bo"], X_slices)
    x2 = [layernorm(x, p["ln2_g"], p["ln2_b"], eps) for x in h1]
    X2 = all_gather_sequence(x2, batch, seq)
    A_i = column_parallel_linear(X2, p["A"], p["b1"], n_shards, act=gelu)
    P_i = row_parallel_linear(A_i, p["B"], n_shards)
    return reduce_scatter_partials(P_i, batch, seq, n_shards, p["b2"], h1)


def transformer_layer_sp_backward(X_slices: list, p: dict, dY_slices: list,
                                  batch: int, seq: int, n_heads: int,
                                  n_shards: int, eps: float = 1e-5,
                                  causal: bool = True) -> dict:
    """Backward of transformer_layer_sp: each forward all-gather becomes a
    reduce-scatter and each reduce-scatter an all-gather. dY's slices are
    all-gathered for the MLP block; its partial input gradients are
    reduce-scattered into the slices, where LN2's backward and the residual
    give dh1; dh1 is all-gathered for the attention block, whose partials are
    reduce-scattered, LN1's backward applied on the slices and dh1 added.
    Returns dX as N slices and every parameter gradient."""
    x1 = [layernorm(x, p["ln1_g"], p["ln1_b"], eps) for x in X_slices]
    X1 = all_gather_sequence(x1, batch, seq)
    h1 = transformer_layer_sp_block_out(X_slices, p, batch, seq, n_heads, n_shards, eps, causal)
    x2 = [layernorm(x, p["ln2_g"], p["ln2_b"], eps) for x in h1]
    X2 = all_gather_sequence(x2, batch, seq)
    dYg = all_gather_sequence(dY_slices, batch, seq)
    gm = mlp_backward_sharded(X2, p["A"], p["b1"], p["B"], dYg, n_shards, residual=False)
    g2 = sequence_shard(reduce_partials(gm["dX_partials"]), batch, seq, n_shards)
    h = X_slices[0].shape[-1]
    dh1, dg2, db2n = [], 0.0, 0.0
    for hs_, gs_, dys in zip(h1, g2, dY_slices):   # slices [b][S/N][h]: rows of h
        dx, dg, db = layernorm_backward(hs_.reshape(-1, h), p["ln2_g"], gs_.reshape(-1, h), eps)
        dh1.append(dys + dx.reshape(dys.shape))
        dg2, db2n = dg2 + dg, db2n + db
    dh1g = all_gather_sequence(dh1, batch, seq)
    ga = self_attention_backward_sharded(X1, p["Wqkv"], p["bqkv"], p["Wo"], p["bo"], dh1g,
                                         batch, seq, n_heads, n_shards, causal, residual=False)
    g1 = sequence_shard(reduce_partials(ga["dX_partials"]), batch, seq, n_shards)
    dX, dg1, db1n = [], 0.0, 0.0
    for xs_, gs_, dhs in zip(X_slices, g1, dh1):
        dx, dg, db = layernorm_backward(xs_.reshape(-1, h), p["ln1_g"], gs_.reshape(-1, h), eps)
        dX.append(dhs + dx.reshape(dhs.shape))
        dg1, db1n = dg1 + dg, db1n + db
    return dict(dX=dX, dWqkv=ga["dWqkv"], dbqkv=ga["dbqkv"], dWo=ga["dWo"], dbo=ga["dbo"],
                dA=gm["dA"], db1=gm["db1"], dB=gm["dB"], db2=gm["db2"],
                dln1_g=dg1, dln1_b=db1n, dln2_g=dg2, dln2_b=db2n)


def transformer_layer_sp_block_out(X_slices: list, p: dict, batch: int, seq: int,
                                   n_heads: int, n_shards: int, eps: float = 1e-5,
                                   causal: bool = True) -> list:
    """h1 = X + Attn(LN1(X)) of the sequence-parallel layer, as slices."""
    h = X_slices[0].shape[-1]
    d = h // n_heads
    hs = h // n_shards
    x1 = [layernorm(x, p["ln1_g"], p["ln1_b"], eps) for x in X_slices]
    X1 = all_gather_sequence(x1, batch, seq)
    QKV_i = column_parallel_linear(X1, p["Wqkv"], p["bqkv"], n_shards,
                                   kind=SPLIT_QKV_HEADS, head_dim=d)
    O_i = [attention_heads(q[:, :hs], q[:, hs:2 * hs], q[:, 2 * hs:],
                           batch, seq, n_heads // n_shards, causal)
           for q in QKV_i]
    P_i = row_parallel_linear(O_i, p["Wo"], n_shards)
    return reduce_scatter_partials(P_i, batch, seq, n_shards, p["bo"], X_slices)


# --------------------------------------------------------------------------
# the same definitions restricted to a subset of output token rows
# (used to check full-size workloads on sampled rows)
# --------------------------------------------------------------------------

def mlp_rows(X, A, b1, B, b2, residual, rows) -> np.ndarray:
    """Rows ``rows`` of mlp(): every output row depends on its input row only."""
    R = None if residual is None else residual[rows]
    return mlp(X[rows], A, b1, B, b2, R)


def self_attention_rows(X, Wqkv, bqkv, Wo, bo, residual, batch: int,
                        seq: int, n_heads: int, rows,
                        causal: bool = True) -> np.ndarray:
    """Rows ``rows`` of self_attention(). Query row r (sequence r // seq,
    position r % seq) attends to the keys of its own sequence (only up to
    its position when causal), so K and V are projected for the whole
    sequences the sampled rows belong to, Q for the sampled rows only."""
    rows = np.asarray(rows, dtype=np.int64)
    h = X.shape[1]
    d = h // n_heads
    Wq, Wk, Wv = Wqkv[:, :h], Wqkv[:, h:2 * h], Wqkv[:, 2 * h:]
    bq, bk, bv = bqkv[:h], bqkv[h:2 * h], bqkv[2 * h:]
    O = np.zeros((len(rows), h))
    for s in np.unique(rows // seq):
        sel = np.nonzero(rows // seq == s)[0]
        Xs = X[s * seq:(s + 1) * seq]
        K = linear(Xs, Wk, bk)
        V = linear(Xs, Wv, bv)
        Q = linear(X[rows[sel]], Wq, bq)
        pos = rows[sel] - s * seq
        for k in range(n_heads):
            c = slice(k * d, (k + 1) * d)
            S = (Q[:, c] @ K[:, c].T) / math.sqrt(d)
            if causal:
                S = np.where(np.arange(seq)[None, :] <= pos[:, None], S,
                             -np.inf)
            O[sel, c] = softmax_rows(S) @ V[:, c]
    R = None if residual is None else residual[rows]
    return reduce_partials([linear(O, Wo)], bo, R)


def transformer_layer_rows(X, p: dict, batch: int, seq: int, n_heads: int,
                           rows, eps: float = 1e-5,
                           causal: bool = True) -> np.ndarray:
    """Rows ``rows`` of transformer_layer()."""
    rows = np.asarray(rows, dtype=np.int64)
    x1 = layernorm(X, p["ln1_g"], p["ln1_b"], eps)
    h1 = self_attention_rows(x1, p["Wqkv"], p["bqkv"], p["Wo"], p["bo"], X,
                             batch, seq, n_heads, rows, causal)
    x2 = layernorm(h1, p["ln2_g"], p["ln2_b"], eps)
    return mlp(x2, p["A"], p["b1"], p["B"], p["b2"], h1)


# --------------------------------------------------------------------------
# algorithmic work, for throughput figures
# --------------------------------------------------------------------------

def gemm_flops(m: int, n: int, k: int) -> int:
    return 2 * m * n * k


def attention_flops(batch: int, seq: int, n_heads: int, d: int,
                    causal: bool) -> float:
    """QK^T and PV: 4 S^2 d per (sequence, head); half of it when causal."""
    f = 4.0 * seq * seq * d * n_heads * batch
    return f / 2 if causal else f
