"""Seeded synthetic inputs shared by the tests, the benchmark and smoke().

This module only draws numbers and converts bit patterns. It holds none of
the tensor-parallel method's arithmetic (no matmul, no activation, no
reduction), so both the CPU oracle (through the tests) and the CUDA path can
be fed the same bytes without sharing any code that computes the method.

Recipe (fixed, seed 0 unless a caller asks otherwise):
  * one ``numpy.random.Generator(Philox(seed))`` per workload;
  * tensors are drawn in a fixed order: X, then the weights in layer order
    (W_QKV, W_O, A, B), then the biases in the same order;
  * every draw is ``standard_normal(float32) * std`` rounded once to bf16
    (round-to-nearest-even); the bf16 bit patterns are the inputs;
  * LayerNorm gamma = 1 and beta = 0 (exactly representable);
  * the residual R of an MLP or attention block is X itself.

The five workloads are the shapes of the Megatron-LM tensor-parallel MLP,
attention and layer examples: the page-1 worked example
(Linear(1024 -> 4096) on 32 tokens, tensor_model_parallel_size = 2), a
4 x 2048-token MLP, a 16-head causal attention block, a full pre-LN layer,
and a large MLP swept over shard counts. A gated (SwiGLU) MLP of the
4 x 2048-token MLP's shape is added for the gated variant, and a
grouped-query attention block of the attention block's shape (16 query
heads, 4 key/value heads, 8 shards: key/value heads duplicated).
"""
from __future__ import annotations

import numpy as np

# name -> workload description (shapes, value distributions, shard count)
CONFIGS = {
    "mlp_32x1024_f4096_n2": dict(
        kind="mlp", batch=1, seq=32, h=1024, ffn=4096, n_shards=2,
        x_std=1.0, w_std=0.02, b_std=0.0, residual=False),
    "mlp_8192x1024_f4096_n4": dict(
        kind="mlp", batch=4, seq=2048, h=1024, ffn=4096, n_shards=4,
        x_std=1.0, w_std=0.02, b_std=0.01, residual=True),
    "attn_4x2048_h2048_16x128_n8": dict(
        kind="attn", batch=4, seq=2048, h=2048, n_heads=16, n_shards=8,
        causal=True, x_std=1.0, w_std=0.02, b_std=0.01, residual=True),
    "layer_2x2048_h4096_32x128_f16384_n8": dict(
        kind="layer", batch=2, seq=2048, h=4096, n_heads=32, ffn=16384,
        n_shards=8, causal=True, x_std=1.0, w_std=0.02, b_std=0.01,
        ln_eps=1e-5),
    "attn_gqa_4x2048_h2048_16q4kv_n8": dict(
        kind="attn_gqa", batch=4, seq=2048, h=2048, n_heads=16, n_kv_heads=4,
        n_shards=8, causal=True, x_std=1.0, w_std=0.02, b_std=0.01, residual=True),
    "swiglu_8192x1024_f4096_n4": dict(
        kind="swiglu", batch=4, seq=2048, h=1024, ffn=4096, n_shards=4,
        x_std=1.0, w_std=0.02, b_std=0.01, residual=True),
    "mlp_2048x12288_f49152_sweep": dict(
        kind="mlp", batch=1, seq=2048, h=12288, ffn=49152, n_shards=1,
        sweep=(1, 2, 4, 8, 16), x_std=0.02, w_std=0.02, b_std=0.0,
        residual=False),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns exactly to float64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def _draw(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    if std == 0.0:
        return np.zeros(shape, dtype=np.uint16)
    x = rng.standard_normal(size=shape, dtype=np.float32)
    x *= np.float32(std)
    return f32_to_bf16_bits(x)


def config(name: str, **overrides) -> dict:
    cfg = dict(CONFIGS[name])
    cfg["name"] = name
    cfg.update(overrides)
    return cfg


def make_inputs(cfg: dict, seed: int = 0) -> dict:
    """Draw the logical (unsharded) bf16 inputs of a workload.

    Returns a dict of uint16 arrays (bf16 bits), row-major:
      X [M, h]; MLP: A [h, F], b1 [F], B [F, h], b2 [h];
      attention: Wqkv [h, 3h] (= [W_Q | W_K | W_V]), bqkv [3h], Wo [h, h], bo [h];
      layer: both sets plus ln1_g, ln1_b, ln2_g, ln2_b [h];
      swiglu (gated MLP): Wg, Wu [h, F], B [F, h], b2 [h];
      attn_gqa: Wqkv [h, (n_q + 2 n_kv) d], Wo [h, h], bqkv, bo.
    """
    rng = np.random.Generator(np.random.Philox(seed))
    kind = cfg["kind"]
    M = cfg["batch"] * cfg["seq"]
    h = cfg["h"]
    out = {"X": _draw(rng, (M, h), cfg["x_std"])}
    w, b = cfg["w_std"], cfg["b_std"]
    if kind in ("attn", "layer"):
        out["Wqkv"] = _draw(rng, (h, 3 * h), w)
        out["Wo"] = _draw(rng, (h, h), w)
    if kind == "attn_gqa":
        d = h // cfg["n_heads"]
        qkv_cols = (cfg["n_heads"] + 2 * cfg["n_kv_heads"]) * d
        out["Wqkv"] = _draw(rng, (h, qkv_cols), w)
        out["Wo"] = _draw(rng, (h, h), w)
        out["bqkv"] = _draw(rng, (qkv_cols,), b)
        out["bo"] = _draw(rng, (h,), b)
    if kind in ("mlp", "layer"):
        F = cfg["ffn"]
        out["A"] = _draw(rng, (h, F), w)
        out["B"] = _draw(rng, (F, h), w)
    if kind == "swiglu":
        F = cfg["ffn"]
        out["Wg"] = _draw(rng, (h, F), w)
        out["Wu"] = _draw(rng, (h, F), w)
        out["B"] = _draw(rng, (F, h), w)
        out["b2"] = _draw(rng, (h,), b)
    if kind in ("attn", "layer"):
        out["bqkv"] = _draw(rng, (3 * h,), b)
        out["bo"] = _draw(rng, (h,), b)
    if kind in ("mlp", "layer"):
        out["b1"] = _draw(rng, (cfg["ffn"],), b)
        out["b2"] = _draw(rng, (h,), b)
    if kind == "layer":
        one = f32_to_bf16_bits(np.ones(h, dtype=np.float32))
        zero = np.zeros(h, dtype=np.uint16)
        out["ln1_g"], out["ln1_b"] = one.copy(), zero.copy()
        out["ln2_g"], out["ln2_b"] = one.copy(), zero.copy()
    return out


def sample_rows(batch: int, seq: int, stride: int = 64) -> np.ndarray:
    """Deterministic token-row sample: every ``stride``-th row of each
    sequence plus its first and last row (sorted, unique)."""
    rows = []
    for s in range(batch):
        base = s * seq
        rows.extend(range(base, base + seq, stride))
        rows.append(base)
        rows.append(base + seq - 1)
    return np.unique(np.asarray(rows, dtype=np.int64))
