"""The C-ABI library on the host (no GPU): it loads, exports every function
include/tp.h declares, and its host-side logic (status strings, workspace
sizes, the shard index map, argument checks that return before any CUDA
call) behaves as documented."""
import ctypes

import numpy as np
import pytest

from oracle import tp_oracle as O

tp = pytest.importorskip("tensor_transformer_layer_linear_b200.tp")


def test_exports_every_header_function():
    names = tp.header_functions()
    assert len(names) >= 18
    for n in names:
        assert hasattr(tp.lib, n), n
    for must in ("tp_shard_weights", "tp_column_linear", "tp_row_linear", "tp_reduce_partials",
                 "tp_mlp_forward", "tp_attn_forward", "tp_layer_forward"):
        assert must in names


def test_status_strings():
    for st in range(8):
        assert tp.tp_status_string(st).startswith("TP_")
    assert "unknown" in tp.tp_status_string(99)


@pytest.mark.parametrize("kind", [tp.TP_SPLIT_COLUMN, tp.TP_SPLIT_ROW, tp.TP_SPLIT_QKV_HEADS,
                                  tp.TP_SPLIT_GATE_UP])
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_index_map_matches_oracle(kind, n):
    h, d = 2048, 128
    h_in, h_out = (h, 3 * h) if kind == tp.TP_SPLIT_QKV_HEADS else (h, 4 * h)
    owner, local = tp.tp_shard_index_map(kind, h_in, h_out, n, d)
    o_owner, o_local = O.shard_index_map(kind, h_in, h_out, n, d)
    assert np.array_equal(owner.astype(np.int64), o_owner)
    assert np.array_equal(local, o_local)


def test_index_map_rejects_indivisible():
    with pytest.raises(tp.TPError) as e:
        tp.tp_shard_index_map(tp.TP_SPLIT_COLUMN, 8, 12, 5)
    assert e.value.status == tp.TP_ERR_SHAPE
    with pytest.raises(tp.TPError):
        tp.tp_shard_index_map(tp.TP_SPLIT_QKV_HEADS, 384, 3 * 384, 8, 128)  # 3 heads


def test_workspace_bytes():
    M, h, F, N = 4096, 4096, 16384, 8
    mlp = tp.tp_workspace_bytes(tp.TP_WS_MLP, M, h, F, N)
    assert mlp >= M * F * 2 + N * M * h * 4
    attn = tp.tp_workspace_bytes(tp.TP_WS_ATTN, M, h, 0, N)
    assert attn >= M * 3 * h * 2 + M * h * 2 + N * M * h * 4
    layer = tp.tp_workspace_bytes(tp.TP_WS_LAYER, M, h, F, N)
    assert layer >= mlp + attn - N * M * h * 4
    assert tp.tp_workspace_bytes(tp.TP_WS_MLP, 0, h, F, N) == 0
    assert tp.tp_workspace_bytes(99, M, h, F, N) == 0
    # backward passes: the recomputed activations, gradients and partials fit
    mlp_b = tp.tp_workspace_bytes(tp.TP_WS_MLP_BWD, M, h, F, N)
    assert mlp_b >= 3 * M * F * 2 + N * M * h * 4
    core = tp.tp_workspace_bytes(tp.TP_WS_ATTN_CORE_BWD, M, h, 0, N)
    assert core >= h * (M + 128) * 4          # the fp32 dQ accumulator
    attn_b = tp.tp_workspace_bytes(tp.TP_WS_ATTN_BWD, M, h, 0, N)
    assert attn_b >= core + 2 * M * 3 * h * 2 + 2 * M * h * 2 + N * M * h * 4
    layer_b = tp.tp_workspace_bytes(tp.TP_WS_LAYER_BWD, M, h, F, N)
    assert layer_b >= attn_b + 3 * M * F * 2 + 4 * M * h * 2
    assert tp.tp_workspace_bytes(tp.TP_WS_LAYER_BWD, M, h, 0, N) == 0
    assert tp.tp_workspace_bytes(tp.TP_WS_LN_BWD, M, h, 0, N) > 0


def test_argument_errors_return_before_launch():
    L = tp.lib
    fake = 1 << 20   # never dereferenced: every call below fails its checks first
    assert L.tp_column_linear(None, 32, 64, fake, None, 64, 2, 0, fake, None) == tp.TP_ERR_NULL
    assert L.tp_column_linear(fake, 32, 64, fake, None, 66, 2, 0, fake, None) == tp.TP_ERR_SHAPE
    assert L.tp_column_linear(fake, 32, 60, fake, None, 64, 2, 0, fake, None) == tp.TP_ERR_SHAPE
    assert L.tp_column_linear(fake, 32, 64, fake, None, 64, 2, 7, fake, None) == tp.TP_ERR_UNSUPPORTED
    assert L.tp_column_linear(fake + 2, 32, 64, fake, None, 64, 2, 0, fake, None) == tp.TP_ERR_ALIGN
    assert L.tp_row_linear(fake, 32, 66, fake, 64, 2, fake, None) == tp.TP_ERR_SHAPE
    assert L.tp_row_linear(fake, 32, 64, fake, 64, 0, fake, None) == tp.TP_ERR_SHAPE
    assert L.tp_reduce_partials(None, 2, 4, 64, None, None, fake, None) == tp.TP_ERR_NULL
    assert L.tp_reduce_partials(fake, 2, 4, 60, None, None, fake, None) == tp.TP_ERR_SHAPE
    assert L.tp_layernorm(fake, 4, 16392, fake, fake, 1e-5, fake, None) == tp.TP_ERR_SHAPE
    assert L.tp_attention(fake, 2, 64, 1024, 16, 1, 3, fake, None) == tp.TP_ERR_SHAPE
    assert L.tp_attention(fake, 2, 64, 1024, 16, 1, 4, fake, None) == tp.TP_ERR_UNSUPPORTED
    assert L.tp_shard_weights(fake, 64, 96, 4, tp.TP_SPLIT_QKV_HEADS, 16, fake, None) == tp.TP_ERR_SHAPE
    assert L.tp_shard_weights(fake, 64, 96, 4, 9, 16, fake, None) == tp.TP_ERR_SHAPE
    ws_small = 16
    assert L.tp_mlp_forward(fake, 32, 64, 256, 2, fake, None, fake, None, None, fake, ws_small,
                            fake, None) == tp.TP_ERR_WORKSPACE
    w = tp.tp_layer_weights()
    assert L.tp_layer_forward(fake, 1, 32, 256, 2, 1024, 2, ctypes.byref(w), 1e-5, fake,
                              1 << 30, fake, None) == tp.TP_ERR_NULL
