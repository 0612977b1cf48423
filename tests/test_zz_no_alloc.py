"""tp_mlp_forward_noalloc: the MLP block for callers that cannot allocate
device memory (no device allocator to hand, or all device memory already
reserved by their framework), so they cannot pass a workspace. Its scratch is
a fixed library-owned device array shared by every call; these tests check,
through the C ABI, that two calls in a row each give the result of the
workspace-taking tp_mlp_forward on the same inputs, and that a problem too
large for the array is refused before anything runs.

Kept in a file that pytest collects last; it also passes alone in a fresh
process.
"""
import numpy as np
import pytest

from tensor_transformer_layer_linear_b200 import synth

from helpers import assert_parity, from_dev_bf16, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tp():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tensor_transformer_layer_linear_b200 import tp as _tp
    return _tp


def _shard(tp, W_dev, h_in, h_out, kind, n):
    out = torch.empty(h_in * h_out, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(W_dev, h_in, h_out, n, kind, 0, out)
    return out


def test_noalloc_matches_workspace_call_on_two_calls(tp):
    cfg = dict(kind="mlp", batch=2, seq=96, h=512, ffn=2048, x_std=1.0, w_std=0.05,
               b_std=0.05, residual=True)
    M, h, F, n = 192, 512, 2048, 4
    assert tp.tp_workspace_bytes(tp.TP_WS_MLP, M, h, F, n) <= tp.TP_NOALLOC_WS_BYTES
    for seed in (21, 22):   # two calls in a row, on different inputs
        inp = synth.make_inputs(cfg, seed=seed)
        dev = {k: to_dev(v) for k, v in inp.items()}
        A_s = _shard(tp, dev["A"], h, F, tp.TP_SPLIT_COLUMN, n)
        B_s = _shard(tp, dev["B"], F, h, tp.TP_SPLIT_ROW, n)
        nb = tp.tp_workspace_bytes(tp.TP_WS_MLP, M, h, F, n)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        Y_ref = torch.empty((M, h), dtype=torch.int16, device="cuda")
        tp.tp_mlp_forward(dev["X"], M, h, F, n, A_s, dev["b1"], B_s, dev["b2"], dev["X"], ws, nb,
                          Y_ref)
        Y = torch.full((M, h), 0x7FC0, dtype=torch.int16, device="cuda")   # NaN-filled
        tp.tp_mlp_forward_noalloc(dev["X"], M, h, F, n, A_s, dev["b1"], B_s, dev["b2"], dev["X"],
                                  Y)
        assert tp.tp_get_last_error() == tp.TP_OK
        assert_parity(from_dev_bf16(Y), from_dev_bf16(Y_ref), f"seed {seed}")


def test_noalloc_rejects_problems_beyond_the_array(tp):
    M, h, F, n = 4096, 1024, 4096, 4
    assert tp.tp_workspace_bytes(tp.TP_WS_MLP, M, h, F, n) > tp.TP_NOALLOC_WS_BYTES
    fake = 1 << 20   # never dereferenced: the size check comes first
    st = tp.lib.tp_mlp_forward_noalloc(fake, M, h, F, n, fake, None, fake, None, None, fake, None)
    assert st == tp.TP_ERR_WORKSPACE
    assert tp.tp_get_last_error() == tp.TP_OK
