"""The failure path on a B200, without a GPU fault: a bounded wait that
expires (a one-thread kernel waiting on an mbarrier nothing arrives on)
records a bit in the device's error word, tp_get_last_error reports
TP_ERR_TIMEOUT once and clears it, and the context stays usable: a GEMM run
right after is still exact."""
import numpy as np
import pytest

from oracle import tp_oracle as O
from tensor_transformer_layer_linear_b200 import synth

from helpers import f64, from_dev_bf16, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tp():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tensor_transformer_layer_linear_b200 import tp as _tp
    return _tp


def test_expired_wait_is_reported_and_the_context_survives(tp):
    assert tp.tp_get_last_error() == tp.TP_OK
    tp.tp_selftest_wait_timeout(20000)  # 20 ms
    assert tp.tp_get_last_error() == tp.TP_ERR_TIMEOUT
    assert tp.tp_get_last_error() == tp.TP_OK  # the word was cleared
    # a column GEMM on integer-valued inputs afterwards is still exact
    rng = np.random.default_rng(1500)
    # entries in {-1, 0, 1} and K = 128: every sum is an integer of magnitude
    # <= 128, exact in fp32 and in bf16
    B, h_in, h_out, n = 256, 128, 512, 2
    X = synth.f32_to_bf16_bits(rng.integers(-1, 2, size=(B, h_in)).astype(np.float32))
    W = synth.f32_to_bf16_bits(rng.integers(-1, 2, size=(h_in, h_out)).astype(np.float32))
    Ws = torch.empty(h_in * h_out, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(to_dev(W), h_in, h_out, n, tp.TP_SPLIT_COLUMN, 0, Ws)
    Y = torch.empty((n, B, h_out // n), dtype=torch.int16, device="cuda")
    tp.tp_column_linear(to_dev(X), B, h_in, Ws, None, h_out, n, tp.TP_ACT_NONE, Y)
    assert tp.tp_get_last_error() == tp.TP_OK
    got = from_dev_bf16(Y)
    ref = f64(X) @ f64(W)
    for i in range(n):
        w = h_out // n
        assert np.array_equal(got[i], ref[:, i * w:(i + 1) * w])


def test_selftest_limit_is_checked(tp):
    for bad in (0, 1000001):
        with pytest.raises(tp.TPError) as e:
            tp.tp_selftest_wait_timeout(bad)
        assert e.value.status == tp.TP_ERR_SHAPE
