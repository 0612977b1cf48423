"""tp_layer_forward and tp_mlp_backward captured in a CUDA graph on a B200.

The block calls launch kernels only (no host synchronisation, no
allocation), so a caller can capture a whole layer step once and replay it:
the replay must give the same bits as the same calls made eagerly, for new
input values written into the captured buffers before each replay.
"""
import numpy as np
import pytest

from tensor_transformer_layer_linear_b200 import synth

from helpers import to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tp():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tensor_transformer_layer_linear_b200 import tp as _tp
    return _tp


def _shard(tp, W_dev, h_in, h_out, kind, n, head_dim=0):
    out = torch.empty(h_in * h_out, dtype=torch.int16, device="cuda")
    tp.tp_shard_weights(W_dev, h_in, h_out, n, kind, head_dim, out)
    return out


def test_layer_forward_graph_replay(tp):
    cfg = dict(kind="layer", batch=2, seq=160, h=512, n_heads=4, ffn=2048, x_std=1.0,
               w_std=0.05, b_std=0.05, ln_eps=1e-5)
    b, s, h, nh, F, n = 2, 160, 512, 4, 2048, 2
    M = b * s
    inp = synth.make_inputs(cfg, seed=11)
    dev = {k: to_dev(v) for k, v in inp.items()}
    w = tp.make_layer_weights(
        ln1_gamma=dev["ln1_g"], ln1_beta=dev["ln1_b"],
        Wqkv_shards=_shard(tp, dev["Wqkv"], h, 3 * h, 2, n, h // nh),
        bqkv_shards=_shard(tp, dev["bqkv"], 1, 3 * h, 2, n, h // nh),
        Wo_shards=_shard(tp, dev["Wo"], h, h, 1, n), bo=dev["bo"],
        ln2_gamma=dev["ln2_g"], ln2_beta=dev["ln2_b"],
        A_shards=_shard(tp, dev["A"], h, F, 0, n), b1_shards=dev["b1"],
        B_shards=_shard(tp, dev["B"], F, h, 1, n), b2=dev["b2"])
    nb = tp.tp_workspace_bytes(tp.TP_WS_LAYER, M, h, F, n)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    X = dev["X"].clone()
    Y_graph = torch.empty((M, h), dtype=torch.int16, device="cuda")
    Y_eager = torch.empty_like(Y_graph)

    def step(out):
        tp.tp_layer_forward(X, b, s, h, nh, F, n, w, 1e-5, ws, nb, out)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(Y_graph)          # first calls set up the kernels outside the capture
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(Y_graph)
    rng = np.random.default_rng(12)
    for _ in range(2):
        X.copy_(to_dev(synth.f32_to_bf16_bits(rng.standard_normal((M, h), dtype=np.float32))))
        graph.replay()
        step(Y_eager)
        torch.cuda.synchronize()
        assert tp.tp_get_last_error() == tp.TP_OK
        assert torch.equal(Y_graph, Y_eager)


def test_mlp_backward_graph_replay(tp):
    rng = np.random.default_rng(13)
    M, h, F, n = 256, 256, 1024, 2
    bits = lambda shape, std: to_dev(synth.f32_to_bf16_bits(
        rng.standard_normal(shape, dtype=np.float32) * np.float32(std)))
    X, A, B, b1, dY = bits((M, h), 1.0), bits((h, F), 0.05), bits((F, h), 0.05), bits((F,), 0.05), \
        bits((M, h), 1.0)
    A_s = _shard(tp, A, h, F, 0, n)
    B_s = _shard(tp, B, F, h, 1, n)
    nb = tp.tp_workspace_bytes(tp.TP_WS_MLP_BWD, M, h, F, n)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")

    def outputs():
        return dict(dX=torch.empty((M, h), dtype=torch.int16, device="cuda"),
                    dA=torch.empty(h * F, dtype=torch.float32, device="cuda"),
                    db1=torch.empty(F, dtype=torch.float32, device="cuda"),
                    dB=torch.empty(F * h, dtype=torch.float32, device="cuda"),
                    db2=torch.empty(h, dtype=torch.float32, device="cuda"))
    g_out, e_out = outputs(), outputs()

    def step(o):
        tp.tp_mlp_backward(X, M, h, F, n, A_s, b1, B_s, dY, True, ws, nb, o["dX"], o["dA"],
                           o["db1"], o["dB"], o["db2"])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(g_out)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(g_out)
    dY.copy_(bits((M, h), 1.0))
    graph.replay()
    step(e_out)
    torch.cuda.synchronize()
    assert tp.tp_get_last_error() == tp.TP_OK
    for k in g_out:
        assert torch.equal(g_out[k], e_out[k]), k
