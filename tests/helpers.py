"""Shared test helpers: bf16 bit arrays <-> torch tensors, the parity gate.

With TP_PARITY_LOG set to a file path, every parity check appends its
observed errors to that file as one JSON line."""
import json
import os

import numpy as np

from tensor_transformer_layer_linear_b200 import synth

# Value tolerance of the parity gate: max|gpu - oracle| <= MAX_REL * max|oracle|
# and ||gpu - oracle||_F / ||oracle||_F <= FRO_REL.
MAX_REL = 2e-2
FRO_REL = 5e-3

# Gate for backward outputs: a backward re-traverses the forward's
# bf16-stored intermediates (x1, QKV, O, P, h1, x2, GeLU(Z)) and adds its own
# (GeLU'(Z), dZ, dh1, dO, P, dS, dQKV; grouped key/value gradients also sum a
# group of query heads), about twice as many bf16 roundings (relative error
# <= 2^-9 each, RMS 2^-9/sqrt 3) in the longest chain as the forward, so the
# Frobenius bound doubles. Backward tests that pass the forward gate keep it.
BWD_FRO_REL = 1e-2


def to_dev(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def from_dev_bf16(t) -> np.ndarray:
    """Device bf16 (int16 bits) -> float64 numpy."""
    return synth.bf16_bits_to_f64(t.cpu().numpy().view(np.uint16))


def f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f64(bits)


def assert_parity(gpu: np.ndarray, ref: np.ndarray, what: str = "",
                  max_rel: float = MAX_REL, fro_rel: float = FRO_REL) -> dict:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    err = np.abs(gpu - ref)
    scale = np.max(np.abs(ref))
    fro = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300)
    stats = dict(max_abs=float(err.max()), max_ref=float(scale), fro_rel=float(fro))
    log = os.environ.get("TP_PARITY_LOG")
    if log:   # observed errors, one JSON line per check (for the tolerance notes)
        with open(log, "a") as f:
            f.write(json.dumps(dict(test=os.environ.get("PYTEST_CURRENT_TEST", ""), what=what,
                                    max_rel_gate=max_rel, fro_gate=fro_rel,
                                    max_rel=stats["max_abs"] / max(stats["max_ref"], 1e-300),
                                    **stats)) + "\n")
    assert err.max() <= max_rel * scale, f"{what}: max error {stats}"
    assert fro <= fro_rel, f"{what}: Frobenius error {stats}"
    return stats
