"""Test helpers: expert banks built by the oracle's quantizer from seeded
synthetic weights, device upload helpers, and the tolerance check."""
import numpy as np

from streamed_quantized_expert_b200 import synth

_CACHE = {}


def oracle_bank(orc, n_rows, H, I, g, b_gu, b_d, seed=0):
    """uint8 [n_rows, slot_bytes]: row r = quantized synth.expert_weights(seed, r)."""
    key = (n_rows, H, I, g, b_gu, b_d, seed)
    if key not in _CACHE:
        rows = [orc.build_slot(*synth.expert_weights(seed, r, H, I), g, b_gu, b_d) for r in range(n_rows)]
        _CACHE[key] = np.stack(rows)
    return _CACHE[key]


def assert_close(y, ref, tol=2e-2, what="y"):
    """|y - r| <= tol * max(|r|, rms of r's row), elementwise."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    rms = np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True))
    bound = tol * np.maximum(np.abs(ref), rms)
    err = np.abs(y - ref)
    bad = err > bound
    normwise = float(np.max(np.linalg.norm(y - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)))
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; max err/bound "
                           f"{float(np.max(err / np.maximum(bound, 1e-30))):.3g}; normwise {normwise:.3g}")
    return normwise
