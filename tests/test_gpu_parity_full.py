"""GPU vs oracle at the full sizes of the prefill and batched-decode
workloads, every output row compared (within 2e-2 of max(|ref|, row rms),
elementwise):

  * a Flash-Next-like prefill chunk: 1024 tokens, 512 experts, top-10,
    H 2048, I 512, 3-bit g64, routed by the log-Zipf-biased logits of the
    benchmark (about 440 active experts, 7 passes of 64, the hottest expert
    with about 750 tokens = 6 token tiles);
  * a mixed-class prefill chunk: 4096 tokens, 4-bit gate/up with 6-bit down
    (the second size class) and the 4/4-bit class (about 510 active experts,
    8 passes, the hottest expert with about 3000 tokens = 24 token tiles);
  * Coder-like batched decode (128 experts, top-8, H 2048, I 768, 4-bit g64)
    at 32 and 64 tokens on the tensor-core path and on the GEMV path.

The oracle rows are evaluated pair by pair on a thread pool (bit-identical to
one oracle call, see tests/_bank.py).  Experts are R distinct quantized weight
sets (R prime, so experts that share a weight set are never a pass or a
power of two apart), each resident in its own slot of a permuted pool."""
import numpy as np
import pytest

from streamed_quantized_expert_b200 import ops, synth
from tests._bank import assert_close, oracle_bank_parallel, oracle_rows_parallel
from tests.test_gpu_ffn import TOL, Setup

pytestmark = pytest.mark.gpu

R = 61


def _routed(orc, E, k, T, layer, seed=0):
    logits = synth.router_logits(seed, layer, T, E)
    ids, w, _ = orc.route(logits, k)
    return ids, w.astype(np.float32)


def _passes(ids, E):
    n_act = int((np.bincount(ids.ravel(), minlength=E) > 0).sum())
    return [(p, 64) for p in range(0, n_act, 64)], n_act


def test_flash_next_prefill_chunk_every_row(orc):
    E, k, H, I, g, T = 512, 10, 2048, 512, 64, 1024
    oracle_bank_parallel(orc, R, H, I, g, 3, 3, 21)
    s = Setup(orc, E, k, H, I, g, 3, 3, R=R, seed=21)
    assert ops.moe_ffn_kernel_path(s.d, T, True) == ops.MOE_PATH_TC_PREFILL
    ids, w = _routed(orc, E, k, T, layer=0)
    counts = np.bincount(ids.ravel(), minlength=E)
    passes, n_act = _passes(ids, E)
    assert n_act > 400 and counts.max() > 5 * 128  # nearly all experts; a 6-tile expert
    x = synth.activations(0, 0, T, H)
    y, err = s.gpu(x, ids, w, T, passes=passes, sorted_x=True)
    assert err == 0
    assert_close(y, oracle_rows_parallel(orc, x, s.geom, ids, w, s.slots_np), TOL, what="prefill T=1024")


@pytest.mark.parametrize("bd,layer", [(6, 0), (4, 1)])
def test_mixed_class_prefill_chunk_every_row(orc, bd, layer):
    E, k, H, I, g, T = 512, 10, 2048, 512, 64, 4096
    oracle_bank_parallel(orc, R, H, I, g, 4, bd, 22)
    s = Setup(orc, E, k, H, I, g, 4, bd, R=R, seed=22)
    ids, w = _routed(orc, E, k, T, layer=layer)
    counts = np.bincount(ids.ravel(), minlength=E)
    passes, n_act = _passes(ids, E)
    assert n_act > 500 and counts.max() > 20 * 128
    x = synth.activations(0, layer, T, H)
    y, err = s.gpu(x, ids, w, T, passes=passes, sorted_x=True)
    assert err == 0
    assert_close(y, oracle_rows_parallel(orc, x, s.geom, ids, w, s.slots_np), TOL, what=f"prefill T=4096 4/{bd}")


@pytest.mark.parametrize("T", [12, 32, 64])
@pytest.mark.parametrize("sorted_x", [True, False])
def test_coder_batched_decode_every_row(orc, T, sorted_x):
    E, k, H, I, g = 128, 8, 2048, 768, 64
    oracle_bank_parallel(orc, R, H, I, g, 4, 4, 23)
    s = Setup(orc, E, k, H, I, g, 4, 4, R=R, seed=23)
    want = ops.MOE_PATH_TC_PREFILL if sorted_x else ops.MOE_PATH_GEMV
    assert ops.moe_ffn_kernel_path(s.d, T, sorted_x) == want
    x = synth.activations(1, 3, T, H)
    ids, w = _routed(orc, E, k, T, layer=3, seed=1)
    y, err = s.gpu(x, ids, w, T, sorted_x=sorted_x)
    assert err == 0
    assert_close(y, oracle_rows_parallel(orc, x, s.geom, ids, w, s.slots_np), TOL, what=f"coder T={T}")
