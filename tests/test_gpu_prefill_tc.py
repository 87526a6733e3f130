"""GPU vs oracle for the expert FFN on the tcgen05 grouped GEMM (prefill
chunks and batched decode, wherever the fused decode kernel does not apply, with sorted activations):
dequantised weight tiles in the
128-byte swizzled layout, token tiles by TMA, fp32 accumulators in TMEM.
Within 2e-2 of max(|ref|, row rms) elementwise on sampled token rows (the
oracle computes them one by one), and equal to the GEMV path within the
same tolerance on every row."""
import numpy as np
import pytest

from streamed_quantized_expert_b200 import ops, synth
from tests._bank import assert_close
from tests.test_gpu_ffn import Setup, TOL

pytestmark = pytest.mark.gpu


def _case(orc, E, k, H, I, g, bg, bd, T, R, seed, routing="random"):
    s = Setup(orc, E, k, H, I, g, bg, bd, R, seed)
    x = synth.activations(seed, 1, T, H)
    if routing == "random":
        ids, w = synth.random_routing(seed, T, E, k)
    else:  # Zipf-skewed: a few experts get most tokens (several token tiles each)
        logits = synth.router_logits(seed, 0, T, E, beta=1.0)
        ids, w, _ = orc.route(logits, k)
        w = w.astype(np.float32)
    assert ops.moe_ffn_kernel_path(s.d, T, True) == ops.MOE_PATH_TC_PREFILL
    return s, x, ids, w


def _check(orc, s, x, ids, w, T, passes=None, ntok=6):
    y, err = s.gpu(x, ids, w, T, passes=passes, sorted_x=True)
    assert err == 0
    assert np.isfinite(y).all()
    tok = np.unique(np.linspace(0, T - 1, ntok).astype(int))
    assert_close(y[tok], s.oracle(orc, x, ids, w, tok), TOL)
    return y


def test_flash_next_prefill_passes(orc):
    # 512 experts, top-10, H 2048, I 512, 3-bit g64; passes of 64 active experts
    s, x, ids, w = _case(orc, 512, 10, 2048, 512, 64, 3, 3, 300, R=8, seed=11)
    passes = [(p, 64) for p in range(0, 512, 64)]
    _check(orc, s, x, ids, w, 300, passes)


def test_mixed_class_prefill_4_6(orc):
    # 4-bit gate/up, 6-bit down (the second size class), Zipf routing
    s, x, ids, w = _case(orc, 512, 10, 2048, 512, 64, 4, 6, 384, R=8, seed=12, routing="zipf")
    passes = [(p, 64) for p in range(0, 512, 64)]
    _check(orc, s, x, ids, w, 384, passes)


def test_coder_shape_prefill(orc):
    # 128 experts, top-8, H 2048, I 768, 4-bit g64 (I = 6 blocks of 128)
    s, x, ids, w = _case(orc, 128, 8, 2048, 768, 64, 4, 4, 512, R=6, seed=13)
    _check(orc, s, x, ids, w, 512, [(0, 64), (64, 64)])


@pytest.mark.parametrize("T", [7, 8, 9])
def test_few_tokens_past_the_fused_range(orc, T):
    # top-10 at 7 and 8 tokens (70 and 80 pairs) is past the fused decode kernel: every row, and the
    # same values as the GEMV kernels within the tolerance
    s, x, ids, w = _case(orc, 64, 10, 256, 128, 64, 3, 3, T, R=5, seed=30 + T)
    y = _check(orc, s, x, ids, w, T, ntok=T)
    y2, err = s.gpu(x, ids, w, T, sorted_x=False)
    assert err == 0
    assert_close(y, y2, TOL)


@pytest.mark.parametrize("g,bg,bd", [(32, 3, 4), (128, 6, 3), (64, 4, 4)])
def test_groups_widths_multi_tile_experts(orc, g, bg, bd):
    # 8 experts, top-2, 600 tokens: ~150 tokens per expert -> 2 token tiles each
    s, x, ids, w = _case(orc, 8, 2, 384, 256, g, bg, bd, 600, R=8, seed=g + bg + bd)
    _check(orc, s, x, ids, w, 600, ntok=8)


def test_matches_gemv_path_every_row(orc):
    s, x, ids, w = _case(orc, 64, 4, 512, 256, 64, 4, 4, 320, R=8, seed=14)
    assert ops.moe_ffn_kernel_path(s.d, 320, False) == ops.MOE_PATH_GEMV
    tc, e1 = s.gpu(x, ids, w, 320, sorted_x=True)
    gemv, e2 = s.gpu(x, ids, w, 320, sorted_x=False)
    assert e1 == 0 and e2 == 0
    assert_close(tc, gemv.astype(np.float64), TOL)


def test_non_resident_expert_flagged_on_tc_path(orc):
    s, x, ids, w = _case(orc, 64, 4, 512, 256, 64, 4, 4, 320, R=8, seed=15)
    table = s.table.clone()
    gone = int(ids[0, 0])
    table[gone] = -1
    y, err = s.gpu(x, ids, w, 320, table=table, sorted_x=True)
    assert err & ops.DEV_ERR_NOT_RESIDENT
    # the expert is skipped: token rows that never routed to it are unaffected
    keep = np.array([t for t in range(320) if gone not in ids[t]][:4])
    assert_close(y[keep], s.oracle(orc, x, ids, w, keep), TOL)


@pytest.mark.parametrize("T", [32, 64])
def test_coder_batched_decode_on_tensor_cores(orc, T):
    # batched decode (Coder-like: 128 experts, top-8, H 2048, I 768, 4-bit g64) with sorted x
    # takes the tensor-core path from 32 tokens, one call over every expert (split into
    # launches of 64 experts inside the library)
    s, x, ids, w = _case(orc, 128, 8, 2048, 768, 64, 4, 4, T, R=6, seed=16 + T)
    _check(orc, s, x, ids, w, T, passes=[(0, 128)], ntok=4)
