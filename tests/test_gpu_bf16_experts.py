"""Unquantized BF16 experts (RFC "stream MoE experts from disk in
from_pretrained", "How the prototype works", item "Cache": BF16 experts run
through the grouped experts kernel), through the C ABI, against the oracle:
16-bit slots (rows of bf16 values) on the tcgen05 grouped GEMM at every T,
alone and mixed with a quantized projection; every row compared."""
import numpy as np
import pytest
import torch

from streamed_quantized_expert_b200 import ops, synth
from tests._bank import assert_close
from tests.test_gpu_ffn import TOL, Setup

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,bits", [(1, (16, 16)), (6, (16, 16)), (40, (16, 16)), (300, (16, 16)),
                                    (64, (16, 4)), (33, (4, 16))])
def test_bf16_experts_every_row(orc, T, bits):
    E, k, H, I, g = 48, 4, 512, 256, 64
    s = Setup(orc, E, k, H, I, g, *bits, R=5, seed=51)
    assert ops.moe_ffn_kernel_path(s.d, T, True) == ops.MOE_PATH_TC_PREFILL
    x = synth.activations(51, 0, T, H)
    ids, w = synth.random_routing(51, T, E, k)
    y, err = s.gpu(x, ids, w, T, sorted_x=True)
    assert err == 0
    assert_close(y, s.oracle(orc, x, ids, w), TOL)


def test_bf16_experts_coder_shapes_every_row(orc):
    # Coder-like shapes (E 128, top-8, H 2048, I 768) at 64 tokens, BF16 experts
    E, k, H, I, g, T = 128, 8, 2048, 768, 64, 64
    s = Setup(orc, E, k, H, I, g, 16, 16, R=7, seed=52)
    x = synth.activations(52, 0, T, H)
    logits = synth.router_logits(52, 0, T, E)
    ids, w, _ = orc.route(logits, k)
    y, err = s.gpu(x, ids, w.astype(np.float32), T, sorted_x=True)
    assert err == 0
    assert_close(y, s.oracle(orc, x, ids, w), TOL)


def test_bf16_experts_need_sorted_x(orc):
    s = Setup(orc, 16, 2, 256, 128, 64, 16, 16, R=3, seed=53)
    assert ops.moe_ffn_kernel_path(s.d, 4, False) == -1
    with pytest.raises(ops.MoeError) as ex:
        s.gpu(synth.activations(53, 0, 4, 256), *synth.random_routing(53, 4, 16, 2), 4, sorted_x=False)
    assert ex.value.status == ops.MOE_ERR_UNSUPPORTED
