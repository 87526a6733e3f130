"""moe_expert_ffn_noalloc: the FFN entry point for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).
Checked through the C ABI against moe_expert_ffn, which takes a caller
workspace, on two calls in a row with different inputs.  Kept in a file that
runs last, and self-contained so that it also passes alone."""
import numpy as np
import pytest
import torch

from streamed_quantized_expert_b200 import build, ops, synth
from tests._bank import assert_close

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("T", [6, 16])
def test_noalloc_matches_workspace_entry_point(T):
    # T = 6: the single-launch decode kernel; T = 16: the gate/up + down GEMV kernels
    build.build()
    E, k, H, I, g, b = 64, 4, 512, 256, 64, 4
    d = ops.desc(E, k, H, I, g, b, b)
    assert ops.moe_ffn_kernel_path(d, T, False) == (ops.MOE_PATH_FUSED_DECODE if T <= 8 else ops.MOE_PATH_GEMV)
    sb = ops.moe_slot_bytes(d)
    lay = ops.moe_slot_layout(d)
    pool = torch.zeros((E, sb), dtype=torch.uint8, device="cuda")
    for e in range(E):
        w_gu, w_d = synth.expert_weights_torch(3, e, H, I, "cuda")
        base = pool[e].data_ptr()
        ops.moe_quantize_rows(w_gu, 2 * I, H, g, b, base + lay.gate_up, gate_up_I=I)
        ops.moe_quantize_rows(w_d, H, I, g, b, base + lay.down)
    table = torch.arange(E, dtype=torch.int32, device="cuda")
    ws_b = ops.moe_workspace_bytes(d, T)
    assert ws_b <= ops.moe_noalloc_scratch_bytes()
    ws = torch.zeros(ws_b, dtype=torch.uint8, device="cuda")
    for call in range(2):
        x = dev(synth.activations(10 + call, 0, T, H).view(np.int16))
        ids_np, w_np = synth.random_routing(20 + call, T, E, k)
        ids, w = dev(ids_np), dev(w_np)
        offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        pairs = torch.empty(T * k, dtype=torch.int32, device="cuda")
        active = torch.empty(E, dtype=torch.int32, device="cuda")
        na = torch.zeros(1, dtype=torch.int32, device="cuda")
        ops.moe_sort(ids, None, T, d, offsets, pairs, active, na, None, ws, ws_b)
        err = torch.zeros(2, dtype=torch.int32, device="cuda")
        y_ref = torch.zeros((T, H), dtype=torch.float32, device="cuda")
        y_na = torch.zeros((T, H), dtype=torch.float32, device="cuda")
        ops.moe_expert_ffn(x, T, d, pool, E, table, ids, w, offsets, pairs, active, na, None, 0, E, y_ref, ws, ws_b,
                           err[0:1])
        ops.moe_expert_ffn_noalloc(x, T, d, pool, E, table, ids, w, offsets, pairs, active, na, 0, E, y_na,
                                   err[1:2])
        torch.cuda.synchronize()
        assert err.tolist() == [0, 0]
        assert float(y_ref.abs().max()) > 0.0
        assert_close(y_na.cpu().numpy(), y_ref.cpu().numpy(), 2e-2, what=f"noalloc call {call}")


def test_noalloc_rejects_sizes_past_its_scratch():
    build.build()
    d = ops.desc(64, 4, 512, 256, 64, 4, 4)
    with pytest.raises(ops.MoeError) as ei:  # T above 64
        ops.moe_expert_ffn_noalloc(1 << 20, 65, d, 1 << 24, 64, 1 << 21, 1 << 21, 1 << 21, 1 << 21, 1 << 21,
                                   1 << 21, 1 << 21, 0, 64, 1 << 21, None)
    assert ei.value.status == ops.MOE_ERR_CAPACITY
    big = ops.desc(512, 32, 2048, 4096, 64, 4, 4)  # 64 x 32 pairs x 4096 x 2 B of h > 1 MiB
    with pytest.raises(ops.MoeError) as ei:
        ops.moe_expert_ffn_noalloc(1 << 20, 64, big, 1 << 24, 64, 1 << 21, 1 << 21, 1 << 21, 1 << 21, 1 << 21,
                                   1 << 21, 1 << 21, 0, 64, 1 << 21, None)
    assert ei.value.status == ops.MOE_ERR_CAPACITY
