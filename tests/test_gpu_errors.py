"""Error paths of the expert FFN on the GPU, through the C ABI:

  * a bounded device wait that runs out: the workspace's control block (the
    single-launch decode kernel's per-expert readiness counters) is preset so
    that one counter can never equal its expert's item count; with the wait
    limit lowered to about 1 ms the call reports MOE_DEV_ERR_TIMEOUT and
    returns, the kernel leaves the control block zeroed, and the next call
    matches the oracle;
  * a slot id past the pool reaching the FFN (MOE_DEV_ERR_SLOT_RANGE) on each
    kernel path: the expert is skipped, every other contribution is exact.
Nothing here faults, traps or hangs a GPU: every wait involved is bounded and
every slot id is range-checked before any copy."""
import numpy as np
import pytest
import torch

from streamed_quantized_expert_b200 import ops, synth
from tests._bank import assert_close
from tests.test_gpu_ffn import TOL, Setup, dev

pytestmark = pytest.mark.gpu


def _sorted(s, ids, T, ws, ws_b):
    E, k = s.E, s.k
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pairs = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
    active = torch.empty(E, dtype=torch.int32, device="cuda")
    na = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.moe_sort(dev(ids), None, T, s.d, offsets, pairs, active, na, None, ws, ws_b)
    return offsets, pairs, active, na


def test_readiness_wait_runs_out_then_recovers(orc):
    T = 1
    s = Setup(orc, 64, 4, 512, 256, 64, 4, 4, R=5, seed=31)
    assert ops.moe_ffn_kernel_path(s.d, T, False) == ops.MOE_PATH_FUSED_DECODE
    x = synth.activations(31, 0, T, 512)
    ids, w = synth.random_routing(31, T, 64, 4)
    ws_b = ops.moe_workspace_bytes(s.d, T)
    ws = torch.zeros(ws_b, dtype=torch.uint8, device="cuda")
    offsets, pairs, active, na = _sorted(s, ids, T, ws, ws_b)
    x_d, ids_d, w_d = dev(x.view(np.int16)), dev(ids), dev(w)

    def call():
        y = torch.zeros((T, 512), dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ops.moe_expert_ffn(x_d, T, s.d, s.pool, 64, s.table, ids_d, w_d, offsets, pairs, active, na, None, 0, 64, y,
                           ws, ws_b, err)
        torch.cuda.synchronize()
        return y.cpu().numpy(), int(err.item())

    # the first pass entry's readiness counter (first word of the control block)
    # starts far past its item count: the down CTAs' wait for it runs out
    ws[:4] = torch.tensor([0, 0, 0, 0x40], dtype=torch.uint8, device="cuda")
    ops.moe_set_wait_limit_cycles(2_000_000)
    try:
        _, err = call()
    finally:
        ops.moe_set_wait_limit_cycles(0)
    assert err & ops.DEV_ERR_TIMEOUT
    # the launch's last down CTA zeroed the control block again: the next calls are exact
    assert int(ws[:512].count_nonzero()) == 0
    y, err = call()
    assert err == 0
    assert_close(y, s.oracle(orc, x, ids, w), TOL)
    y2, err = call()
    assert err == 0 and np.array_equal(y, y2)


@pytest.mark.parametrize("T,sorted_x", [(2, False), (16, False), (40, True)])
def test_slot_past_the_pool_is_flagged_and_skipped(orc, T, sorted_x):
    s = Setup(orc, 32, 4, 256, 128, 64, 4, 4, R=5, seed=32)
    want = (ops.MOE_PATH_FUSED_DECODE if T <= 8 else ops.MOE_PATH_TC_PREFILL if sorted_x else ops.MOE_PATH_GEMV)
    assert ops.moe_ffn_kernel_path(s.d, T, sorted_x) == want
    x = synth.activations(32, 0, T, 256)
    ids, w = synth.random_routing(32, T, 32, 4)
    gone = int(ids[0, 2])
    table = s.perm.copy()
    table[gone] = 32 + 7  # the pool has 32 slots
    y, err = s.gpu(x, ids, w, T, table=dev(table), sorted_x=sorted_x)
    assert err & ops.DEV_ERR_SLOT_RANGE
    assert not err & ops.DEV_ERR_NOT_RESIDENT
    w2 = w.copy()
    w2[ids == gone] = 0.0
    assert_close(y, s.oracle(orc, x, ids, w2), TOL)
