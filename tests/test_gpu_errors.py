"""Error paths of the expert FFN on the GPU, through the C ABI:

  * bounded device waits that run out.  The single-launch decode kernel keeps
    a control word at the head of the workspace (launch epoch, arrival count)
    from which each launch takes the tag its h words carry.  Presetting the
    arrival count to half the grid splits a launch's CTAs over two tags, so
    the down side's reads of h (bounded, the wait limit lowered to about 1 ms)
    run out: the call reports MOE_DEV_ERR_TIMEOUT and returns.  A count at or
    past the grid makes every CTA report it without doing any work.  After
    the workspace is zeroed again the next calls match the oracle.  A plain
    run of calls on one workspace needs no zeroing in between (the count is
    complete after every launch).
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


def _item_split(G, nd, n_items, n_act, tile_gu, tile_d):
    """Gate/up items per CTA (the kernel's split: CTAs below nd also own a
    down tile; quotas by bytes)."""
    dn = n_act * tile_d
    tot = n_items * tile_gu + nd * dn

    def bound(c):
        if dn * G <= tot:
            f = max(c * tot - min(c, nd) * G * dn, 0)
            v = f // (G * tile_gu)
        else:
            v = (c - nd) * n_items // (G - nd) if c > nd else 0
        return min(v, n_items)

    return [bound(c + 1) - bound(c) for c in range(G)]


@pytest.mark.parametrize("arrivals", ["half_grid", "past_grid"])
def test_wait_runs_out_then_recovers(orc, arrivals):
    T, E, k, H, I = 1, 64, 4, 512, 1024
    s = Setup(orc, E, k, H, I, 64, 4, 4, R=5, seed=31)
    assert ops.moe_ffn_kernel_path(s.d, T, False) == ops.MOE_PATH_FUSED_DECODE
    G = torch.cuda.get_device_properties(0).multi_processor_count
    lay = ops.moe_slot_layout(s.d)
    split = _item_split(G, H // 16, k * (I // 8), k, lay.gate_up_tile_bytes, lay.down_tile_bytes)
    # every CTA has work (gate/up items or a down tile), so any split of the
    # grid over two tags leaves some down tile reading another tag's h
    assert all(n > 0 or c < H // 16 for c, n in enumerate(split))
    x = synth.activations(31, 0, T, H)
    ids, w = synth.random_routing(31, T, E, k)
    ws_b = ops.moe_workspace_bytes(s.d, T)
    ws = torch.zeros(ws_b, dtype=torch.uint8, device="cuda")
    offsets, pairs, active, na = _sorted(s, ids, T, ws, ws_b)
    x_d, ids_d, w_d = dev(x.view(np.int16)), dev(ids), dev(w)
    ref = s.oracle(orc, x, ids, w)

    def call():
        y = torch.zeros((T, H), dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ops.moe_expert_ffn(x_d, T, s.d, s.pool, E, s.table, ids_d, w_d, offsets, pairs, active, na, None, 0, E, y,
                           ws, ws_b, err)
        torch.cuda.synchronize()
        return y.cpu().numpy(), int(err.item())

    # a few good calls first: the control word carries over, no zeroing needed
    y0, err = call()
    assert err == 0
    assert_close(y0, ref, TOL)
    for _ in range(3):
        y, err = call()
        assert err == 0 and np.array_equal(y, y0)
    word = int(ws[:8].cpu().numpy().view(np.uint64)[0])
    assert word & 0xFFFFFFFF == 0 and word >> 32 == 4  # four complete launches
    count = G // 2 if arrivals == "half_grid" else 1 << 30
    ws[:8] = torch.from_numpy(np.array([(word & ~0xFFFFFFFF) | count], dtype=np.uint64).view(np.uint8)).cuda()
    ops.moe_set_wait_limit_cycles(2_000_000)
    try:
        y, err = call()
    finally:
        ops.moe_set_wait_limit_cycles(0)
    assert err & ops.DEV_ERR_TIMEOUT
    if arrivals == "past_grid":
        assert not y.any()  # no CTA did any work
    # the count stays off until the workspace is zeroed; then the calls are exact again
    ws.zero_()
    y, err = call()
    assert err == 0 and np.array_equal(y, y0)
    y, err = call()
    assert err == 0 and np.array_equal(y, y0)


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
