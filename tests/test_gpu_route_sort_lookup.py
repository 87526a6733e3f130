"""moe_route_sort_lookup (one decode token's routing, sort and slot lookup in
one launch) through the C ABI: every output equal, bit for bit, to those of
moe_route (moe_route_shared with shared experts) + moe_sort + moe_slot_lookup
on the same inputs (which the oracle pins elsewhere), with and without
cache-aware substitution, with misses and an out-of-range slot; and its
routing against the oracle directly."""
import numpy as np
import pytest
import torch

from streamed_quantized_expert_b200 import build, ops, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run(E, k, logits, table, n_slots, L, fused, ns=0, sw=None):
    d = ops.desc(E, k, 64, 32, 32, 4, 4)
    dw = ops.widened(d, ns)
    Ew, kw = E + ns, k + ns
    lg, tab = dev(logits), dev(table)
    swd = None if sw is None else dev(np.array([sw], np.float32))
    z = lambda n, dt=torch.int32: torch.full((n,), -7, dtype=dt, device="cuda")  # noqa: E731
    ids, w, off, pairs = z(kw), z(kw, torch.float32), z(Ew + 1), z(kw)
    act, na, slots, miss, nmiss, err = z(Ew), z(1), z(Ew), z(Ew), z(1), torch.zeros(1, dtype=torch.int32, device="cuda")
    if fused:
        ops.moe_route_sort_lookup(lg, 1, d, L, tab, n_slots, ids, w, off, pairs, act, na, slots, miss, nmiss, err,
                                  n_shared=ns, shared_w=swd)
    else:
        if ns:
            ops.moe_route_shared(lg, 1, d, L, tab, ns, swd, ids, w)
        else:
            ops.moe_route(lg, 1, d, L, tab, ids, w)
        ws_b = ops.moe_workspace_bytes(dw, 1)
        ws = torch.zeros(max(ws_b, 256), dtype=torch.uint8, device="cuda")
        ops.moe_sort(ids, None, 1, dw, off, pairs, act, na, None, ws, ws_b)
        ops.moe_slot_lookup(tab, act, na, 0, Ew, n_slots, slots, miss, nmiss, err)
    torch.cuda.synchronize()
    n, nm = int(na.item()), int(nmiss.item())
    return {"ids": ids.cpu().numpy(), "w": w.cpu().numpy(), "off": off.cpu().numpy(), "pairs": pairs.cpu().numpy(),
            "n": n, "active": act.cpu().numpy()[:n], "slots": slots.cpu().numpy()[:n], "nm": nm,
            "miss": miss.cpu().numpy()[:nm], "err": int(err.item())}


@pytest.mark.parametrize("E,k", [(8, 2), (64, 4), (128, 8), (512, 10), (1000, 32)])
@pytest.mark.parametrize("L", [0.0, 0.15])
def test_one_launch_equals_three_calls(orc, E, k, L):
    rng = np.random.default_rng(E + k)
    for step in range(3):
        logits = synth.router_logits(5, 0, 1, E, step=step)
        if step == 2:  # ties: equal logits across experts
            logits = np.round(logits * 2.0) / 2.0
        n_slots = E // 2 + 1
        table = np.full(E, -1, np.int32)
        res = rng.choice(E, n_slots - 1, replace=False)
        table[res] = rng.permutation(n_slots - 1).astype(np.int32)
        if step == 1:
            table[res[0]] = n_slots + 3  # out of range: flagged by the lookup
        a = run(E, k, logits, table, n_slots, L, True)
        b = run(E, k, logits, table, n_slots, L, False)
        for key in a:
            assert np.array_equal(a[key], b[key]), (key, a[key], b[key])
        ids, w, _ = orc.route(logits, k, L, table)
        assert np.array_equal(a["ids"], ids[0])
        assert np.max(np.abs(a["w"] - w[0])) <= 1e-5  # the oracle's weights (fp64 sum) within fp32 rounding


@pytest.mark.parametrize("E,k,ns", [(64, 4, 1), (128, 8, 2), (512, 24, 8), (1000, 30, 2), (16, 16, 3)])
@pytest.mark.parametrize("L", [0.0, 0.15])
def test_one_launch_with_shared_experts(orc, E, k, ns, L):
    """Shared experts E .. E + ns - 1 after the top k (up to 32 pairs in all),
    one shared expert without a slot and misses among the routed ones."""
    rng = np.random.default_rng(E * 3 + k + ns)
    for step in range(2):
        logits = synth.router_logits(6, 0, 1, E, step=step)
        n_slots = E // 2 + ns + 1
        table = np.full(E + ns, -1, np.int32)
        res = rng.choice(E, E // 2, replace=False)
        perm = rng.permutation(n_slots).astype(np.int32)
        table[res] = perm[:E // 2]
        table[E:] = perm[E // 2:E // 2 + ns]
        if step == 1:
            table[E + ns - 1] = -1  # a shared expert without a slot: listed last among the misses
        sw = None if step == 0 else 0.375
        a = run(E, k, logits, table, n_slots, L, True, ns, sw)
        b = run(E, k, logits, table, n_slots, L, False, ns, sw)
        for key in a:
            assert np.array_equal(a[key], b[key]), (key, a[key], b[key])
        ids, w, _ = orc.route(logits, k, L, table[:E])
        assert np.array_equal(a["ids"][:k], ids[0])
        assert np.array_equal(a["ids"][k:], np.arange(E, E + ns))
        assert np.all(a["w"][k:] == (1.0 if sw is None else sw))
        assert a["n"] == k + ns and np.array_equal(a["active"], np.sort(a["ids"]))
        if step == 1:
            assert a["miss"][-1] == E + ns - 1


def test_more_than_one_token_is_unsupported():
    d = ops.desc(64, 4, 64, 32, 32, 4, 4)
    z = lambda n, dt=torch.int32: torch.zeros((n,), dtype=dt, device="cuda")  # noqa: E731
    with pytest.raises(ops.MoeError) as ei:
        ops.moe_route_sort_lookup(z(128, torch.float32), 2, d, 0.0, z(64), 64, z(8), z(8, torch.float32), z(65),
                                  z(8), z(64), z(1), z(64), z(64), z(1), z(1))
    assert ei.value.status == ops.MOE_ERR_UNSUPPORTED


def test_more_than_32_pairs_with_shared_experts_is_unsupported():
    d = ops.desc(64, 30, 64, 32, 32, 4, 4)
    z = lambda n, dt=torch.int32: torch.zeros((n,), dtype=dt, device="cuda")  # noqa: E731
    with pytest.raises(ops.MoeError) as ei:
        ops.moe_route_sort_lookup(z(64, torch.float32), 1, d, 0.0, z(67), 64, z(33), z(33, torch.float32), z(68),
                                  z(33), z(67), z(1), z(67), z(67), z(1), z(1), n_shared=3)
    assert ei.value.status == ops.MOE_ERR_UNSUPPORTED
