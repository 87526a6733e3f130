"""moe_route_sort_lookup (one decode token's routing, sort and slot lookup in
one launch) through the C ABI: every output equal, bit for bit, to those of
moe_route + moe_sort + moe_slot_lookup on the same inputs (which the oracle
pins elsewhere), with and without cache-aware substitution, with misses and
an out-of-range slot; and its routing against the oracle directly."""
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


def run(E, k, logits, table, n_slots, L, fused):
    d = ops.desc(E, k, 64, 32, 32, 4, 4)
    lg, tab = dev(logits), dev(table)
    z = lambda n, dt=torch.int32: torch.full((n,), -7, dtype=dt, device="cuda")  # noqa: E731
    ids, w, off, pairs = z(k), z(k, torch.float32), z(E + 1), z(k)
    act, na, slots, miss, nmiss, err = z(E), z(1), z(E), z(E), z(1), torch.zeros(1, dtype=torch.int32, device="cuda")
    if fused:
        ops.moe_route_sort_lookup(lg, 1, d, L, tab, n_slots, ids, w, off, pairs, act, na, slots, miss, nmiss, err)
    else:
        ops.moe_route(lg, 1, d, L, tab, ids, w)
        ws_b = ops.moe_workspace_bytes(d, 1)
        ws = torch.zeros(max(ws_b, 256), dtype=torch.uint8, device="cuda")
        ops.moe_sort(ids, None, 1, d, off, pairs, act, na, None, ws, ws_b)
        ops.moe_slot_lookup(tab, act, na, 0, E, n_slots, slots, miss, nmiss, err)
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


def test_more_than_one_token_is_unsupported():
    d = ops.desc(64, 4, 64, 32, 32, 4, 4)
    z = lambda n, dt=torch.int32: torch.zeros((n,), dtype=dt, device="cuda")  # noqa: E731
    with pytest.raises(ops.MoeError) as ei:
        ops.moe_route_sort_lookup(z(128, torch.float32), 2, d, 0.0, z(64), 64, z(8), z(8, torch.float32), z(65),
                                  z(8), z(64), z(1), z(64), z(64), z(1), z(1))
    assert ei.value.status == ops.MOE_ERR_UNSUPPORTED
