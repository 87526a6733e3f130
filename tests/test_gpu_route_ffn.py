"""moe_route_expert_ffn (every stage of one decode token of a resident layer
in one launch; RFC "How the prototype works", item "Cache") through the C
ABI: its routing, sort and lookup equal those of moe_route_sort_lookup bit
for bit, its y is the oracle's, with and without cache-aware substitution,
and a routed expert without a slot is listed as a miss, flagged and skipped."""
import numpy as np
import pytest
import torch

from streamed_quantized_expert_b200 import ops, synth
from tests._bank import assert_close
from tests.test_gpu_ffn import Setup, dev

pytestmark = pytest.mark.gpu
TOL = 2e-2


def run_both(s, logits, x, L=0.0, table=None):
    """(one launch, stages launch + FFN) outputs as numpy dicts."""
    E, k, H = s.E, s.k, s.H
    tab = s.table if table is None else table
    lg, xd = dev(logits), dev(x.view(np.int16))
    ws_b = ops.moe_workspace_bytes(s.d, 1)
    out = []
    for fused in (True, False):
        z = lambda n, dt=torch.int32: torch.full((n,), -7, dtype=dt, device="cuda")  # noqa: E731
        ws = torch.zeros(ws_b, dtype=torch.uint8, device="cuda")
        ids, w, off, pairs = z(k), z(k, torch.float32), z(E + 1), z(k)
        act, na, slots, miss, nm = z(E), z(1), z(E), z(E), z(1)
        y = torch.full((1, H), 3.0, dtype=torch.float32, device="cuda")  # overwritten by the one-launch call
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        if fused:
            ops.moe_route_expert_ffn(xd, lg, 1, s.d, L, s.pool, E, tab, ids, w, off, pairs, act, na, slots, miss, nm,
                                     y, ws, ws_b, err)
        else:
            ops.moe_route_sort_lookup(lg, 1, s.d, L, tab, E, ids, w, off, pairs, act, na, slots, miss, nm, err)
            y.zero_()
            ops.moe_expert_ffn(xd, 1, s.d, s.pool, E, tab, ids, w, off, pairs, act, na, None, 0, E, y, ws, ws_b, err)
        torch.cuda.synchronize()
        n, m = int(na.item()), int(nm.item())
        out.append({"ids": ids.cpu().numpy(), "w": w.cpu().numpy(), "off": off.cpu().numpy(),
                    "pairs": pairs.cpu().numpy(), "n": n, "active": act.cpu().numpy()[:n],
                    "slots": slots.cpu().numpy()[:n], "m": m, "miss": miss.cpu().numpy()[:m],
                    "y": y.cpu().numpy(), "err": int(err.item())})
    return out


STAGES = ("ids", "w", "off", "pairs", "n", "active", "slots", "m", "miss")


@pytest.mark.parametrize("E,k,H,I,g,bg,bd", [
    (512, 10, 512, 256, 64, 3, 3),
    (64, 4, 256, 128, 32, 4, 4),
    (128, 8, 512, 128, 128, 3, 6),
    (1000, 8, 256, 128, 64, 4, 4),
])
def test_route_ffn_matches_stages_and_oracle(orc, E, k, H, I, g, bg, bd):
    s = Setup(orc, E, k, H, I, g, bg, bd, R=5, seed=E + k)
    for step in range(2):
        logits = synth.router_logits(7, 0, 1, E, step=step)
        x = synth.activations(7, 0, 1, H, step=step)
        f, sep = run_both(s, logits, x)
        for key in STAGES:
            assert np.array_equal(f[key], sep[key]), key
        ids, w, _ = orc.route(logits, k)
        assert np.array_equal(f["ids"], ids[0])
        assert f["err"] == 0 and f["m"] == 0
        assert_close(f["y"], s.oracle(orc, x, ids, w), TOL)
        assert_close(f["y"], sep["y"], TOL)


def test_route_ffn_substitution_and_missing_expert(orc):
    E, k, H, I, g = 128, 6, 256, 128, 64
    s = Setup(orc, E, k, H, I, g, 4, 4, R=5, seed=3)
    logits = synth.router_logits(9, 0, 1, E)
    x = synth.activations(9, 0, 1, H)
    table = s.perm.copy()
    table[np.argsort(-logits[0])[[0, 2]]] = -1  # two of the best experts have no slot
    L = 0.05
    f, sep = run_both(s, logits, x, L=L, table=dev(table))
    for key in STAGES:
        assert np.array_equal(f[key], sep[key]), key
    ids, w, _ = orc.route(logits, k, L, table)
    assert np.array_equal(f["ids"], ids[0])
    gone = np.isin(ids, np.nonzero(table < 0)[0])
    assert f["m"] == int(gone.sum())
    w2 = w.copy()
    w2[gone] = 0.0
    if gone.any():
        assert f["err"] & ops.DEV_ERR_NOT_RESIDENT
    assert_close(f["y"], s.oracle(orc, x, ids, w2), TOL)


def test_route_ffn_takes_one_token_only(orc):
    s = Setup(orc, 64, 4, 256, 128, 64, 4, 4, R=3, seed=1)
    T = 2
    ws_b = ops.moe_workspace_bytes(s.d, T)
    ws = torch.zeros(ws_b, dtype=torch.uint8, device="cuda")
    z = lambda *sh, dt=torch.int32: torch.zeros(sh, dtype=dt, device="cuda")  # noqa: E731
    with pytest.raises(ops.MoeError) as ei:
        ops.moe_route_expert_ffn(z(T, 256, dt=torch.int16), z(T, 64, dt=torch.float32), T, s.d, 0.0, s.pool, 64,
                                 s.table, z(T, 4), z(T, 4, dt=torch.float32), z(65), z(T * 4), z(64), z(1), z(64),
                                 z(64), z(1), z(T, 256, dt=torch.float32), ws, ws_b, z(1))
    assert ei.value.status == ops.MOE_ERR_UNSUPPORTED
