"""Always-on shared experts (BigMoeOnEdge docs/limitations.md, "Limitations",
bullet "Shared experts stay resident"), through the C ABI, against the
oracle: moe_route_shared appends the shared experts to every token's top-k,
and the widened layer (E + n_shared experts, k + n_shared per token) runs the
shared experts in the same moe_expert_ffn launch as the routed ones, on each
kernel path."""
import numpy as np
import pytest
import torch

from streamed_quantized_expert_b200 import ops, synth
from tests._bank import assert_close
from tests.test_gpu_ffn import TOL, Setup, dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,E,k,ns,gated,L", [(1, 512, 10, 1, False, 0.0), (1, 512, 10, 2, True, 0.15),
                                              (5, 128, 8, 1, True, 0.0), (300, 512, 10, 1, False, 0.0),
                                              (64, 64, 4, 8, True, 0.0)])
def test_route_shared(orc, T, E, k, ns, gated, L):
    logits = synth.router_logits(T + 3, 1, T, E)
    table = np.where(synth.rng(E, 2).random(E) < 0.25, np.arange(E), -1).astype(np.int32)
    gate = synth.rng(T, 5).uniform(0.1, 1.0, T).astype(np.float32) if gated else None
    ids_ref, w_ref, _ = orc.route_shared(logits, k, ns, gate, L, table)
    ids = torch.full((T, k + ns), -7, dtype=torch.int32, device="cuda")
    w = torch.zeros((T, k + ns), dtype=torch.float32, device="cuda")
    ops.moe_route_shared(dev(logits), T, ops.desc(E, k, 64, 32, 32, 4), L, dev(table), ns,
                         dev(gate) if gated else None, ids, w)
    torch.cuda.synchronize()
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    got = w.cpu().numpy()
    assert np.max(np.abs(got[:, :k] - w_ref[:, :k])) <= 1e-5
    assert np.array_equal(got[:, k:].astype(np.float64), w_ref[:, k:])  # the gate (or 1), exactly


def test_route_shared_rejects_too_many(orc):
    d = ops.desc(64, 4, 64, 32, 32, 4)
    x = torch.zeros((1, 64), dtype=torch.float32, device="cuda")
    ids = torch.zeros((1, 13), dtype=torch.int32, device="cuda")
    w = torch.zeros((1, 13), dtype=torch.float32, device="cuda")
    with pytest.raises(ops.MoeError):
        ops.moe_route_shared(x, 1, d, 0.0, None, 9, None, ids, w)


@pytest.mark.parametrize("T,ns,gated,sorted_x", [(1, 1, False, False), (4, 2, True, False), (16, 1, True, False),
                                                 (40, 1, False, True), (64, 2, True, True)])
def test_shared_experts_in_the_ffn_launch(orc, T, ns, gated, sorted_x):
    E, k, H, I, g = 60, 4, 512, 256, 64
    s = Setup(orc, E + ns, k + ns, H, I, g, 4, 4, R=7, seed=41)  # widened layer: experts E.. are shared
    want = (ops.MOE_PATH_FUSED_DECODE if T <= 8 else ops.MOE_PATH_TC_PREFILL if sorted_x else ops.MOE_PATH_GEMV)
    assert ops.moe_ffn_kernel_path(s.d, T, sorted_x) == want
    logits = synth.router_logits(41, 0, T, E)
    gate = synth.rng(T, 6).uniform(0.1, 1.0, T).astype(np.float32) if gated else None
    ids_d = torch.empty((T, k + ns), dtype=torch.int32, device="cuda")
    w_d = torch.empty((T, k + ns), dtype=torch.float32, device="cuda")
    ops.moe_route_shared(dev(logits), T, ops.desc(E, k, H, I, g, 4, 4), 0.0, None, ns, dev(gate) if gated else None,
                         ids_d, w_d)
    torch.cuda.synchronize()
    ids, w = ids_d.cpu().numpy(), w_d.cpu().numpy()
    ids_ref, w_ref, _ = orc.route_shared(logits, k, ns, gate)
    assert np.array_equal(ids, ids_ref)
    x = synth.activations(41, 0, T, H)
    y, err = s.gpu(x, ids, w, T, sorted_x=sorted_x)
    assert err == 0
    assert_close(y, s.oracle(orc, x, ids, w), TOL)
    # the shared experts' share is real: without them the result differs
    w0 = w.copy()
    w0[:, k:] = 0.0
    assert not np.allclose(y, s.oracle(orc, x, ids, w0), rtol=0.1, atol=0.0)


def test_streamer_decode_and_prefill_with_shared_expert(orc):
    # a 25%-resident routed cache with installs, plus one shared expert per layer in
    # pinned slots: every layer's y against the oracle over the widened routing
    from streamed_quantized_expert_b200.runtime import LayerSpec, Streamer
    from tests._bank import oracle_bank
    from tests.test_gpu_pipeline import initial_fill

    E, k, H, I, g, S, T, ns = 256, 4, 256, 128, 64, 64, 80, 1
    bank = oracle_bank(orc, 9, H, I, g, 4, 4, seed=77)
    specs, host_slots = [], []
    for l in range(2):
        perm = synth.bank_permutation(77, l, E) % 8  # rows 0..7 routed, row 8 the shared expert
        shared = torch.from_numpy(bank[8:9].copy())
        specs.append(LayerSpec(ops.desc(E, k, H, I, g, 4, 4), torch.from_numpy(bank).pin_memory(), perm.tolist(),
                               shared))
        host_slots.append([bank[perm[e]] for e in range(E)] + [bank[8]])
    st = Streamer(specs, S, max_tokens=T, n_shared=ns)
    initial_fill(st, 77, S)
    for l in range(2):
        x = synth.activations(77, l, T, H)
        logits = synth.router_logits(77, l, T, E)
        y = st.prefill_layer(l, dev(x.view(np.int16)), dev(logits), T)
        ids, w, _ = orc.route_shared(logits, k, ns)
        assert np.array_equal(st.ids[:T].cpu().numpy(), ids)
        assert_close(y.cpu().numpy(), orc.expert_ffn(x, H, I, g, 4, 4, ids, w, host_slots[l]), TOL)
    for step in range(4):
        for l in range(2):
            x = synth.activations(77, l, 1, H, step=step + 1)
            logits = synth.router_logits(77, l, 1, E, step=step + 1)
            table_before = st.table_dev[l, :E].cpu().numpy()
            y = st.decode_layer(l, dev(x.view(np.int16)), dev(logits), 1, L=0.15)
            ids, w, _ = orc.route_shared(logits, k, ns, None, 0.15, table_before)
            assert np.array_equal(st.ids[:1].cpu().numpy(), ids)
            assert_close(y.cpu().numpy(), orc.expert_ffn(x, H, I, g, 4, 4, ids, w, host_slots[l]), TOL)
            assert int(st.table_dev[l, E]) >= st.cache.class_slots(0)  # the shared slot never moves
    assert st.installs > 0
    assert st.check_dev_err() == 0
