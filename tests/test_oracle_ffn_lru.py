"""Pins for stages 4-5 (SwiGLU expert FFN + weighted combine) and the host
slot-cache model.

The RFC: experts are "gated, concatenated, untransposed, no bias" (SwiGLU,
gate rows then up rows, stored [out, in]).  1bit-MONSTER PR #137: one LRU per
class (per layer with --per-layer), empty slots taken first.
"""
import numpy as np
import pytest

from streamed_quantized_expert_b200 import synth
from tests import _format_np as F


def _bank(orc, E, H, I, g, b_gu, b_d, seed=0):
    slots, dense = [], []
    off, n = orc.slot_layout(H, I, g, b_gu, b_d)
    for e in range(E):
        w_gu, w_d = synth.expert_weights(seed, e, H, I)
        s = orc.build_slot(w_gu, w_d, g, b_gu, b_d)
        slots.append(s)
        # dequantise with the independent numpy decoder
        pg = s[off[0]: off[0] + 2 * I // 16 * off[2]]
        pd = s[off[1]: off[1] + H // 16 * off[3]]
        gu_stored = F.dequant_rows(pg, 2 * I, H, g, b_gu)
        gu_logical = gu_stored[[F.gate_up_storage_row(R, I) for R in range(2 * I)]]
        dense.append((gu_logical.astype(np.float64),
                      F.dequant_rows(pd, H, I, g, b_d).astype(np.float64)))
    return slots, dense


def _dense_moe(x, dense, ids, w, I):
    """Textbook dense MoE: every expert's SwiGLU MLP on every token, combined
    with a [T, E] weight matrix that is zero outside each token's top-k."""
    T = x.shape[0]
    E = len(dense)
    M = np.zeros((T, E))
    for t in range(T):
        for j in range(ids.shape[1]):
            M[t, ids[t, j]] += w[t, j]
    Wgu = np.stack([d[0] for d in dense])  # [E, 2I, H]
    Wd = np.stack([d[1] for d in dense])   # [E, H, I]
    gu = np.einsum("eoh,th->teo", Wgu, x)
    gate, up = gu[..., :I], gu[..., I:]
    h = gate / (1.0 + np.exp(-gate)) * up
    o = np.einsum("ehi,tei->teh", Wd, h)
    return np.einsum("te,teh->th", M, o)


@pytest.mark.parametrize("b_gu,b_d", [(4, 4), (3, 3), (4, 6), (16, 16), (16, 4)])
def test_ffn_vs_dense_moe(orc, b_gu, b_d):
    E, k, H, I, g, T = 8, 2, 64, 32, 32, 4
    slots, dense = _bank(orc, E, H, I, g, b_gu, b_d)
    x = synth.activations(0, 0, T, H)
    logits = synth.router_logits(0, 0, T, E, beta=0.0)
    ids, w, _ = orc.route(logits, k)
    y = orc.expert_ffn(x, H, I, g, b_gu, b_d, ids, w, slots)
    ref = _dense_moe(synth.bf16_bits_to_f32(x).astype(np.float64), dense, ids, w, I)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)


def test_single_expert_is_plain_mlp(orc):
    E, H, I, g = 4, 128, 64, 64
    slots, dense = _bank(orc, E, H, I, g, 4, 4, seed=5)
    x = synth.activations(1, 0, 3, H)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ids = np.array([[2], [0], [3]], np.int32)
    y = orc.expert_ffn(x, H, I, g, 4, 4, ids, np.ones((3, 1)), slots)
    for t in range(3):
        Wgu, Wd = dense[ids[t, 0]]
        a, u = Wgu[:I] @ xf[t], Wgu[I:] @ xf[t]
        ref = Wd @ (a * u / (1.0 + np.exp(-a)))
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("n_shared,gated", [(1, False), (2, True)])
def test_shared_experts_vs_textbook_moe(orc, n_shared, gated):
    # textbook MoE with always-on shared experts: y_t = sum_j w_tj E_j(x_t) +
    # sum_s g_t S_s(x_t), every expert a dense SwiGLU MLP from the numpy decoder
    E, k, H, I, g, T = 8, 2, 64, 32, 32, 5
    slots, dense = _bank(orc, E + n_shared, H, I, g, 4, 4, seed=3)
    x = synth.activations(4, 0, T, H)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    logits = synth.router_logits(4, 0, T, E, beta=0.0)
    gate = synth.rng(9, T).uniform(0.2, 1.0, T).astype(np.float32) if gated else None
    ids, w, _ = orc.route_shared(logits, k, n_shared, gate)
    r_ids, r_w, _ = orc.route(logits, k)
    assert np.array_equal(ids[:, :k], r_ids) and np.array_equal(w[:, :k], r_w)
    assert np.all(ids[:, k:] == np.arange(E, E + n_shared))
    y = orc.expert_ffn(x, H, I, g, 4, 4, ids, w, slots)
    ref = _dense_moe(xf, dense[:E], r_ids, r_w, I)
    for s in range(n_shared):
        Wgu, Wd = dense[E + s]
        for t in range(T):
            a, u = Wgu[:I] @ xf[t], Wgu[I:] @ xf[t]
            ref[t] += (float(gate[t]) if gated else 1.0) * (Wd @ (a * u / (1.0 + np.exp(-a))))
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)


def test_zero_input_gives_zero_output(orc):
    slots, _ = _bank(orc, 2, 64, 32, 32, 3, 3)
    x = np.zeros((2, 64), np.uint16)
    ids = np.array([[0, 1], [1, 0]], np.int32)
    y = orc.expert_ffn(x, 64, 32, 32, 3, 3, ids, np.full((2, 2), 0.5), slots)
    assert np.all(y == 0.0)


def test_token_subset_matches_full(orc):
    slots, _ = _bank(orc, 8, 64, 32, 32, 4, 4)
    x = synth.activations(2, 0, 6, 64)
    ids, w = synth.random_routing(2, 6, 8, 2)
    full = orc.expert_ffn(x, 64, 32, 32, 4, 4, ids, w.astype(np.float64), slots)
    sub = orc.expert_ffn(x, 64, 32, 32, 4, 4, ids, w.astype(np.float64), slots, tokens=[4, 1])
    assert np.array_equal(sub, full[[4, 1]])


class NaiveLru:
    """Recency list, least recent first; empty slots start at the front."""

    def __init__(self, n_slots, placed):
        self.order = [s for s in range(n_slots) if s not in dict(placed).values()] + [s for _, s in placed]
        self.owner = {s: e for e, s in placed}

    def step(self, experts):
        where = {e: s for s, e in self.owner.items()}
        used = {where[e] for e in experts if e in where}
        for e in experts:
            if e in where:
                self.order.remove(where[e])
                self.order.append(where[e])
        out = []
        for e in experts:
            if e in where:
                continue
            cand = [s for s in self.order if s not in used]
            if not cand:
                out.append(-1)
                continue
            s = cand[0]
            self.owner[s] = e
            used.add(s)
            self.order.remove(s)
            self.order.append(s)
            out.append(s)
        return out


@pytest.mark.parametrize("n_slots,E,npass", [(16, 64, 6), (8, 20, 8), (4, 10, 6)])
def test_lru_vs_naive(orc, n_slots, E, npass):
    r = np.random.default_rng(n_slots)
    placed = [(int(e), i) for i, e in enumerate(r.choice(E, n_slots // 2, replace=False))]
    m = orc.LruModel(E, n_slots)
    m.place([e for e, _ in placed], [s for _, s in placed])
    naive = NaiveLru(n_slots, placed)
    for _ in range(200):
        experts = np.sort(r.choice(E, npass, replace=False)).astype(np.int32)
        got, fail = m.step(experts)
        ref = naive.step(experts.tolist())
        assert got.tolist() == ref
        assert fail == ref.count(-1)
        for s, e in naive.owner.items():
            assert m.table[e] == s


def test_lru_empty_slots_first(orc):
    m = orc.LruModel(10, 4)
    m.place([7, 8], [2, 3])
    got, _ = m.step(np.array([1, 2], np.int32))
    assert got.tolist() == [0, 1]
    got, _ = m.step(np.array([3], np.int32))
    assert got.tolist() == [2]  # now the least recent occupied slot (expert 7's)
    assert m.table[7] == -1 and m.table[3] == 2
