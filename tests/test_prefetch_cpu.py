"""Guessed prefetch on the host (RFC "How the prototype works", item "Reads":
the next two layers' experts are guessed by running their routers on the
current hidden states and read in the background; PR #50717 commit note:
guessed reads still in flight are skipped, not waited for):

  * the oracle's router projection against closed forms;
  * moe_cache_reserve / moe_cache_commit against a hand-worked scenario and
    against a naive model under random use: reserved slots are never
    victims, guesses stay out of the table until committed, a commit either
    enters the guess or frees the slot."""
import numpy as np
import pytest

from streamed_quantized_expert_b200 import ops, synth


def test_router_logits_closed_forms(orc):
    T, E, H = 3, 5, 64
    x = synth.activations(3, 0, T, H)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    # unit rows: row e picks input h_e
    pick = np.array([0, 7, 63, 7, 31])
    W = np.zeros((E, H), np.uint16)
    W[np.arange(E), pick] = 0x3F80  # bf16 1.0
    bias = np.array([0.5, -1.0, 0.0, 2.0, 0.25], np.float32)
    got = orc.router_logits(x, W, bias, 0.25)
    assert np.array_equal(got, 0.25 * xf[:, pick] + bias[None, :].astype(np.float64))
    # a row equal to a token's own state gives its squared norm; negating the row negates the logit
    W2 = np.stack([x[1], x[1] ^ 0x8000])
    got2 = orc.router_logits(x[1:2], W2, None, 1.0)
    assert np.isclose(got2[0, 0], float(xf[1] @ xf[1]), rtol=1e-15) and got2[0, 1] == -got2[0, 0]


def test_hidden_stream_correlation():
    xs = synth.bf16_bits_to_f32(synth.hidden_stream(5, 4, 64, 512)).astype(np.float64)
    for l in range(3):
        a, b = xs[l].ravel(), xs[l + 1].ravel()
        r = a @ b / np.sqrt((a @ a) * (b @ b))
        assert abs(r - 1 / np.sqrt(1.25)) < 0.02  # sigma = 0.5
        assert abs(np.std(xs[l + 1]) - 1.0) < 0.02


def _cache(E=16, S=4, placed=((3, 0), (5, 1))):
    c = ops.SlotCache(E, 2, S)
    c.place(1, [e for e, _ in placed], [c.layer_base(1) + s for _, s in placed])
    return c


def test_reserve_commit_scenario(orc):
    c = _cache()
    base = c.layer_base(1)
    # slots 2 and 3 are empty: taken first; resident experts 3, 5 and a repeat are skipped
    got = c.reserve(1, [3, 9, 9, 11, 5])
    assert got == [(9, base + 2), (11, base + 3)]
    tab = list(c.table(1))
    assert tab[9] == -1 and tab[11] == -1  # not entered yet
    assert c.reserve(1, [9]) == []  # already in flight
    # the next guess takes the least recently used resident slot (expert 3's), evicting it
    assert c.reserve(1, [12]) == [(12, base + 0)]
    assert c.table(1)[3] == -1
    # a step never takes a reserved slot: only slot 1 (expert 5) is free to evict
    st, inst = c.step(1, [7])
    assert st == ops.MOE_OK and inst == [(7, base + 1)]
    st, inst = c.step(1, [7, 8])
    assert st == ops.MOE_ERR_CAPACITY  # every other slot has a copy in flight
    # commits: 9 enters; 12 was installed normally meanwhile -> its reserved slot frees
    assert c.commit(1, base + 2) is True and c.table(1)[9] == base + 2
    c2 = _cache()
    b2 = c2.layer_base(1)
    c2.reserve(1, [12])
    c2.step(1, [12])
    slot12 = c2.table(1)[12]
    assert slot12 >= 0
    assert c2.commit(1, b2 + 2) is False and c2.table(1)[12] == slot12
    with pytest.raises(ops.MoeError):
        c2.commit(1, b2 + 2)  # no reservation any more


class Naive:
    """Recency list per slot plus reservations, the rules written out."""

    def __init__(self, S):
        self.owner = [-1] * S
        self.pend = [-1] * S
        self.stamp = [0] * S
        self.clock = 0

    def table(self, e):
        return self.owner.index(e) if e in self.owner else -1

    def free_lru(self, exclude):
        cand = [s for s in range(len(self.owner)) if self.pend[s] < 0 and s not in exclude]
        return min(cand, key=lambda s: self.stamp[s]) if cand else -1

    def step(self, experts):
        used = {s for s in range(len(self.owner)) if self.pend[s] >= 0}
        for e in experts:
            if self.table(e) >= 0:
                s = self.table(e)
                used.add(s)
                self.clock += 1
                self.stamp[s] = self.clock
        out = []
        for e in experts:
            if self.table(e) >= 0:
                continue
            cand = [s for s in range(len(self.owner)) if s not in used]
            if not cand:
                out.append((e, -1))
                continue
            s = min(cand, key=lambda s: self.stamp[s])
            self.owner[s] = e
            used.add(s)
            self.clock += 1
            self.stamp[s] = self.clock
            out.append((e, s))
        return out

    def reserve(self, experts):
        out = []
        for e in experts:
            if self.table(e) >= 0 or e in self.pend:
                continue
            s = self.free_lru(set())
            if s < 0:
                break
            self.owner[s] = -1
            self.pend[s] = e
            self.clock += 1
            self.stamp[s] = self.clock
            out.append((e, s))
        return out

    def commit(self, s):
        e, self.pend[s] = self.pend[s], -1
        if self.table(e) < 0:
            self.owner[s] = e
            self.clock += 1
            self.stamp[s] = self.clock
            return True
        self.stamp[s] = 0
        return False


def test_reserve_commit_vs_naive(orc):
    E, S = 40, 8
    c = ops.SlotCache(E, 1, S)
    m = Naive(S)
    r = synth.rng(21)
    for it in range(400):
        op = r.integers(0, 3)
        if op == 0:
            ex = sorted(set(r.integers(0, E, 3).tolist()))
            st, inst = c.step(0, ex)
            ref = m.step(ex)
            assert [(e, s) for e, s in inst] == ref
        elif op == 1:
            ex = r.integers(0, E, 3).tolist()
            assert c.reserve(0, ex) == m.reserve(ex)
        else:
            pend = [s for s in range(S) if m.pend[s] >= 0]
            if pend:
                s = int(r.choice(pend))
                assert c.commit(0, s) == m.commit(s)
        tab = list(c.table(0))
        assert tab == [m.table(e) for e in range(E)]
