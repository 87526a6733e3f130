"""Pins for stage 1 (route_topk with cache-aware substitution).

BigMoeOnEdge commit note on cache-aware substitution: resident experts get
their score raised by L times the token's score range, the top-k is taken
again, and the same number of experts runs.
"""
import numpy as np
import pytest

from streamed_quantized_expert_b200 import synth


def _full_sort_topk(orc, l, k, L, resident):
    """Brute force: sort all E keys (u' desc, l desc, e asc), take k."""
    u = orc.exp_portable(l - l.max())
    up = u.copy()
    if L > 0:
        boost = np.float32(L) * (np.float32(1.0) - u.min())
        up = np.where(resident, u + boost, u).astype(np.float32)
    order = sorted(range(l.size), key=lambda e: (-float(up[e]), -float(l[e]), e))
    return np.array(order[:k], np.int32)


@pytest.mark.parametrize("E,k,T", [(8, 2, 40), (128, 8, 20), (512, 10, 8), (16, 16, 5), (4, 1, 10)])
@pytest.mark.parametrize("L", [0.0, 0.15, 0.6])
def test_selection_vs_full_sort(orc, E, k, T, L):
    logits = synth.router_logits(3, E + k, T, E)
    table = np.where(synth.rng(5, E).random(E) < 0.3, np.arange(E), -1).astype(np.int32)
    ids, w, _ = orc.route(logits, k, L, table)
    for t in range(T):
        ref = _full_sort_topk(orc, logits[t], k, L, table >= 0)
        assert np.array_equal(ids[t], ref)


def test_L0_is_plain_logit_order(orc):
    # closed form at L = 0: u is non-decreasing in l, so the key reduces to (l desc, e asc)
    logits = synth.router_logits(11, 0, 64, 512)
    logits[3, 10:20] = logits[3, 5]  # exact ties -> lower id first
    ids, _, _ = orc.route(logits, 10, 0.0, None)
    for t in range(64):
        ref = np.lexsort((np.arange(512), -logits[t].astype(np.float64)))[:10]
        assert np.array_equal(ids[t], ref)


def test_weights_are_renormalised_softmax(orc):
    logits = synth.router_logits(2, 1, 50, 128)
    ids, w, _ = orc.route(logits, 8, 0.0, None)
    p = np.exp(logits.astype(np.float64) - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ref = np.take_along_axis(p, ids, axis=1)
    ref /= ref.sum(axis=1, keepdims=True)
    assert np.allclose(w, ref, rtol=1e-6, atol=0)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-12)


def test_boost_on_u_selects_as_boost_on_softmax(orc):
    # reading: selecting on u + L(1 - min u) equals selecting on the boosted
    # normalised softmax s + L(max s - min s); checked in float64 on inputs
    # whose keys are well separated
    r = np.random.default_rng(7)
    for _ in range(50):
        E, k, L = 64, 6, 0.15
        l = np.sort(r.choice(np.arange(-400, 400), E, replace=False))[::-1].astype(np.float32) / np.float32(100)
        r.shuffle(l)
        res = r.random(E) < 0.4
        s = np.exp(l.astype(np.float64) - l.max())
        s /= s.sum()
        sp = s + L * (s.max() - s.min()) * res
        ref = np.argsort(-sp, kind="stable")[:k]
        srt = np.sort(sp)[::-1]
        if np.min(np.abs(np.diff(srt[: k + 1]))) < 1e-6:
            continue
        ids, _, _ = orc.route(l[None, :], k, L, np.where(res, 0, -1).astype(np.int32))
        assert set(ids[0].tolist()) == set(ref.tolist())


def test_noop_when_none_or_all_resident(orc):
    logits = synth.router_logits(4, 2, 32, 512)
    base, wb, _ = orc.route(logits, 10, 0.0, None)
    for table in (np.full(512, -1, np.int32), np.arange(512, dtype=np.int32)):
        ids, w, _ = orc.route(logits, 10, 0.15, table)
        assert np.array_equal(ids, base)
        assert np.array_equal(w, wb)


def test_substitution_monotone_in_resident_count(orc):
    logits = synth.router_logits(8, 3, 200, 512)
    table = np.where(synth.rng(9).random(512) < 0.25, 1, -1).astype(np.int32)
    base, _, _ = orc.route(logits, 10, 0.0, table)
    sub, _, _ = orc.route(logits, 10, 0.15, table)
    assert np.all((table[sub] >= 0).sum(1) >= (table[base] >= 0).sum(1))
    assert (table[sub] >= 0).sum() > (table[base] >= 0).sum()  # it does act
    assert sub.shape == base.shape  # the same number of experts runs


def test_large_L_picks_only_resident(orc):
    # closed form: for L > 1 every boosted resident score exceeds 1 >= any unboosted one
    logits = synth.router_logits(10, 4, 50, 128)
    table = np.where(synth.rng(12).random(128) < 0.2, 0, -1).astype(np.int32)
    assert (table >= 0).sum() >= 8
    ids, _, _ = orc.route(logits, 8, 2.0, table)
    assert np.all(table[ids] >= 0)


def test_golden_substitution_example(orc):
    # Worked by hand (tests/golden/route_example.txt)
    rows = [l.split() for l in open(__file__.replace("test_oracle_route.py", "golden/route_example.txt"))
            if l.strip() and not l.startswith("#")]
    d = {r[0]: r[1:] for r in rows}
    logits = np.array([d["logits"]], np.float32).astype(np.float32)
    table = np.array(d["table"], np.int32)
    for key, L in (("L0", 0.0), ("L015", 0.15)):
        ids, w, _ = orc.route(logits, 2, L, table)
        assert ids[0].tolist() == [int(v) for v in d[f"ids_{key}"]]
        assert np.allclose(w[0], [float(v) for v in d[f"w_{key}"]], atol=1e-4)
