"""Pins for stage 2 (moe_sort: tokens grouped by expert, passes of 64 active
experts; transformers PR #50717 notes and the RFC's "Prefill") and stage 3
(expert -> slot lookup with a miss list; RFC "How the prototype works")."""
import numpy as np
import pytest

from streamed_quantized_expert_b200 import synth


@pytest.mark.parametrize("T,E,k", [(0, 8, 2), (1, 512, 10), (4, 8, 2), (64, 128, 8), (1024, 512, 10), (37, 16, 16)])
def test_sort_vs_brute_force(orc, T, E, k):
    ids, _ = synth.random_routing(T + 1, T, E, k)
    offsets, pairs, active = orc.sort(ids, E)
    flat = ids.reshape(-1)
    ref = sorted(range(T * k), key=lambda i: (int(flat[i]), i))
    assert pairs.tolist() == ref
    hist = np.bincount(flat, minlength=E) if T else np.zeros(E, np.int64)
    assert offsets.tolist() == [0] + np.cumsum(hist).tolist()
    assert active.tolist() == [e for e in range(E) if hist[e] > 0]
    assert sorted(pairs.tolist()) == list(range(T * k))  # a permutation


def test_sort_all_to_one_expert(orc):
    ids = np.full((50, 1), 7, np.int32)
    offsets, pairs, active = orc.sort(ids, 16)
    assert active.tolist() == [7]
    assert offsets[7] == 0 and offsets[8] == 50 and offsets[16] == 50
    assert pairs.tolist() == list(range(50))


def test_lookup_vs_brute_force(orc):
    E, n_slots = 512, 192
    r = synth.rng(21)
    table = np.full(E, -1, np.int32)
    res = r.choice(E, n_slots, replace=False)
    table[res] = r.permutation(n_slots)
    active = np.sort(r.choice(E, 300, replace=False)).astype(np.int32)
    for pb, pl in [(0, 64), (64, 64), (256, 64), (290, 64), (0, 512), (300, 10)]:
        slots, miss, bad = orc.slot_lookup(table, active, pb, pl, n_slots)
        seg = active[pb: pb + pl]
        assert slots.tolist() == table[seg].tolist()
        assert miss.tolist() == [int(e) for e in seg if table[e] < 0]
        assert bad == 0


def test_lookup_flags_out_of_range_slot(orc):
    table = np.array([0, 5, -1, 2], np.int32)
    slots, miss, bad = orc.slot_lookup(table, np.array([0, 1, 2], np.int32), 0, 64, 4)
    assert bad == 1 and miss.tolist() == [2] and slots.tolist() == [0, 5, -1]
