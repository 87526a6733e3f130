"""All five stages with installs, through the runtime over the C ABI, against
the oracle: decode with LRU misses installed from pinned host rows, decode
with cache-aware substitution over two size classes, a prefill chunk in
passes of 64 experts with installs between passes, and the mixed-class
prefill-then-decode sequence."""
import numpy as np
import pytest
import torch

from streamed_quantized_expert_b200 import build, ops, synth
from streamed_quantized_expert_b200.runtime import LayerSpec, Streamer
from tests._bank import assert_close, oracle_bank

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def make(orc, n_layers, E, k, H, I, g, bits, S, R, seed=0):
    """bits: per layer (b_gu, b_d).  Bank of R rows per size class, pinned."""
    banks, specs, host_slots = {}, [], []
    for l in range(n_layers):
        bg, bd = bits[l]
        if (bg, bd) not in banks:
            banks[(bg, bd)] = oracle_bank(orc, R, H, I, g, bg, bd, seed=seed + 100 * bg + bd)
        bank = banks[(bg, bd)]
        perm = synth.bank_permutation(seed, l, E) % R
        specs.append(LayerSpec(ops.desc(E, k, H, I, g, bg, bd), torch.from_numpy(bank).pin_memory(), perm.tolist()))
        host_slots.append([bank[perm[e]] for e in range(E)])
    return specs, host_slots


def initial_fill(st, seed, S):
    placed = []
    for l in range(st.n_layers):
        rank = synth.popularity_rank(seed, l, st.E)
        hot = np.argsort(rank)[:S]  # most popular experts first
        rel = synth.slot_permutation(seed, l, S)
        st.place(l, hot.tolist(), rel.tolist())
        placed.append((hot.astype(np.int32), rel.astype(np.int32) + st.cache.layer_base(l)))
    return placed


@pytest.mark.parametrize("meta_host", ["pinned", "pageable"])
def test_decode_with_installs(orc, meta_host):
    """pinned: the one-token routing kernel writes the active list to the
    host buffer and the driver waits for its sequence word; pageable (memory
    the device cannot address): the driver copies the list back and
    synchronises instead."""
    E, k, H, I, g, S = 512, 10, 2048, 512, 64, 192
    specs, host_slots = make(orc, 2, E, k, H, I, g, [(3, 3), (3, 3)], S, R=12)
    st = Streamer(specs, S, max_tokens=1)
    if meta_host == "pageable":
        st.meta_pin = torch.zeros(st.meta_pin.numel(), dtype=torch.int32)
        st._bufs.meta_host = st.meta_pin.data_ptr()
    placed = initial_fill(st, 0, S)
    models = []
    for l in range(2):
        m = orc.LruModel(E, S, slot_base=st.cache.layer_base(l))
        m.place(*placed[l])
        models.append(m)
    total_inst = 0
    for step in range(6):
        for l in range(2):
            x = synth.activations(0, l, 1, H, step=step)
            logits = synth.router_logits(0, l, 1, E, step=step)
            y = st.decode_layer(l, dev(x.view(np.int16)), dev(logits), 1)
            got = y.cpu().numpy()
            ids, w, _ = orc.route(logits, k)
            assert np.array_equal(st.ids[:1].cpu().numpy(), ids)
            assert_close(got, orc.expert_ffn(x, H, I, g, 3, 3, ids, w, host_slots[l]), TOL)
            total_inst += len([e for e in sorted(ids[0]) if models[l].table[e] < 0])
            models[l].step(np.sort(ids[0]).astype(np.int32))
            assert np.array_equal(st.table_dev[l].cpu().numpy(), models[l].table)
    assert st.check_dev_err() == 0
    assert total_inst > 0 and st.installs == total_inst


def test_substitution_two_size_classes(orc):
    # 4-bit gate/up; 6-bit down on every 4th layer (l % 4 == 0); 25% resident; L = 0.15
    E, k, H, I, g, S, L = 512, 10, 2048, 512, 64, 128, 0.15
    bits = [(4, 6), (4, 4)]
    specs, host_slots = make(orc, 2, E, k, H, I, g, bits, S, R=8, seed=5)
    st = Streamer(specs, S, max_tokens=1)
    assert len(st.pools) == 2
    initial_fill(st, 5, S)
    for step in range(4):
        for l in range(2):
            x = synth.activations(5, l, 1, H, step=step)
            logits = synth.router_logits(5, l, 1, E, step=step)
            table_before = st.table_dev[l].cpu().numpy()
            y = st.decode_layer(l, dev(x.view(np.int16)), dev(logits), 1, L=L)
            ids, w, _ = orc.route(logits, k, L, table_before)
            assert np.array_equal(st.ids[:1].cpu().numpy(), ids)
            assert np.max(np.abs(st.w[:1].cpu().numpy() - w)) <= 1e-5
            assert_close(y.cpu().numpy(), orc.expert_ffn(x, H, I, g, *bits[l], ids, w, host_slots[l]), TOL)
    assert st.check_dev_err() == 0


def test_prefill_passes_with_installs(orc):
    E, k, H, I, g, S, T = 512, 10, 2048, 512, 64, 128, 256
    specs, host_slots = make(orc, 1, E, k, H, I, g, [(3, 3)], S, R=8, seed=9)
    st = Streamer(specs, S, max_tokens=T)
    initial_fill(st, 9, S)
    x = synth.activations(9, 0, T, H)
    logits = synth.router_logits(9, 0, T, E)
    y = st.prefill_layer(0, dev(x.view(np.int16)), dev(logits), T)
    ids, w, _ = orc.route(logits, k)
    assert np.array_equal(st.ids[:T].cpu().numpy(), ids)
    assert st.installs > 0
    tok = np.array([0, 7, 100, T - 1])
    assert_close(y.cpu().numpy()[tok], orc.expert_ffn(x, H, I, g, 3, 3, ids, w, host_slots[0], tok), TOL)
    assert st.check_dev_err() == 0


def test_prefill_then_decode_sequence_two_classes(orc):
    # the mixed-class sequence at reduced size: a prefill chunk through a 25%-resident two-class cache
    # (passes of 64 experts, installs between passes), then decode steps with cache-aware substitution
    # (L = 0.15) from the cache the prefill left; every layer's y, routing and slot table against the oracle
    E, k, H, I, g, S, T, L = 256, 4, 256, 128, 64, 64, 96, 0.15  # a pass of 64 experts needs 64 slots
    bits = [(4, 6), (4, 4)]
    specs, host_slots = make(orc, 2, E, k, H, I, g, bits, S, R=7, seed=13)
    st = Streamer(specs, S, max_tokens=T)
    placed = initial_fill(st, 13, S)
    models = []
    for l in range(2):
        m = orc.LruModel(E, S, slot_base=st.cache.layer_base(l))
        m.place(*placed[l])
        models.append(m)
    for l in range(2):
        x = synth.activations(13, l, T, H)
        logits = synth.router_logits(13, l, T, E)
        y = st.prefill_layer(l, dev(x.view(np.int16)), dev(logits), T)
        ids, w, _ = orc.route(logits, k)
        assert np.array_equal(st.ids[:T].cpu().numpy(), ids)
        active = np.unique(ids).astype(np.int32)
        assert active.size > 64  # at least two passes
        for p in range(0, active.size, 64):
            models[l].step(active[p:p + 64])
        assert np.array_equal(st.table_dev[l].cpu().numpy(), models[l].table)
        assert_close(y.cpu().numpy(), orc.expert_ffn(x, H, I, g, *bits[l], ids, w, host_slots[l]), TOL)
    inst_prefill = st.installs
    assert inst_prefill > 0
    for step in range(6):
        for l in range(2):
            x = synth.activations(13, l, 1, H, step=step + 1)
            logits = synth.router_logits(13, l, 1, E, step=step + 1)
            table_before = st.table_dev[l].cpu().numpy()
            assert np.array_equal(table_before, models[l].table)
            y = st.decode_layer(l, dev(x.view(np.int16)), dev(logits), 1, L=L)
            ids, w, _ = orc.route(logits, k, L, table_before)
            assert np.array_equal(st.ids[:1].cpu().numpy(), ids)
            models[l].step(np.sort(ids[0]).astype(np.int32))
            assert_close(y.cpu().numpy(), orc.expert_ffn(x, H, I, g, *bits[l], ids, w, host_slots[l]), TOL)
    assert st.check_dev_err() == 0
