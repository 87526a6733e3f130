"""The C-ABI library loads, exports every symbol include/moe.h declares, and
its host-only parts (sizes, argument checks, slot cache) behave -- no GPU."""
import os
import re

import numpy as np
import pytest

from streamed_quantized_expert_b200 import build, ops, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert len(declared) >= 18
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(ops.ABI_SYMBOLS) == declared


def test_sizes_match_oracle(lib, orc):
    for (E, k, H, I, g, bg, bd) in [(8, 2, 64, 32, 32, 4, 4), (512, 10, 2048, 512, 64, 3, 3),
                                     (128, 8, 2048, 768, 64, 4, 4), (512, 10, 2048, 512, 64, 4, 6)]:
        d = ops.desc(E, k, H, I, g, bg, bd)
        off, n = orc.slot_layout(H, I, g, bg, bd)
        lay = ops.moe_slot_layout(d)
        assert ops.moe_slot_bytes(d) == n == lay.slot_bytes
        assert [lay.gate_up, lay.down, lay.gate_up_tile_bytes, lay.down_tile_bytes] == off


def test_argument_checks(lib):
    bad = [ops.desc(8, 9, 64, 32, 32, 4), ops.desc(8, 2, 64, 32, 48, 4), ops.desc(8, 2, 64, 32, 32, 5),
           ops.desc(8, 2, 65, 32, 32, 4), ops.desc(2048, 2, 64, 32, 32, 4)]
    for d in bad:
        assert ops.moe_slot_bytes(d) == 0
        assert ops.moe_workspace_bytes(d, 4) == 0
    d = ops.desc(8, 2, 64, 32, 32, 4)
    with pytest.raises(ops.MoeError) as ei:
        ops.moe_route(None, 4, d, 0.0, None, None, None)
    assert ei.value.status == ops.MOE_ERR_INVALID
    with pytest.raises(ops.MoeError) as ei:
        ops.moe_route(1 << 20, 4, d, 0.5, None, 1 << 21, 1 << 22)  # L > 0 needs a slot table
    assert ei.value.status == ops.MOE_ERR_INVALID
    with pytest.raises(ops.MoeError) as ei:
        ops.moe_install_slots(1 << 20, 256, 4, [1 << 21], [4])  # slot id past the pool
    assert ei.value.status == ops.MOE_ERR_INVALID
    with pytest.raises(ops.MoeError) as ei:
        ops.moe_quantize_rows(1 << 20, 16, 64, 32, 5, 1 << 21)
    assert ei.value.status == ops.MOE_ERR_UNSUPPORTED
    with pytest.raises(ops.MoeError) as ei:  # workspace too small
        ops.moe_expert_ffn(1 << 20, 4, d, 1 << 24, 8, 1 << 21, 1 << 21, 1 << 21, 1 << 21, 1 << 21, 1 << 21,
                           1 << 21, None, 0, 8, 1 << 21, 1 << 24, 16, None)
    assert ei.value.status == ops.MOE_ERR_CAPACITY
    p = 1 << 21  # checked before any launch: no device memory is touched
    one = (p, p, p, p, p, p, p, p, p, p)
    with pytest.raises(ops.MoeError) as ei:  # at most 8 shared experts
        ops.moe_route_sort_lookup(p, 1, d, 0.0, p, 8, *one, n_shared=9)
    assert ei.value.status == ops.MOE_ERR_INVALID
    with pytest.raises(ops.MoeError) as ei:  # k + n_shared above 32
        ops.moe_route_sort_lookup(p, 1, ops.desc(64, 30, 64, 32, 32, 4), 0.0, p, 64, *one, n_shared=3)
    assert ei.value.status == ops.MOE_ERR_UNSUPPORTED
    with pytest.raises(ops.MoeError) as ei:  # one token only
        ops.moe_route_sort_lookup(p, 2, d, 0.0, p, 8, *one)
    assert ei.value.status == ops.MOE_ERR_UNSUPPORTED
    assert ops.status_string(ops.MOE_ERR_TIMEOUT) == "device wait timed out"


@pytest.mark.parametrize("S,E,npass", [(16, 64, 6), (8, 20, 8), (4, 10, 6)])
def test_slot_cache_matches_oracle_lru(lib, orc, S, E, npass):
    r = np.random.default_rng(S)
    placed = r.choice(E, S // 2, replace=False).astype(np.int32)
    c = ops.SlotCache(E, 3, S, layer_class=[0, 1, 0])
    m = orc.LruModel(E, S, slot_base=c.layer_base(2))
    assert c.layer_base(2) == S and c.layer_base(1) == 0 and c.class_slots(0) == 2 * S
    c.place(2, placed, [c.layer_base(2) + i for i in range(len(placed))])
    m.place(placed, [c.layer_base(2) + i for i in range(len(placed))])
    for _ in range(200):
        pe = np.sort(r.choice(E, npass, replace=False)).astype(np.int32)
        missing = [int(e) for e in pe if m.table[e] < 0]
        st, inst = c.step(2, pe.tolist())
        got, fail = m.step(pe)
        assert [s for _, s in inst] == got.tolist()
        assert [e for e, _ in inst] == missing
        assert (st == ops.MOE_ERR_CAPACITY) == (fail > 0)
        assert list(c.table(2)) == m.table.tolist()
    h, mi, ev = c.stats()
    assert h + mi == 200 * npass
    c.close()


def test_slot_cache_capacity(lib):
    c = ops.SlotCache(10, 1, 2)
    st, inst = c.step(0, [1, 2, 3])
    assert st == ops.MOE_ERR_CAPACITY and inst[-1] == (3, -1)


def test_kernel_path_choice_and_workspace_growth(lib):
    # host-only decisions: the fused single-launch decode up to T*k <= 64 (T <= 8), the GEMV kernels
    # without sorted x, -1 for an invalid shape; the workspace counts the per-pair output buffer of the
    # tensor-core path (which runs wherever the fused decode kernel does not, given sorted x)
    d = ops.desc(512, 10, 2048, 512, 64, 3, 3)
    assert ops.moe_ffn_kernel_path(d, 1, False) == ops.MOE_PATH_FUSED_DECODE
    assert ops.moe_ffn_kernel_path(d, 6, False) == ops.MOE_PATH_FUSED_DECODE
    assert ops.moe_ffn_kernel_path(d, 7, False) == ops.MOE_PATH_GEMV  # 70 pairs > 64
    assert ops.moe_ffn_kernel_path(d, 300, False) == ops.MOE_PATH_GEMV
    assert ops.moe_ffn_kernel_path(d, 0, False) == -1
    assert ops.moe_ffn_kernel_path(ops.desc(8, 2, 64, 32, 48, 4, 4), 4, False) == -1  # group 48
    per_pair_o = 10 * 2048 * 4
    for T in (1, 8, 9, 32):  # every token adds at least its pairs' outputs for the tensor-core path
        assert ops.moe_workspace_bytes(d, T + 1) - ops.moe_workspace_bytes(d, T) >= per_pair_o
    assert ops.moe_ffn_kernel_path(d, 9, False) == ops.MOE_PATH_GEMV  # (with sorted x: tcgen05, on a GPU)
