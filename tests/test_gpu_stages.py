"""GPU vs oracle, stage by stage, through the C ABI: the routing exp, the
quantizer, dequantisation (bit-exact), route (ids bit-exact, weights 1e-5),
sort and slot lookup (bit-exact)."""
import struct

import numpy as np
import pytest
import torch

from streamed_quantized_expert_b200 import build, ops, synth
from tests._bank import oracle_bank

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    torch.cuda.init()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_exp_bit_exact_on_every_float_in_domain(orc):
    top = struct.unpack("<I", struct.pack("<f", 87.0))[0]
    chunk = 1 << 26
    x = torch.empty(chunk, dtype=torch.float32, device="cuda")
    out = torch.empty_like(x)
    for start in range(0, top + 1, chunk):
        n = min(chunk, top + 1 - start)
        bits = (np.arange(start, start + n, dtype=np.uint64) | 0x80000000).astype(np.uint32)
        x[:n] = torch.from_numpy(bits.view(np.float32)).cuda()
        ops.moe_exp_portable(x, n, out)
        ref = orc.exp_portable_neg_bits(start, n)
        got = out[:n].cpu().numpy()
        if not np.array_equal(got.view(np.uint32), ref.view(np.uint32)):
            i = int(np.argmax(got.view(np.uint32) != ref.view(np.uint32)))
            pytest.fail(f"exp mismatch at bits {start + i:#x}: gpu {got[i]!r} cpu {ref[i]!r}")


@pytest.mark.parametrize("rows,K,g,b", [(16, 64, 32, 4), (48, 2048, 64, 3), (16, 512, 64, 6), (16, 768, 128, 4),
                                        (16, 32, 32, 3), (64, 2048, 64, 4), (32, 768, 64, 16), (16, 96, 32, 16)])
def test_quantize_bit_exact(orc, rows, K, g, b):
    w = (synth.rng(rows, K, g, b).standard_normal((rows, K), dtype=np.float32) * np.float32(0.02))
    w[0, :g] = np.float32(0.5)  # constant group
    w[1, :] = 0.0
    ref = orc.quantize_rows(w, g, b)
    proj = torch.zeros(ref.shape, dtype=torch.uint8, device="cuda")
    ops.moe_quantize_rows(dev(w), rows, K, g, b, proj)
    torch.cuda.synchronize()
    assert np.array_equal(proj.cpu().numpy(), ref)


@pytest.mark.parametrize("bg,bd", [(3, 4), (16, 16), (16, 6)])
def test_quantize_gate_up_order_bit_exact(orc, bg, bd):
    # a whole expert through moe_quantize_rows (gate/up row order) vs the oracle's slot builder
    H, I, g = 256, 64, 64
    w_gu, w_d = synth.expert_weights(4, 0, H, I)
    ref = orc.build_slot(w_gu, w_d, g, bg, bd)
    d = ops.desc(8, 2, H, I, g, bg, bd)
    lay = ops.moe_slot_layout(d)
    slot = torch.zeros(lay.slot_bytes, dtype=torch.uint8, device="cuda")
    base = slot.data_ptr()
    ops.moe_quantize_rows(dev(w_gu), 2 * I, H, g, bg, base + lay.gate_up, gate_up_I=I)
    ops.moe_quantize_rows(dev(w_d), H, I, g, bd, base + lay.down)
    torch.cuda.synchronize()
    assert np.array_equal(slot.cpu().numpy(), ref)


@pytest.mark.parametrize("H,I,g,bg,bd", [(64, 32, 32, 4, 4), (2048, 512, 64, 3, 3), (256, 128, 64, 4, 6),
                                         (2048, 768, 64, 4, 4), (384, 256, 128, 6, 3), (256, 96, 32, 16, 16),
                                         (512, 256, 64, 16, 4)])
def test_dequant_slot_bit_exact(orc, H, I, g, bg, bd):
    bank = oracle_bank(orc, 3, H, I, g, bg, bd, seed=H + I)
    d = ops.desc(8, 2, H, I, g, bg, bd)
    pool = dev(bank.reshape(-1))
    out32 = torch.empty(2 * I * H + H * I, dtype=torch.float32, device="cuda")
    out16 = torch.empty(2 * I * H + H * I, dtype=torch.int16, device="cuda")
    for s in range(3):
        ops.moe_dequant_slot(pool, s, d, out32, out16)
        torch.cuda.synchronize()
        gu, dn = orc.dequant_slot(bank[s], H, I, g, bg, bd)
        ref = np.concatenate([gu.reshape(-1), dn.reshape(-1)])
        got = out32.cpu().numpy()
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
        assert np.array_equal(out16.cpu().numpy().view(np.uint16), synth.to_bf16_bits(ref))


@pytest.mark.parametrize("T,E,k", [(1, 512, 10), (4, 8, 2), (64, 128, 8), (1024, 512, 10), (37, 33, 5),
                                   (3, 1024, 32), (0, 16, 2)])
@pytest.mark.parametrize("L", [0.0, 0.15])
def test_route(orc, T, E, k, L):
    logits = synth.router_logits(T + E, 0, T, E)
    if T > 2:
        logits[1, :] = logits[1, 0]  # all-equal row: lowest ids win
        logits[2, 5:12] = logits[2].max()  # ties at the top
    table = np.where(synth.rng(E, k).random(E) < 0.25, np.arange(E), -1).astype(np.int32)
    ids_ref, w_ref, _ = orc.route(logits, k, L, table)
    ids = torch.full((max(T, 1), k), -7, dtype=torch.int32, device="cuda")
    w = torch.zeros((max(T, 1), k), dtype=torch.float32, device="cuda")
    ops.moe_route(dev(logits) if T else 1 << 20, T, ops.desc(E, k, 64, 32, 32, 4), L, dev(table), ids, w)
    torch.cuda.synchronize()
    if T == 0:
        return
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert np.max(np.abs(w.cpu().numpy() - w_ref)) <= 1e-5


@pytest.mark.parametrize("T,E,k", [(1, 512, 10), (4, 8, 2), (64, 128, 8), (102, 512, 10), (1024, 512, 10),
                                   (4096, 512, 10), (300, 1024, 7)])
def test_sort(orc, T, E, k):
    ids_np, _ = synth.random_routing(T, T, E, k)
    for t in range(T // 2 if T >= 300 else 0):  # a hot expert: 3 at rank 0 in half the tokens
        row = ids_np[t]
        if 3 in row:
            j = int(np.where(row == 3)[0][0])
            row[0], row[j] = row[j], row[0]
        else:
            row[0] = 3
    H = 64
    x_np = synth.activations(T, 0, T, H)
    d = ops.desc(E, k, H, 32, 32, 4)
    ws_b = ops.moe_workspace_bytes(d, T)
    ws = torch.zeros(ws_b, dtype=torch.uint8, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pairs = torch.empty(T * k, dtype=torch.int32, device="cuda")
    active = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    na = torch.zeros(1, dtype=torch.int32, device="cuda")
    xs = torch.empty((T * k, H), dtype=torch.int16, device="cuda")
    ops.moe_sort(dev(ids_np), dev(x_np.view(np.int16)), T, d, offsets, pairs, active, na, xs, ws, ws_b)
    torch.cuda.synchronize()
    o_ref, p_ref, a_ref = orc.sort(ids_np, E)
    assert np.array_equal(offsets.cpu().numpy(), o_ref)
    assert np.array_equal(pairs.cpu().numpy(), p_ref)
    n = int(na.item())
    assert n == a_ref.size and np.array_equal(active.cpu().numpy()[:n], a_ref)
    # x_sorted holds the gathered rows in fp16 (IEEE round to nearest even; |x| < 65504 here)
    want = synth.bf16_bits_to_f32(x_np[p_ref // k]).astype(np.float16).view(np.uint16)
    assert np.array_equal(xs.cpu().numpy().view(np.uint16), want)


def test_slot_lookup(orc):
    E, S = 512, 192
    r = synth.rng(77)
    table = np.full(E, -1, np.int32)
    table[r.choice(E, S, replace=False)] = r.permutation(S)
    table[17] = S + 5  # corrupt entry
    active = np.sort(r.choice(E, 300, replace=False)).astype(np.int32)
    if 17 not in active:
        active = np.sort(np.r_[active[:-1], 17]).astype(np.int32)
    act_d = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    act_d[: active.size] = dev(active)
    na = torch.tensor([active.size], dtype=torch.int32, device="cuda")
    for pb, pl in [(0, 64), (64, 64), (256, 64), (0, 512), (299, 64), (400, 64)]:
        slots = torch.full((max(pl, 1),), -9, dtype=torch.int32, device="cuda")
        miss = torch.full((max(pl, 1),), -9, dtype=torch.int32, device="cuda")
        nm = torch.zeros(1, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ops.moe_slot_lookup(dev(table), act_d, na, pb, pl, S, slots, miss, nm, err)
        torch.cuda.synchronize()
        s_ref, m_ref, bad = orc.slot_lookup(table, active, pb, pl, S)
        assert np.array_equal(slots.cpu().numpy()[: s_ref.size], s_ref)
        assert int(nm.item()) == m_ref.size and np.array_equal(miss.cpu().numpy()[: m_ref.size], m_ref)
        assert (int(err.item()) & ops.DEV_ERR_SLOT_RANGE != 0) == bool(bad)
