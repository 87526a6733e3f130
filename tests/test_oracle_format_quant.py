"""Pins for the slot format, the affine quantizer and the dequant closed form.

The RFC says experts are stored in MLX's affine format, one contiguous row per
expert; 1bit-MONSTER PR #137 keys size classes by the bytes one expert needs.
"""
import numpy as np
import pytest

from tests import _format_np as F


@pytest.mark.parametrize("b", [3, 4, 6])
@pytest.mark.parametrize("K", [32, 64, 128, 512, 768, 2048])
def test_code_roundtrip_and_independent_decoder(orc, b, K):
    r = np.random.default_rng(b * 1000 + K)
    rows = 16
    rb = orc.row_bytes(K, b)
    assert rb == F.ceil128(K) * b // 8
    q = np.zeros((rows, rb), np.uint8)
    codes = r.integers(0, 1 << b, size=(rows, K))
    for i in range(rows):
        for k in range(K):
            orc.set_code(q, K, i, k, b, int(codes[i, k]))
    for i in range(rows):
        assert [orc.get_code(q, K, i, k, b) for k in range(K)] == codes[i].tolist()
    assert np.array_equal(F.decode_rows(q, K, b), codes)


@pytest.mark.parametrize("b", [3, 4, 6])
def test_layout_is_a_bijection(orc, b):
    # every bit of an 8-row group of 128-input blocks belongs to exactly one
    # (row, input, code bit): setting the codes one by one to all-ones adds b
    # new bits each time and ends with every byte 0xFF
    q = np.zeros((8, orc.row_bytes(128, b)), np.uint8)
    seen = 0
    for row in range(8):
        for k in range(128):
            orc.set_code(q, 128, row, k, b, (1 << b) - 1)
            n = int(np.unpackbits(q).sum())
            assert n == seen + b
            seen = n
    assert np.all(q == 0xFF)
    # the numpy description agrees: unit-word-bit triples cover a unit exactly once
    U, W, B = F._bit_positions(128, b)
    flat = ((U * b + W) * 32 + B).reshape(-1)
    assert np.array_equal(np.sort(flat), np.arange(128 * b))


def test_slot_sizes_for_the_workload_shapes(orc):
    # H=2048, I=512, g=64, 3-bit: q 1,179,648 + scale/bias 196,608
    assert orc.slot_bytes(2048, 512, 64, 3, 3) == 1_376_256
    # mixed classes: 4/4-bit and 4/6-bit
    assert orc.slot_bytes(2048, 512, 64, 4, 4) == 1_769_472
    assert orc.slot_bytes(2048, 512, 64, 4, 6) == 2_031_616
    # H=2048, I=768, 4-bit g64
    assert orc.slot_bytes(2048, 768, 64, 4, 4) == 2_654_208
    off, n = orc.slot_layout(2048, 512, 64, 3, 3)
    assert off == [0, 786_432, 1_179_648, 1_310_720] and all(o % 256 == 0 for o in off)


@pytest.mark.parametrize("b,g", [(3, 64), (4, 32), (4, 64), (6, 64), (4, 128), (3, 32)])
def test_quantizer_properties(orc, b, g):
    r = np.random.default_rng(b * 7 + g)
    K = 256
    w = (r.standard_normal((32, K)) * 0.02).astype(np.float32)
    w[3, :g] = np.float32(0.0123)  # constant group
    q, sb = orc.quantize_rows(w, g, b)
    codes = F.decode_rows(q, K, b)
    assert codes.min() >= 0 and codes.max() <= (1 << b) - 1
    deq = orc.dequant_rows(q, sb, K, g, b)
    sbr = F.sb_rows(sb, 32, sb.size // 32)
    s = ((sbr & 0xFFFF).astype(np.uint32) << 16).view(np.float32)
    bias = ((sbr >> 16).astype(np.uint32) << 16).view(np.float32)
    # scale = bf16 of (max-min)/(2^b-1); bias = bf16 of the group minimum
    wg = w.reshape(32, K // g, g)
    assert np.all(np.abs(s[:, : K // g] - (wg.max(2) - wg.min(2)) / ((1 << b) - 1)) <= np.abs(s[:, : K // g]) * 2 ** -8 + 1e-30)
    assert np.all(np.abs(bias[:, : K // g] - wg.min(2)) <= np.abs(wg.min(2)) * 2 ** -8)
    # |w - deq| <= scale/2 + bf16 rounding of scale and bias over the whole code range
    si = np.repeat(s[:, : K // g], g, axis=1)
    bi = np.repeat(bias[:, : K // g], g, axis=1)
    slack = si / 2 + np.abs(si) * ((1 << b) - 1) * 2 ** -8 + np.abs(bi) * 2 ** -8 + 1e-9
    assert np.all(np.abs(w - deq) <= slack)
    # a constant group dequantises to its bias exactly, which is bf16(w)
    assert np.all(deq[3, :g] == bias[3, 0]) and s[3, 0] == 0.0


def test_padded_groups_are_zero(orc):
    w = (np.random.default_rng(1).standard_normal((16, 32)) * 0.02).astype(np.float32)
    q, sb = orc.quantize_rows(w, 32, 4)
    assert q.shape == (16, 64) and sb.shape == (16, 4)
    sbr = F.sb_rows(sb, 16, 4)
    assert np.all(sbr[:, 1:] == 0) and np.all(sbr[:, 0] != 0)


@pytest.mark.parametrize("b", [3, 4, 6])
def test_dequant_is_single_rounding_fma(orc, b):
    r = np.random.default_rng(b)
    K, g = 512, 64
    w = (r.standard_normal((16, K)) * 0.05).astype(np.float32)
    q, sb = orc.quantize_rows(w, g, b)
    assert np.array_equal(orc.dequant_rows(q, sb, K, g, b).view(np.uint32),
                          F.dequant_rows(q, sb, K, g, b).view(np.uint32))


def test_slot_sections_roundtrip(orc):
    r = np.random.default_rng(3)
    H, I, g = 128, 64, 32
    w_gu = (r.standard_normal((2 * I, H)) * 0.02).astype(np.float32)
    w_d = (r.standard_normal((H, I)) * 0.02).astype(np.float32)
    slot = orc.build_slot(w_gu, w_d, g, 4, 6)
    off, n = orc.slot_layout(H, I, g, 4, 6)
    assert slot.size == n
    gu, dn = orc.dequant_slot(slot, H, I, g, 4, 6)
    q = slot[off[0]: off[0] + 2 * I * orc.row_bytes(H, 4)].reshape(2 * I, -1)
    sb = slot[off[2]: off[2] + 2 * I * orc.row_groups(H, g) * 4].view(np.uint32).reshape(2 * I, -1)
    stored = F.dequant_rows(q, sb, H, g, 4)
    logical = stored[[F.gate_up_storage_row(R, I) for R in range(2 * I)]]
    assert np.array_equal(gu, logical)
    # gate rows first, then up rows: the quantised gate block reproduces w_gu[:I]
    assert np.max(np.abs(gu - w_gu)) < 0.02
    qd = slot[off[1]: off[1] + H * orc.row_bytes(I, 6)].reshape(H, -1)
    sd = slot[off[3]: off[3] + H * orc.row_groups(I, g) * 4].view(np.uint32).reshape(H, -1)
    assert np.array_equal(dn, F.dequant_rows(qd, sd, I, g, 6))
