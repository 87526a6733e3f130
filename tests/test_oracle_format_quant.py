"""Pins for the slot format, the affine quantizer and the dequant closed form.

The RFC says experts are stored in MLX's affine format, one contiguous row per
expert; 1bit-MONSTER PR #137 keys size classes by the bytes one expert needs.
"""
import numpy as np
import pytest

from streamed_quantized_expert_b200 import synth
from tests import _format_np as F


@pytest.mark.parametrize("b", [3, 4, 6])
@pytest.mark.parametrize("K", [32, 64, 128, 512, 768, 2048])
def test_code_roundtrip_and_independent_decoder(orc, b, K):
    r = np.random.default_rng(b * 1000 + K)
    rows, g = 32, 32
    rb = orc.row_bytes(K, b)
    assert rb == F.ceil128(K) * b // 8
    assert orc.tile_bytes(K, g, b) == F.geometry(K, g, b)[2]
    proj = np.zeros(rows // 16 * orc.tile_bytes(K, g, b), np.uint8)
    codes = r.integers(0, 1 << b, size=(rows, K))
    for i in range(rows):
        for k in range(K):
            orc.set_code(proj, K, g, i, k, b, int(codes[i, k]))
    for i in range(rows):
        assert [orc.get_code(proj, K, g, i, k, b) for k in range(K)] == codes[i].tolist()
    assert np.array_equal(F.decode_rows(proj, rows, K, g, b), codes)


@pytest.mark.parametrize("b", [3, 4, 6])
def test_layout_is_a_bijection(orc, b):
    # every bit of an 8-row group of 128-input blocks belongs to exactly one
    # (row, input, code bit): setting the codes one by one to all-ones adds b
    # new bits each time and ends with every byte 0xFF
    g = 128
    proj = np.zeros(orc.tile_bytes(128, g, b), np.uint8)
    codes = proj[: 16 * orc.row_bytes(128, b)]  # the tile's code bytes (a view)
    seen = 0
    for row in range(16):
        for k in range(128):
            orc.set_code(proj, 128, g, row, k, b, (1 << b) - 1)
            n = int(np.unpackbits(proj).sum())
            assert n == seen + b
            seen = n
    assert np.all(codes == 0xFF) and np.all(proj[codes.size:] == 0)
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
    # 64 gate/up tiles of 16 x 768 B codes + 16 x 32 words; 128 down tiles of 16 x 192 B + 16 x 8 words
    assert off == [0, 917_504, 14_336, 3_584] and n == 1_376_256


@pytest.mark.parametrize("b,g", [(3, 64), (4, 32), (4, 64), (6, 64), (4, 128), (3, 32)])
def test_quantizer_properties(orc, b, g):
    r = np.random.default_rng(b * 7 + g)
    K = 256
    w = (r.standard_normal((32, K)) * 0.02).astype(np.float32)
    w[3, :g] = np.float32(0.0123)  # constant group
    proj = orc.quantize_rows(w, g, b)
    codes = F.decode_rows(proj, 32, K, g, b)
    assert codes.min() >= 0 and codes.max() <= (1 << b) - 1
    deq = orc.dequant_rows(proj, 32, K, g, b)
    sbr = F.sb_rows(proj, 32, K, g, b)
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
    proj = orc.quantize_rows(w, 32, 4)
    assert proj.shape == (1, 16 * 64 + 16 * 4 * 4)
    sbr = F.sb_rows(proj, 16, 32, 32, 4)
    assert np.all(sbr[:, 1:] == 0) and np.all(sbr[:, 0] != 0)


@pytest.mark.parametrize("b", [3, 4, 6])
def test_dequant_is_single_rounding_fma(orc, b):
    r = np.random.default_rng(b)
    K, g = 512, 64
    w = (r.standard_normal((16, K)) * 0.05).astype(np.float32)
    proj = orc.quantize_rows(w, g, b)
    assert np.array_equal(orc.dequant_rows(proj, 16, K, g, b).view(np.uint32),
                          F.dequant_rows(proj, 16, K, g, b).view(np.uint32))


def test_slot_sections_roundtrip(orc):
    r = np.random.default_rng(3)
    H, I, g = 128, 64, 32
    w_gu = (r.standard_normal((2 * I, H)) * 0.02).astype(np.float32)
    w_d = (r.standard_normal((H, I)) * 0.02).astype(np.float32)
    slot = orc.build_slot(w_gu, w_d, g, 4, 6)
    off, n = orc.slot_layout(H, I, g, 4, 6)
    assert slot.size == n
    gu, dn = orc.dequant_slot(slot, H, I, g, 4, 6)
    pg = slot[off[0]: off[0] + 2 * I // 16 * off[2]]
    stored = F.dequant_rows(pg, 2 * I, H, g, 4)
    logical = stored[[F.gate_up_storage_row(R, I) for R in range(2 * I)]]
    assert np.array_equal(gu, logical)
    # gate rows first, then up rows: the quantised gate block reproduces w_gu[:I]
    assert np.max(np.abs(gu - w_gu)) < 0.02
    pd = slot[off[1]: off[1] + H // 16 * off[3]]
    assert np.array_equal(dn, F.dequant_rows(pd, H, I, g, 6))


def test_bf16_experts_format(orc):
    # BF16 experts (RFC "How the prototype works", item "Cache"): a projection
    # is its rows of bf16 values, row-major, rows padded to 128 inputs, no
    # scale/bias words; the "quantizer" rounds to bf16 (nearest even)
    H, I = 208, 96  # neither a multiple of 128
    w_gu, w_d = synth.expert_weights(4, 1, H, I)
    slot = orc.build_slot(w_gu, w_d, 32, 16, 16)
    off, nbytes = orc.slot_layout(H, I, 32, 16, 16)
    assert off[2] == 16 * 256 * 2 and off[3] == 16 * 128 * 2  # tile = 16 padded rows, 2 bytes per input
    assert off[1] == 2 * I * 256 * 2 and nbytes == off[1] + H * 128 * 2
    gu, dn = orc.dequant_slot(slot, H, I, 32, 16, 16)
    assert np.array_equal(gu, synth.bf16_bits_to_f32(synth.to_bf16_bits(w_gu)))
    assert np.array_equal(dn, synth.bf16_bits_to_f32(synth.to_bf16_bits(w_d)))
    # the padding is zero and the storage rows are the gate/up interleave
    pg = slot[:off[1]].view("<u2").reshape(2 * I, 256)
    assert not pg[:, H:].any()
    R = 100  # up row 100 - 96 = 4 -> storage row 16 * 0 + 8 + 4
    assert np.array_equal(pg[12, :H], synth.to_bf16_bits(w_gu[R]))
