"""GPU vs oracle for stages 4-5 (dequant + SwiGLU FFN + combine) through the
C ABI, at the workload shapes: within 2e-2 of max(|ref|, row rms) elementwise
(the stated bf16-level tolerance); plus invariants (slot permutation, pass
splitting, skipped non-resident experts)."""
import numpy as np
import pytest
import torch

from streamed_quantized_expert_b200 import build, ops, synth
from tests._bank import assert_close, oracle_bank

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


class Setup:
    """Bank of R distinct quantized experts; expert e -> bank row e % R; every
    expert resident at slot perm[e] of a pool of E slots."""

    def __init__(self, orc, E, k, H, I, g, bg, bd, R, seed=0, perm_seed=1):
        self.E, self.k, self.H, self.I = E, k, H, I
        self.d = ops.desc(E, k, H, I, g, bg, bd)
        self.geom = (H, I, g, bg, bd)
        self.bank = oracle_bank(orc, R, H, I, g, bg, bd, seed)
        self.sb = self.bank.shape[1]
        self.row = np.arange(E) % R
        self.perm = synth.rng(perm_seed, E).permutation(E).astype(np.int32)
        bank_d = dev(self.bank)
        self.pool = torch.empty((E, self.sb), dtype=torch.uint8, device="cuda")
        self.pool[torch.from_numpy(self.perm).long().cuda()] = bank_d[torch.from_numpy(self.row).long().cuda()]
        self.table = dev(self.perm)
        self.slots_np = [self.bank[self.row[e]] for e in range(E)]

    def gpu(self, x, ids, w, T, passes=None, table=None, sorted_x=False):
        E, k = self.E, self.k
        ws_b = ops.moe_workspace_bytes(self.d, T)
        ws = torch.zeros(ws_b, dtype=torch.uint8, device="cuda")
        offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        pairs = torch.empty(max(T * k, 1), dtype=torch.int32, device="cuda")
        active = torch.empty(E, dtype=torch.int32, device="cuda")
        na = torch.zeros(1, dtype=torch.int32, device="cuda")
        ids_d, w_d, x_d = dev(ids), dev(w), dev(x.view(np.int16))
        xs = torch.empty((max(T * k, 1), self.H), dtype=torch.int16, device="cuda") if sorted_x else None
        ops.moe_sort(ids_d, x_d if sorted_x else None, T, self.d, offsets, pairs, active, na, xs, ws, ws_b)
        y = torch.zeros((T, self.H), dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        tab = self.table if table is None else table
        for pb, pl in passes or [(0, E)]:
            ops.moe_expert_ffn(x_d, T, self.d, self.pool, E, tab, ids_d, w_d, offsets, pairs, active, na, xs,
                               pb, pl, y, ws, ws_b, err)
        torch.cuda.synchronize()
        return y.cpu().numpy(), int(err.item())

    def oracle(self, orc, x, ids, w, tokens=None):
        return orc.expert_ffn(x, *self.geom, ids, w.astype(np.float64), self.slots_np, tokens)


def _case(orc, E, k, H, I, g, bg, bd, T, R, seed=0):
    s = Setup(orc, E, k, H, I, g, bg, bd, R, seed)
    x = synth.activations(seed, 1, T, H)
    ids, w = synth.random_routing(seed, T, E, k)
    return s, x, ids, w


def test_tiny_layer_full_route(orc):
    # 8 experts, top-2, H 64, I 32, 4-bit g32, 4 tokens, logits N(0,1), seed 0
    s = Setup(orc, 8, 2, 64, 32, 32, 4, 4, R=8)
    x = synth.activations(0, 0, 4, 64)
    logits = synth.router_logits(0, 0, 4, 8, beta=0.0)
    ids_ref, w_ref, _ = orc.route(logits, 2)
    ids = torch.empty((4, 2), dtype=torch.int32, device="cuda")
    w = torch.empty((4, 2), dtype=torch.float32, device="cuda")
    ops.moe_route(dev(logits), 4, s.d, 0.0, s.table, ids, w)
    torch.cuda.synchronize()
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    y, err = s.gpu(x, ids.cpu().numpy(), w.cpu().numpy(), 4)
    assert err == 0
    assert_close(y, orc.expert_ffn(x, 64, 32, 32, 4, 4, ids_ref, w_ref, s.slots_np), TOL)


@pytest.mark.parametrize("T", [1, 2, 5])
def test_flash_next_decode_shapes(orc, T):
    s, x, ids, w = _case(orc, 512, 10, 2048, 512, 64, 3, 3, T, R=12)
    y, err = s.gpu(x, ids, w, T)
    assert err == 0
    assert_close(y, s.oracle(orc, x, ids, w), TOL)


@pytest.mark.parametrize("T", [1, 8, 32, 64])
def test_coder_batched_decode_shapes(orc, T):
    s, x, ids, w = _case(orc, 128, 8, 2048, 768, 64, 4, 4, T, R=10, seed=3)
    y, err = s.gpu(x, ids, w, T)
    assert err == 0
    tok = np.arange(T) if T <= 8 else np.array([0, 1, T // 2, T - 1])
    assert_close(y[tok], s.oracle(orc, x, ids, w, tok), TOL)


def test_mixed_class_down_6bit(orc):
    s, x, ids, w = _case(orc, 512, 10, 2048, 512, 64, 4, 6, 3, R=10, seed=5)
    y, err = s.gpu(x, ids, w, 3)
    assert err == 0
    assert_close(y, s.oracle(orc, x, ids, w), TOL)


@pytest.mark.parametrize("g,bg,bd", [(32, 3, 4), (128, 6, 6), (64, 6, 3), (32, 4, 6)])
def test_group_and_width_grid(orc, g, bg, bd):
    s, x, ids, w = _case(orc, 16, 4, 384, 256, g, bg, bd, 9, R=6, seed=g + bg)
    y, err = s.gpu(x, ids, w, 9)
    assert err == 0
    assert_close(y, s.oracle(orc, x, ids, w), TOL)


@pytest.mark.parametrize("T", [65, 300])
def test_unfused_combine_and_passes(orc, T):
    # T > 64 takes the per-pair output + combine path; passes of 64 experts
    s, x, ids, w = _case(orc, 512, 10, 2048, 512, 64, 3, 3, T, R=8, seed=7)
    passes = [(p, 64) for p in range(0, 512, 64)]
    y, err = s.gpu(x, ids, w, T, passes=passes)
    assert err == 0
    tok = np.array([0, 1, T // 3, T - 1])
    assert_close(y[tok], s.oracle(orc, x, ids, w, tok), TOL)


def test_pass_splitting_invariance(orc):
    s, x, ids, w = _case(orc, 256, 8, 512, 256, 64, 4, 4, 16, R=6, seed=9)
    one, _ = s.gpu(x, ids, w, 16)
    split, _ = s.gpu(x, ids, w, 16, passes=[(p, 64) for p in range(0, 256, 64)])
    np.testing.assert_allclose(split, one, rtol=1e-5, atol=1e-6)


def test_slot_permutation_invariance(orc):
    a = Setup(orc, 64, 4, 512, 256, 64, 3, 3, R=8, perm_seed=1)
    b = Setup(orc, 64, 4, 512, 256, 64, 3, 3, R=8, perm_seed=2)
    assert not np.array_equal(a.perm, b.perm)
    x = synth.activations(2, 2, 5, 512)
    ids, w = synth.random_routing(2, 5, 64, 4)
    ya, _ = a.gpu(x, ids, w, 5)
    yb, _ = b.gpu(x, ids, w, 5)
    assert np.array_equal(ya, yb)


def test_non_resident_expert_is_flagged_and_skipped(orc):
    s, x, ids, w = _case(orc, 32, 4, 256, 128, 64, 4, 4, 6, R=5, seed=11)
    gone = int(ids[0, 1])
    table = s.perm.copy()
    table[gone] = -1
    y, err = s.gpu(x, ids, w, 6, table=dev(table))
    assert err & ops.DEV_ERR_NOT_RESIDENT
    w2 = w.copy()
    w2[ids == gone] = 0.0
    assert_close(y, s.oracle(orc, x, ids, w2), TOL)
