"""Guessed prefetch on the GPU (RFC "How the prototype works", item "Reads":
the next two layers' experts are guessed by running their routers on the
current hidden states and read in the background; PR #50717 commit note:
install_ahead skips guessed reads still in flight), through the C ABI:

  * moe_router_logits against the oracle's router projection;
  * decode steps through moe_decode_layer_ahead over a residual stream of
    hidden states, with the next two layers' routers evaluated on each
    layer's state: every layer's routing and y match the oracle (guesses only
    move installs earlier), every expert in a table has its own bytes in its
    slot, and guesses do enter the tables."""
import numpy as np
import pytest
import torch

from streamed_quantized_expert_b200 import ops, synth
from streamed_quantized_expert_b200.runtime import LayerSpec, Streamer
from tests._bank import assert_close, oracle_bank
from tests.test_gpu_pipeline import initial_fill

pytestmark = pytest.mark.gpu
TOL = 2e-2


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("T,E,H", [(1, 512, 2048), (5, 128, 1024), (64, 8, 64)])
def test_router_logits(orc, T, E, H):
    x = synth.activations(7, 0, T, H)
    W = synth.router_weights(7, 0, E, H)
    bias = synth.router_bias(7, 0, E)
    scale = 1.0 / np.sqrt(H)
    out = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ops.moe_router_logits(dev(x.view(np.int16)), T, dev(W.view(np.int16)), dev(bias), scale, E, H, out)
    torch.cuda.synchronize()
    ref = orc.router_logits(x, W, bias, scale)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    Wf = synth.bf16_bits_to_f32(W).astype(np.float64)
    bound = 1e-6 * scale * (np.abs(xf) @ np.abs(Wf).T) + 1e-6 * np.abs(bias)[None, :]  # fp32 accumulation
    assert np.all(np.abs(out.cpu().numpy() - ref) <= bound)


def test_decode_with_guessed_prefetch(orc):
    n_layers, E, k, H, I, g, S = 4, 256, 4, 256, 128, 64, 48
    bank = oracle_bank(orc, 8, H, I, g, 4, 4, seed=91)
    specs, host_slots = [], []
    for l in range(n_layers):
        perm = synth.bank_permutation(91, l, E) % 8
        specs.append(LayerSpec(ops.desc(E, k, H, I, g, 4, 4), torch.from_numpy(bank).pin_memory(), perm.tolist()))
        host_slots.append([bank[perm[e]] for e in range(E)])
    st = Streamer(specs, S, max_tokens=1)
    initial_fill(st, 91, S)
    Wr = [synth.router_weights(91, l, E, H) for l in range(n_layers)]
    br = [synth.router_bias(91, l, E) for l in range(n_layers)]
    Wr_d = [dev(w.view(np.int16)) for w in Wr]
    br_d = [dev(b) for b in br]
    scale = 1.0 / np.sqrt(H)
    glog = torch.empty((2, 1, E), dtype=torch.float32, device="cuda")
    for step in range(10):
        xs = synth.hidden_stream(91, n_layers, 1, H, step=step)
        for l in range(n_layers):
            x = xs[l]
            logits = orc.router_logits(x, Wr[l], br[l], scale).astype(np.float32)  # the real routing's input
            x_d = dev(x.view(np.int16))
            guesses = []
            for dist in (1, 2):
                gl = l + dist
                if gl < n_layers:
                    ops.moe_router_logits(x_d, 1, Wr_d[gl], br_d[gl], scale, E, H, glog[dist - 1], st.stream)
                    guesses.append((gl, glog[dist - 1]))
            y = st.decode_layer_ahead(l, x_d, dev(logits), 1, 0.0, guesses)
            ids, w, _ = orc.route(logits, k)
            assert np.array_equal(st.ids[:1].cpu().numpy(), ids)
            assert_close(y.cpu().numpy(), orc.expert_ffn(x, H, I, g, 4, 4, ids, w, host_slots[l]), TOL)
    torch.cuda.synchronize()
    st.ahead.synchronize()
    stats = st.prefetch.stats()
    assert stats["started"] > 0 and stats["entered"] > 0
    # every expert the host tables name has its own bytes in its slot (a device
    # table catches up with its layer's reservations when that layer next runs)
    sb = st.class_bytes[0]
    pool = st.pools[0].cpu().numpy()
    for l in range(n_layers):
        tab = np.array(list(st.cache.table(l)))
        for e in np.nonzero(tab >= 0)[0]:
            s = int(tab[e])
            assert np.array_equal(pool[s * sb:(s + 1) * sb], host_slots[l][e]), (l, e, s)
    assert st.check_dev_err() == 0
