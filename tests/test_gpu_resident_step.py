"""A decode step of a fully resident model (RFC "How the prototype works",
item "Cache": when every expert is resident, layers never synchronise with
the host) through the native driver, captured once as a CUDA graph of every
layer's moe_decode_layer call and replayed on new inputs: each layer's
routing and y against the oracle, with no install and no device error."""
import numpy as np
import pytest
import torch

from streamed_quantized_expert_b200 import build, ops, synth
from streamed_quantized_expert_b200.runtime import Streamer
from tests._bank import assert_close
from tests.test_gpu_pipeline import make

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()


@pytest.mark.parametrize("T,bits", [(1, [(3, 3), (3, 3), (4, 6), (3, 3)]), (5, [(4, 4)] * 4)])
def test_resident_step_as_one_graph(orc, T, bits):
    n_layers, E, k, H, I, g = 4, 64, 4, 256, 128, 64
    specs, host_slots = make(orc, n_layers, E, k, H, I, g, bits, E, R=6, seed=31)
    st = Streamer(specs, E, max_tokens=T, stream=torch.cuda.Stream())  # a graph captures a non-default stream
    for l in range(n_layers):  # every expert of every layer in a slot
        st.place(l, list(range(E)), synth.slot_permutation(31, l, E).tolist())
    assert all(st.cache.resident(l) >= E for l in range(n_layers))
    xin = torch.empty((n_layers, T, H), dtype=torch.int16, device="cuda")
    lgin = torch.empty((n_layers, T, E), dtype=torch.float32, device="cuda")
    ys = torch.empty((n_layers, T, H), dtype=torch.float32, device="cuda")
    ids_out = torch.empty((n_layers, T, k), dtype=torch.int32, device="cuda")

    def load(step):
        xs = [synth.activations(31, l, T, H, step=step) for l in range(n_layers)]
        lgs = [synth.router_logits(31, l, T, E, step=step) for l in range(n_layers)]
        xin.copy_(torch.from_numpy(np.stack(xs).view(np.int16)))
        lgin.copy_(torch.from_numpy(np.stack(lgs)))
        return xs, lgs

    def step():
        for l in range(n_layers):
            st.decode_layer(l, xin[l], lgin[l], T, 0.0, y=ys[l])
            with torch.cuda.stream(st.stream):
                ids_out[l].copy_(st.ids[:T])

    load(0)
    torch.cuda.synchronize()  # the inputs are copied on the current stream, the layers run on st.stream
    step()  # eager: first-use setup of the kernels outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=st.stream):
        step()
    torch.cuda.synchronize()
    inst0 = st.installs
    for s in (1, 2):
        xs, lgs = load(s)
        graph.replay()
        torch.cuda.synchronize()
        for l in range(n_layers):
            ids, w, _ = orc.route(lgs[l], k)
            assert np.array_equal(ids_out[l].cpu().numpy(), ids)
            ref = orc.expert_ffn(xs[l], H, I, g, *bits[l], ids, w, host_slots[l])
            assert_close(ys[l].cpu().numpy(), ref, TOL)
    assert st.installs == inst0
    assert st.check_dev_err() == 0
