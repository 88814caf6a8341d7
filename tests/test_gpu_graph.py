"""CUDA-graph replay of decode steps: the step counter lives in device memory
(lores_decode_step_dev), so several layers' steps and the counter advance are captured
once and replayed; every replay must equal the ordinary host-stepped calls bit for bit."""
import numpy as np
import pytest
import torch

from bit_recurrent_state_lores_b200 import synth

from .harness import GpuRun

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def lib():
    from bit_recurrent_state_lores_b200 import lores
    return lores


@pytest.mark.parametrize("axis", [0, 1])
def test_graph_replay_equals_host_steps(axis):
    L = lib()
    wl = synth.Workload("graph", B=4, H=3, d_k=64, d_v=32, steps=6, delta=1, diag=1, group=64,
                        decay="kda", outliers=2, seed=6)
    bits = [8, 4, 32] if axis == 0 else [8, 4, 6]
    hp = synth.head_params(wl)
    layers = 3
    ref = [GpuRun(wl, bits, seed=10 + l, axis=axis) for l in range(layers)]
    gr = [GpuRun(wl, bits, seed=10 + l, axis=axis) for l in range(layers)]
    # static input and output buffers of the graph, one set per layer
    static = [[torch.empty_like(x) for x in synth.step_inputs(wl, 0, hp, device="cuda")]
              for _ in range(layers)]
    outs = [torch.empty(wl.B, wl.H, wl.d_v, device="cuda") for _ in range(layers)]
    t0 = 5
    step = torch.tensor([t0], dtype=torch.int64, device="cuda")
    # warm up once outside capture (first launches load the modules), then reset the state
    for l in range(layers):
        L.lores_decode_step_dev(gr[l].h, *static[l], outs[l], step)
    torch.cuda.synchronize()
    zc, zs = gr[0].export()
    for l in range(layers):
        gr[l].load(np.zeros_like(zc), np.zeros_like(zs))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for l in range(layers):
            L.lores_decode_step_dev(gr[l].h, *static[l], outs[l], step)
        L.lores_advance_step(step, 1)
    for n in range(wl.steps):
        t = t0 + n
        for l in range(layers):
            inp = synth.step_inputs(wl, t, hp, device="cuda", layer=l)
            for dst, src in zip(static[l], inp):
                dst.copy_(src)
            ref[l].step(inp, t)
        g.replay()
        torch.cuda.synchronize()
        for l in range(layers):
            assert torch.equal(outs[l], ref[l].o), (n, l)
    assert int(step.item()) == t0 + wl.steps
    for l in range(layers):
        a, b = ref[l].export(), gr[l].export()
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
        assert gr[l].check() == L.LORES_OK
        ref[l].close()
    del g
    for r in gr:
        r.close()
