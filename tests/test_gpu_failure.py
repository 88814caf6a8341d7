"""The decode kernels' bounded waits, made to run out on purpose.

Every wait of a decode kernel on its own bulk copies gives up after a limit of GPU time:
the warp sets the TIMEOUT flag, lets its other copy in flight land and leaves, so the
call's outputs are incomplete but the GPU context stays usable.  The testing hook
lores_set_fault_injection withholds the copies of one work unit (they are announced to
the unit's barrier and never issued), so the owning warp waits out a short limit.
Nothing faults and nothing is left in flight.  The tests check that the call returns,
that lores_check_errors reports LORES_ERR_TIMEOUT, and that the next ordinary step on
the same handle agrees bit for bit with the oracle started from the handle's state.
"""
import numpy as np
import pytest
import torch

from bit_recurrent_state_lores_b200 import synth

from .harness import GpuRun, OracleTiles, host_tile_inputs

pytestmark = pytest.mark.gpu


def lib():
    from bit_recurrent_state_lores_b200 import lores
    return lores


@pytest.mark.parametrize("bits,B,G,kernel", [([8, 4, 8, 4, 8, 8], 96, 128, 3),
                                             ([8, 4, 8, 4, 8, 8], 96, 32, 1),
                                             ([8, 32, 4, 8, 8, 4], 4, 128, 0)],
                         ids=["tensor-core kernel", "two-rows-per-lane kernel", "general kernel"])
def test_withheld_copy_times_out_and_the_next_step_is_exact(bits, B, G, kernel):
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    L = lib()
    wl = synth.Workload("fail", B=B, H=len(bits), d_k=128, d_v=128, steps=5, decay="tau",
                        group=G, outliers=2, seed=21)
    hp = synth.head_params(wl)
    g = GpuRun(wl, bits, seed=5)
    try:
        assert g.layout.step_kernel == kernel
        per_seq = g.layout.units_per_step // wl.B
        for step in range(2):
            g.step(synth.step_inputs(wl, step, hp, device="cuda"), step)
        assert g.check() == L.LORES_OK
        # withhold unit 3 of sequence 1; every wait gives up after 2 ms
        L.lores_set_fault_injection(g.h, 1, min(3, per_seq - 1), 2000)
        g.step(synth.step_inputs(wl, 2, hp, device="cuda"), 2)
        torch.cuda.synchronize()                   # the call returns
        assert g.check() == L.LORES_ERR_TIMEOUT
        assert g.check() == L.LORES_OK             # the flag is cleared once read
        L.lores_set_fault_injection(g.h, -1, 0, 0)
        # the next ordinary step, from whatever state the incomplete call left
        codes, scales = g.export()
        tiles = [(b, h) for b in range(wl.B) for h in range(wl.H)]
        ref = OracleTiles(wl, bits, 5, tiles)
        for t in tiles:
            ref.load(t, *g.tile(codes, scales, *t))
        inp = synth.step_inputs(wl, 3, hp, device="cuda")
        o = g.step(inp, 3).cpu().numpy()
        out, flags = ref.step(host_tile_inputs(inp, tiles), 3)
        assert g.check() == L.LORES_OK and not any(flags.values())
        codes, scales = g.export()
        for t in tiles:
            gs, gsc = g.tile(codes, scales, *t)
            rs, rsc = ref.state[t]
            assert np.array_equal(gs, rs) and np.array_equal(gsc, rsc), t
            ro = out[t]
            assert np.linalg.norm(o[t] - ro) <= 1e-5 * np.linalg.norm(ro), t
    finally:
        g.close()


def test_injection_arguments_are_checked():
    L = lib()
    h = L.lores_create(2, 2, 128, 64)
    try:
        with pytest.raises(L.LoresError) as e:
            L.lores_set_fault_injection(h, 2, 0, 0)          # sequence out of range
        assert e.value.status == L.LORES_ERR_INVALID_ARG
        with pytest.raises(L.LoresError) as e:
            L.lores_set_fault_injection(h, 0, 10 ** 6, 0)    # unit out of range
        assert e.value.status == L.LORES_ERR_INVALID_ARG
        L.lores_set_fault_injection(h, -1, 0, 0)
    finally:
        L.lores_destroy(h)
