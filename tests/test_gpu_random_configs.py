"""Randomised configurations against the oracle: key width, value rows, group width, per-head
widths (fp32, 4..8 bits, dense planes), delta, decay kind, rounding, batch and heads drawn
from a seeded generator; every tile compared at every step (codes and scales bit-exact,
o within rel-L2 1e-5)."""
import numpy as np
import pytest
import torch

from bit_recurrent_state_lores_b200 import synth

from .harness import GpuRun, OracleTiles, assert_parity, host_tile_inputs, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def draw_config(seed):
    g = np.random.default_rng(seed)
    d_k = int(g.choice([16, 32, 64, 128, 256]))
    d_v = int(4 * g.integers(1, 40))
    groups = [G for G in (16, 32, 64, 128, 256) if G <= d_k]
    G = int(g.choice(groups))
    H = int(g.integers(1, 5))
    B = int(g.integers(1, 4))
    dense = int(g.integers(0, 2))
    bits = [int(g.choice([4, 5, 6, 7, 8, 8, 32])) for _ in range(H)]
    diag = int(g.integers(0, 2))
    return dict(d_k=d_k, d_v=d_v, G=G, H=H, B=B, bits=bits, dense=dense, diag=diag,
                delta=int(g.integers(0, 2)), sr=int(g.integers(0, 2)),
                outliers=int(g.integers(0, 3)))


@pytest.mark.parametrize("seed", list(range(12)))
def test_random_configuration_matches_oracle(seed):
    c = draw_config(1000 + seed)
    wl = synth.Workload("rand", B=c["B"], H=c["H"], d_k=c["d_k"], d_v=c["d_v"], steps=3,
                        delta=c["delta"], diag=c["diag"], group=c["G"],
                        decay="kda" if c["diag"] else "tau",
                        outliers=min(c["outliers"], c["d_v"]), seed=seed)
    hp = synth.head_params(wl)
    tiles = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    g = GpuRun(wl, c["bits"], seed=seed, stochastic=c["sr"], dense=c["dense"])
    ref = OracleTiles(wl, c["bits"], seed, tiles, stochastic=c["sr"], dense=c["dense"])
    for step in range(3):
        inp = synth.step_inputs(wl, step, hp, device="cuda")
        o = g.step(inp, step).cpu().numpy()
        oref, flags = ref.step(host_tile_inputs(inp, tiles), step)
        codes, scales = g.export()
        for t in tiles:
            assert flags[t] == 0
            assert rel_l2(o[t], oref[t]) <= 1e-5, (c, step, t)
            gs, gsc = g.tile(codes, scales, *t)
            rs, rsc = ref.state[t]
            if c["bits"][t[1]] == 32:
                assert np.array_equal(gs, rs), (c, step, t)
                continue
            assert np.array_equal(gs, rs) and np.array_equal(gsc, rsc), (c, step, t)
    assert g.check() == 0
    g.close()
