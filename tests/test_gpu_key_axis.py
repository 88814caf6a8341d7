"""GPU <-> oracle parity of key-axis scale grouping (one scale per key column of a tile),
the comparator that the LoReS paper's Scale Grouping paragraph sets against value-axis
groups.  Same bounds as the value-axis tests: codes and scales bit-exact on the small
shapes, o_t within rel-L2 1e-5."""
import numpy as np
import pytest
import torch

from bit_recurrent_state_lores_b200 import synth
from oracle import oracle as O

from .harness import GpuRun, OracleTiles, assert_parity, host_tile_inputs, rel_l2, tile_cfg

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def lib():
    from bit_recurrent_state_lores_b200 import lores
    return lores


def run_key(wl, bits, seed, tiles, steps, stochastic=1, exact=True, inject=None):
    hp = synth.head_params(wl)
    g = GpuRun(wl, bits, seed, stochastic=stochastic, axis=1)
    ref = OracleTiles(wl, bits, seed, tiles, stochastic=stochastic, axis=1)
    bi = torch.tensor([t[0] for t in tiles])
    hi = torch.tensor([t[1] for t in tiles])
    any_flag = False
    for step in range(steps):
        inp = list(synth.step_inputs(wl, step, hp, device="cuda"))
        if inject is not None:
            inject(step, inp)
        o = g.step(inp, step)[bi, hi].cpu().numpy()
        oref, flags = ref.step(host_tile_inputs(inp, tiles), step)
        any_flag |= any(flags.values())
        # the status reports (and clears) the flag of this step; quantized heads zero their
        # bad columns, so it does not carry over unless an fp32 head keeps a bad entry
        if len(tiles) == wl.B * wl.H:
            want = lib().LORES_ERR_NONFINITE if any(flags.values()) else lib().LORES_OK
            assert g.check() == want, (step, flags)
        codes, scales = g.export()
        for m, t in enumerate(tiles):
            gs, gsc = g.tile(codes, scales, *t)
            rs, rsc = ref.state[t]
            cfg = ref.cfg[t]
            if flags[t] == 0:
                r = rel_l2(o[m], oref[t])
                assert r <= 1e-5, f"step {step} tile {t}: o rel-L2 {r}"
            if cfg.bits == 32:
                if flags[t] == 0:
                    assert np.array_equal(gs, rs), (step, t)
                continue
            nd = assert_parity(cfg, gs, gsc, rs, rsc, f"step {step} tile {t}")
            if exact:
                assert nd == 0 and np.array_equal(gsc, rsc), f"step {step} tile {t} not exact"
    return g, any_flag


KEY_SWEEP = [
    # d_k, d_v, bits, delta, diag, sr, B, H
    (16, 16, [8, 4], 1, 0, 1, 2, 2),
    (32, 36, [8, 6], 0, 1, 1, 2, 2),
    (64, 100, [4, 8, 32], 1, 1, 1, 2, 3),
    (128, 52, [8, 5, 4], 1, 0, 0, 2, 3),      # round to nearest
    (128, 128, [8, 7, 32], 1, 1, 1, 2, 3),
    (256, 64, [8, 4], 1, 0, 1, 2, 2),
    (64, 512, [8, 4], 1, 1, 1, 2, 2),         # tall tile: the two-pass recompute kernel
    (32, 4, [8, 4], 1, 0, 1, 3, 2),           # four rows
    (128, 256, [32, 8], 1, 0, 1, 2, 2),       # 128 KB fp32 tile: one shared-memory stage
]


@pytest.mark.parametrize("d_k,d_v,bits,delta,diag,sr,B,H", KEY_SWEEP)
def test_key_axis_small_shapes_bit_exact(d_k, d_v, bits, delta, diag, sr, B, H):
    wl = synth.Workload("key", B=B, H=H, d_k=d_k, d_v=d_v, steps=5, delta=delta, diag=diag,
                        group=d_k, decay="kda" if diag else "tau", outliers=2, seed=11)
    tiles = [(b, h) for b in range(B) for h in range(H)]
    g, flagged = run_key(wl, bits, seed=5, tiles=tiles, steps=5, stochastic=sr)
    assert not flagged
    assert g.layout.n_groups == 0 and g.layout.scale_count == B * H * d_k
    g.close()


def test_key_axis_nonfinite_column_zeroed_and_flagged():
    # a NaN decay entry alpha_j (diagonal decay, no delta term) poisons one key column only
    wl = synth.Workload("keynan", B=2, H=3, d_k=64, d_v=32, steps=3, delta=0, diag=1,
                        group=64, decay="kda", outliers=0, seed=3)
    bits = [8, 4, 32]

    def inject(step, inp):
        if step == 1:
            inp[3] = inp[3].clone()
            inp[3][1, 0, 9] = float("nan")        # column 9 of tile (1, 0)
            inp[3][0, 1, 40] = float("inf")       # column 40 of tile (0, 1)

    tiles = [(b, h) for b in range(2) for h in range(3)]
    g, flagged = run_key(wl, bits, seed=9, tiles=tiles, steps=3, inject=inject)
    assert flagged
    g.close()


def test_key_axis_load_state_dequant_and_resume():
    L = lib()
    wl = synth.Workload("keyload", B=2, H=3, d_k=128, d_v=48, steps=4, delta=1, diag=1,
                        group=128, decay="kda", outliers=2, seed=4)
    bits = [8, 4, 32]
    g = GpuRun(wl, bits, seed=8, axis=1)
    S = (torch.randn(wl.B, wl.H, wl.d_v, wl.d_k, device="cuda") *
         torch.exp(torch.randn(wl.B, wl.H, 1, wl.d_k, device="cuda")))
    L.lores_load_state(g.h, S, 17)
    codes, scales = g.export()
    Sh = S.cpu().numpy()
    sk = O.step_key(8, 17)
    Sd = g.dequant().cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.H):
            cfg = tile_cfg(wl, bits[h], axis=1)
            gs, gsc = g.tile(codes, scales, b, h)
            if bits[h] == 32:
                assert np.array_equal(gs, Sh[b, h])
                assert np.array_equal(Sd[b, h], Sh[b, h])
                continue
            rc, rs, _ = O.tile_quantize(cfg, Sh[b, h], O.tile_key(sk, b * wl.H + h))
            assert np.array_equal(gs, rc) and np.array_equal(gsc, rs)
            assert np.array_equal(Sd[b, h], O.tile_dequant(cfg, rc, rs))
    # a second handle restored from the export follows the same trajectory bit for bit
    hp = synth.head_params(wl)
    g2 = GpuRun(wl, bits, seed=8, axis=1)
    g2.load(codes, scales)
    for t in range(3):
        inp = synth.step_inputs(wl, t, hp, device="cuda")
        g.step(inp, 20 + t)
        g2.step(inp, 20 + t)
        assert torch.equal(g.o, g2.o)
    a, b = g.export(), g2.export()
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    g.close()
    g2.close()


def test_key_axis_gdn_shape_sampled_tiles():
    # 128 x 128 int8 tiles with outlier rows, 16 steps, sampled tiles free-running
    wl = synth.Workload("keygdn", B=16, H=8, d_k=128, d_v=128, steps=16, delta=1, diag=0,
                        group=128, decay="tau", outliers=4, seed=2)
    tiles = [(0, 0), (15, 7), (5, 3), (9, 6)]
    g, flagged = run_key(wl, [8] * 8, seed=1, tiles=tiles, steps=16, exact=False)
    assert not flagged and g.check() == lib().LORES_OK
    g.close()

