"""GPU <-> oracle parity of dense 5- to 7-bit codes (dense_codes = 1): offset-binary codes
in 4-, 2- and 1-bit planes instead of one byte per code (the pages' INT5 / INT6 states at
their own bit widths).  Codes and scales bit-exact on every tile and step."""
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


def run_dense(wl, bits, seed, steps, stochastic=1, t0=0):
    hp = synth.head_params(wl)
    tiles = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    g = GpuRun(wl, bits, seed, stochastic=stochastic, dense=1)
    ref = OracleTiles(wl, bits, seed, tiles, stochastic=stochastic, dense=1)
    for n in range(steps):
        step = t0 + n
        inp = synth.step_inputs(wl, step, hp, device="cuda")
        o = g.step(inp, step).cpu().numpy()
        oref, flags = ref.step(host_tile_inputs(inp, tiles), step)
        codes, scales = g.export()
        for t in tiles:
            assert flags[t] == 0
            assert rel_l2(o[t], oref[t]) <= 1e-5, (step, t)
            gs, gsc = g.tile(codes, scales, *t)
            rs, rsc = ref.state[t]
            if bits[t[1]] == 32:
                assert np.array_equal(gs, rs)
                continue
            assert np.array_equal(gs, rs), f"step {step} tile {t}: dense bytes differ"
            assert np.array_equal(gsc, rsc)
    assert g.check() == lib().LORES_OK
    return g


CASES = [
    # d_k, d_v, G, bits, delta, diag, sr, B
    (16, 20, 16, [6, 5, 7], 1, 0, 1, 2),
    (32, 36, 16, [5, 7, 8], 1, 1, 1, 2),
    (64, 44, 32, [6, 4, 32], 0, 1, 1, 2),
    (128, 64, 128, [7, 6, 5], 1, 0, 0, 2),     # round to nearest
    (128, 128, 32, [6, 6, 8], 1, 1, 1, 3),
    (256, 32, 64, [5, 6, 7], 1, 0, 1, 2),
]


@pytest.mark.parametrize("d_k,d_v,G,bits,delta,diag,sr,B", CASES)
def test_dense_small_shapes_bit_exact(d_k, d_v, G, bits, delta, diag, sr, B):
    wl = synth.Workload("dense", B=B, H=len(bits), d_k=d_k, d_v=d_v, steps=4, delta=delta,
                        diag=diag, group=G, decay="kda" if diag else "tau", outliers=2, seed=31)
    g = run_dense(wl, bits, seed=4, steps=4, stochastic=sr)
    lay = g.layout
    rowb = [d_k * 4 if b == 32 else (d_k // 2 if b == 4 else
            (d_k if b == 8 else (d_k * b // 8 + 7) // 8 * 8)) for b in bits]
    assert lay.code_bytes == B * d_v * sum(rowb)
    g.close()


def test_dense_load_dequant_resume_and_tokens():
    L = lib()
    wl = synth.Workload("dense-load", B=2, H=3, d_k=64, d_v=40, steps=6, delta=1, diag=1,
                        group=16, decay="kda", outliers=2, seed=12)
    bits = [5, 6, 7]
    g = GpuRun(wl, bits, seed=8, dense=1)
    S = (torch.randn(wl.B, wl.H, wl.d_v, wl.d_k, device="cuda") *
         torch.exp(torch.randn(wl.B, wl.H, wl.d_v, 1, device="cuda")))
    L.lores_load_state(g.h, S, 3)
    codes, scales = g.export()
    Sh = S.cpu().numpy()
    sk = O.step_key(8, 3)
    Sd = g.dequant().cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.H):
            cfg = tile_cfg(wl, bits[h], dense=1)
            gs, gsc = g.tile(codes, scales, b, h)
            rc, rs, _ = O.tile_quantize(cfg, Sh[b, h], O.tile_key(sk, b * wl.H + h))
            assert np.array_equal(gs, rc) and np.array_equal(gsc, rs), (b, h)
            assert np.array_equal(Sd[b, h], O.tile_dequant(cfg, rc, rs))
    hp = synth.head_params(wl)
    g2 = GpuRun(wl, bits, seed=8, dense=1)
    g2.load(codes, scales)
    T = 4
    toks = [synth.step_inputs(wl, 10 + t, hp, device="cuda") for t in range(T)]
    st = [torch.stack([tok[i] for tok in toks]).contiguous() for i in range(5)]
    o2 = torch.empty(T, wl.B, wl.H, wl.d_v, device="cuda")
    L.lores_decode_steps(g2.h, T, *st, o2, 10)
    for t in range(T):
        g.step(toks[t], 10 + t)
        assert torch.equal(g.o, o2[t])
    a, b = g.export(), g2.export()
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    g.close()
    g2.close()


def test_dense_six_bit_state_is_three_quarters_of_int8():
    wl = synth.Workload("dense-size", B=4, H=2, d_k=128, d_v=128, steps=1, group=128, seed=1)
    a = GpuRun(wl, [6, 6], seed=1, dense=1)
    b = GpuRun(wl, [6, 6], seed=1, dense=0)
    assert a.layout.code_bytes * 4 == b.layout.code_bytes * 3
    a.close()
    b.close()
