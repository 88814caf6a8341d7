"""GPU <-> oracle parity of per-channel precision: a bit width per (head, key group), the
abstract's decay-based mixed precision applied over channels.  Rows store their key groups
back to back at their own widths; every group is scaled with its own r.  Small shapes are
bit-exact on every tile and step; the channel-decay workload takes its widths from the
library's decay policy over (head, group) mean decays."""
import numpy as np
import pytest
import torch

from bit_recurrent_state_lores_b200 import synth
from oracle import oracle as O

from .harness import (GpuRun, OracleTiles, assert_parity, host_tile_inputs, rel_l2,
                      sample_tiles, tile_cfg)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def lib():
    from bit_recurrent_state_lores_b200 import lores
    return lores


def random_group_bits(H, ng, seed, uniform_heads=(0,)):
    g = np.random.default_rng(seed)
    out = []
    for h in range(H):
        if h in uniform_heads:
            out.append([int(g.integers(4, 9))] * ng)
        else:
            row = [int(b) for b in g.integers(4, 9, ng)]
            if len(set(row)) == 1 and ng > 1:
                row[-1] = 4 if row[0] != 4 else 8
            out.append(row)
    return out


def run_free(wl, gb, seed, tiles, steps, stochastic=1, exact=True, t0=0):
    hp = synth.head_params(wl)
    nominal = [8] * wl.H
    g = GpuRun(wl, nominal, seed, stochastic=stochastic, group_bits=gb)
    ref = OracleTiles(wl, nominal, seed, tiles, stochastic=stochastic, group_bits=gb)
    bi = torch.tensor([t[0] for t in tiles])
    hi = torch.tensor([t[1] for t in tiles])
    for n in range(steps):
        step = t0 + n
        inp = synth.step_inputs(wl, step, hp, device="cuda")
        o = g.step(inp, step)[bi, hi].cpu().numpy()
        oref, flags = ref.step(host_tile_inputs(inp, tiles), step)
        codes, scales = g.export()
        for m, t in enumerate(tiles):
            assert flags[t] == 0
            r = rel_l2(o[m], oref[t])
            assert r <= 1e-5, f"step {step} tile {t}: o rel-L2 {r}"
            gs, gsc = g.tile(codes, scales, *t)
            rs, rsc = ref.state[t]
            nd = assert_parity(ref.cfg[t], gs, gsc, rs, rsc, f"step {step} tile {t}")
            if exact:
                assert nd == 0 and np.array_equal(gsc, rsc), f"step {step} tile {t} not exact"
    assert g.check() == lib().LORES_OK
    return g


CASES = [
    # d_k, d_v, G, delta, diag, sr, B, H
    (64, 36, 16, 1, 1, 1, 2, 3),
    (64, 40, 32, 0, 1, 1, 2, 3),
    (128, 64, 32, 1, 0, 0, 2, 3),       # round to nearest
    (128, 52, 16, 1, 1, 1, 2, 2),
    (256, 32, 64, 1, 0, 1, 2, 2),
    (32, 100, 16, 1, 1, 1, 2, 3),
]


@pytest.mark.parametrize("d_k,d_v,G,delta,diag,sr,B,H", CASES)
def test_group_bits_small_shapes_bit_exact(d_k, d_v, G, delta, diag, sr, B, H):
    wl = synth.Workload("chan", B=B, H=H, d_k=d_k, d_v=d_v, steps=4, delta=delta, diag=diag,
                        group=G, decay="kda" if diag else "tau", outliers=2, seed=13)
    gb = random_group_bits(H, d_k // G, seed=d_k + d_v + G)
    tiles = [(b, h) for b in range(B) for h in range(H)]
    g = run_free(wl, gb, seed=7, tiles=tiles, steps=4, stochastic=sr)
    lay, offs = lib().lores_get_layout(g.h, H)
    rowb = [sum(G * (4 if b == 4 else 8) // 8 for b in gb[h]) for h in range(H)]
    assert lay.code_bytes == B * d_v * sum(rowb)
    assert list(offs) == [d_v * sum(rowb[:h]) for h in range(H)]
    g.close()


def test_group_bits_load_state_dequant_resume_and_tokens():
    L = lib()
    wl = synth.Workload("chan-load", B=2, H=3, d_k=64, d_v=24, steps=6, delta=1, diag=1,
                        group=16, decay="kda", outliers=2, seed=4)
    gb = random_group_bits(3, 4, seed=99)
    nominal = [8] * 3
    g = GpuRun(wl, nominal, seed=8, group_bits=gb)
    S = (torch.randn(wl.B, wl.H, wl.d_v, wl.d_k, device="cuda") *
         torch.exp(torch.randn(wl.B, wl.H, wl.d_v, 1, device="cuda")))
    L.lores_load_state(g.h, S, 31)
    codes, scales = g.export()
    Sh = S.cpu().numpy()
    sk = O.step_key(8, 31)
    Sd = g.dequant().cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.H):
            cfg = tile_cfg(wl, 8, group_bits=gb[h])
            gs, gsc = g.tile(codes, scales, b, h)
            rc, rs, _ = O.tile_quantize(cfg, Sh[b, h], O.tile_key(sk, b * wl.H + h))
            assert np.array_equal(gs, rc) and np.array_equal(gsc, rs), (b, h)
            assert np.array_equal(Sd[b, h], O.tile_dequant(cfg, rc, rs))
    # a restored handle and a multi-token call follow the single steps bit for bit
    hp = synth.head_params(wl)
    g2 = GpuRun(wl, nominal, seed=8, group_bits=gb)
    g2.load(codes, scales)
    T = 3
    toks = [synth.step_inputs(wl, 40 + t, hp, device="cuda") for t in range(T)]
    st = [torch.stack([tok[i] for tok in toks]).contiguous() for i in range(5)]
    o2 = torch.empty(T, wl.B, wl.H, wl.d_v, device="cuda")
    L.lores_decode_steps(g2.h, T, *st, o2, 40)
    for t in range(T):
        g.step(toks[t], 40 + t)
        assert torch.equal(g.o, o2[t])
    a, b = g.export(), g2.export()
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    g.close()
    g2.close()


def test_channel_decay_policy_workload_sampled_tiles():
    # KDA-style per-channel decays; the slowest 25 % of (head, key group) pairs by mean
    # decay get 8 bits, the rest 4 (the library's policy over flattened groups)
    L = lib()
    wl = synth.Workload("kda-chan", B=16, H=8, d_k=128, d_v=128, steps=12, delta=1, diag=1,
                        group=32, decay="kda_channel", outliers=4, seed=3)
    hp = synth.head_params(wl)
    ng = wl.d_k // wl.G
    gmean = hp["mean_decay_channel"].reshape(wl.H, ng, wl.G).mean(axis=2)
    flat = L.lores_assign_bits_by_decay(gmean.reshape(-1), 0.25, 8, 4)
    gb = [list(flat[h * ng:(h + 1) * ng]) for h in range(wl.H)]
    assert sum(b == 8 for b in flat) == round(0.25 * wl.H * ng)
    assert any(len(set(row)) > 1 for row in gb)
    tiles = [(0, 0), (15, 7), (3, 2), (9, 5), (12, 1)]
    g = run_free(wl, gb, seed=2, tiles=tiles, steps=wl.steps, exact=False)
    g.close()

