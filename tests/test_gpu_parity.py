"""GPU <-> oracle parity through the C ABI, on the seeded synthetic workloads.

Acceptance bounds: o_t and the dequantized state within
rel-L2 1e-5; codes equal except at most 1e-4 of entries at +-1 (the arithmetic is
specified down to the fp32 rounding of every step, so codes are expected to match
exactly, and the small shapes assert that); packing and scale indexing bit-exact.

Small shapes compare every tile at every step.  The full-size workloads compare
sampled tiles free-running over the whole trajectory (tiles are independent, so the
oracle can follow a few of them exactly) and every tile on one teacher-forced step
(the oracle starts from the GPU's exported state).
"""
import numpy as np
import pytest
import torch

from bit_recurrent_state_lores_b200 import synth
from oracle import oracle as O

from .harness import (GpuRun, OracleTiles, assert_parity, host_tile_inputs, lib, mixed_bits,
                      rel_l2, sample_tiles, tile_cfg, unpack_fast)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def run_free(wl, head_bits, seed, tiles, steps, check_every=1, start_state=None, step0=0,
             stochastic=1, exact=False):
    """Run `steps` steps on GPU and oracle, compare o every step and the state every
    `check_every` steps on `tiles`.  Returns the GpuRun (open)."""
    hp = synth.head_params(wl)
    g = GpuRun(wl, head_bits, seed, stochastic=stochastic)
    ref = OracleTiles(wl, head_bits, seed, tiles, stochastic=stochastic)
    if start_state is not None:
        g.load(*start_state)
        codes, scales = start_state
        for t in tiles:
            ref.load(t, *g.tile(codes, scales, *t))
    bi = torch.tensor([t[0] for t in tiles])
    hi = torch.tensor([t[1] for t in tiles])
    for n in range(steps):
        step = step0 + n
        inp = synth.step_inputs(wl, step, hp, device="cuda")
        o = g.step(inp, step)
        og = o[bi, hi].cpu().numpy()
        oref, flags = ref.step(host_tile_inputs(inp, tiles), step)
        for m, t in enumerate(tiles):
            assert flags[t] == 0
            r = rel_l2(og[m], oref[t])
            assert r <= 1e-5, f"step {step} tile {t}: o rel-L2 {r}"
        if (n + 1) % check_every == 0 or n == steps - 1:
            codes, scales = g.export()
            for t in tiles:
                gs, gsc = g.tile(codes, scales, *t)
                rs, rsc = ref.state[t]
                nd = assert_parity(ref.cfg[t], gs, gsc, rs, rsc, f"step {step} tile {t}")
                if exact:
                    assert nd == 0 and (gsc == rsc).all(), f"step {step} tile {t} not exact"
    assert g.check() == 0
    return g


def teacher_forced_all(g, wl, head_bits, seed, step, stochastic=1):
    """One GPU step from its current state versus the oracle on every tile."""
    hp = synth.head_params(wl)
    codes0, scales0 = g.export()
    inp = synth.step_inputs(wl, step, hp, device="cuda")
    o = g.step(inp, step).cpu().numpy()
    codes1, scales1 = g.export()
    q, k, v, a, b = [x.cpu().numpy() for x in inp]
    sk = O.step_key(seed, step)
    worst_o, ndiff = 0.0, 0
    for bb in range(wl.B):
        for hh in range(wl.H):
            cfg = tile_cfg(wl, head_bits[hh], stochastic)
            st, sc = g.tile(codes0, scales0, bb, hh)
            oo, flag, _ = O.tile_step(cfg, st, sc, q[bb, hh], k[bb, hh], v[bb, hh], a[bb, hh],
                                      b[bb, hh], O.tile_key(sk, bb * wl.H + hh))
            assert flag == 0
            worst_o = max(worst_o, rel_l2(o[bb, hh], oo))
            gs, gsc = g.tile(codes1, scales1, bb, hh)
            if cfg.bits == 32:
                assert rel_l2(gs, st) <= 1e-5
                continue
            if not (np.array_equal(gs, st) and np.array_equal(gsc, sc)):
                ndiff += assert_parity(cfg, gs, gsc, st, sc, f"tile {(bb, hh)}")
    assert worst_o <= 1e-5, worst_o
    total = wl.B * wl.H * wl.d_v * wl.d_k
    assert ndiff <= 1e-4 * total
    return ndiff


# ---------------------------------------------------------------------------------------
# tiny oracle case: every tile, every step, bit-exact
# ---------------------------------------------------------------------------------------

def test_tiny_config_bit_exact_every_step():
    wl = synth.workload("tiny")
    bits = [8] * wl.H
    g = run_free(wl, bits, seed=0, tiles=[(0, 0), (0, 1)], steps=wl.steps, exact=True)
    g.close()


# ---------------------------------------------------------------------------------------
# shape / mode sweep on small sizes: every tile, every step
# ---------------------------------------------------------------------------------------

SWEEP = [
    # d_k, d_v, G, bits, delta, diag, sr, B, H
    (16, 16, 16, "8", 1, 0, 1, 3, 2),
    (16, 20, 16, "4", 0, 1, 1, 2, 3),       # ragged d_v: a warp pass spans tiles
    (32, 36, 16, "8", 1, 1, 1, 2, 2),
    (32, 12, 32, "mix", 1, 0, 0, 3, 3),     # round to nearest
    (64, 100, 32, "4", 1, 1, 1, 2, 2),
    (64, 64, 64, "mix", 0, 0, 1, 2, 4),
    (128, 52, 32, "8", 1, 0, 1, 2, 2),
    (128, 128, 16, "mix", 1, 1, 1, 2, 3),
    (128, 64, 128, "32", 1, 1, 1, 2, 2),
    (256, 24, 256, "8", 1, 0, 1, 1, 2),
    (256, 40, 16, "mix", 1, 1, 1, 2, 3),
    (256, 16, 64, "4", 0, 0, 0, 2, 2),
    (128, 64, 32, "b5678", 1, 1, 1, 2, 6),  # 5-, 6-, 7-bit codes (one byte each) with 8/4/32
    (64, 36, 16, "b5678", 0, 0, 0, 2, 6),
]


@pytest.mark.parametrize("d_k,d_v,G,bits,delta,diag,sr,B,H", SWEEP)
def test_small_shapes_every_tile_every_step(d_k, d_v, G, bits, delta, diag, sr, B, H):
    wl = synth.Workload("small", B=B, H=H, d_k=d_k, d_v=d_v, steps=10, delta=delta, diag=diag,
                        group=G, decay="kda" if diag else "tau", outliers=min(2, d_v), seed=d_k + d_v)
    if bits == "mix":
        hb = [(8, 4, 32)[h % 3] for h in range(H)]
    elif bits == "b5678":
        hb = [(6, 5, 8, 4, 7, 32)[h % 6] for h in range(H)]
    else:
        hb = [int(bits)] * H
    tiles = [(b, h) for b in range(B) for h in range(H)]
    g = run_free(wl, hb, seed=1234 + d_k, tiles=tiles, steps=wl.steps, stochastic=sr, exact=True)
    # dequant kernel against the oracle's dequantization
    S = g.dequant().cpu().numpy()
    codes, scales = g.export()
    for (b, h) in tiles:
        st, sc = g.tile(codes, scales, b, h)
        cfg = tile_cfg(wl, hb[h], sr)
        ref = st if cfg.bits == 32 else O.tile_dequant(cfg, st, sc)
        assert np.array_equal(S[b, h], ref)
    g.close()


def test_row_split_small_batch_matches():
    # batch 1 with many rows: the library splits rows across CTAs to fill the GPU
    wl = synth.Workload("split", B=1, H=2, d_k=128, d_v=512, steps=4, decay="tau", seed=9)
    g = run_free(wl, [8, 4], seed=5, tiles=[(0, 0), (0, 1)], steps=4, exact=True)
    assert g.layout.units_per_step > 2
    g.close()


# ---------------------------------------------------------------------------------------
# full-size workloads
# ---------------------------------------------------------------------------------------

def fp32_warmup(wl, seed, steps):
    """fp32 warmup on GPU (fp32 heads) -> dequantized fp32 state on device."""
    g = GpuRun(wl, [32] * wl.H, seed)
    hp = synth.head_params(wl)
    for t in range(steps):
        g.step(synth.step_inputs(wl, t, hp, device="cuda"), t)
    S = g.dequant()
    codes, scales = g.export()
    return g, S, codes


def test_gdn_shaped_with_fp32_warmup():
    wl = synth.workload("gdn")
    bits = [8] * wl.H
    seed = 2
    tiles = sample_tiles(wl, bits, 6)
    # GPU: 64-step fp32 warmup, then quantize with the dither of step 63
    gw, S, wcodes = fp32_warmup(wl, seed, wl.warmup)
    g = GpuRun(wl, bits, seed)
    from bit_recurrent_state_lores_b200 import lores as L
    L.lores_load_state(g.h, S, wl.warmup - 1)
    torch.cuda.synchronize()
    codes, scales = g.export()
    # oracle: its own fp32 warmup of the sampled tiles, then the same quantizer
    ref32 = OracleTiles(wl, [32] * wl.H, seed, tiles)
    hp = synth.head_params(wl)
    for t in range(wl.warmup):
        ref32.step(host_tile_inputs(synth.step_inputs(wl, t, hp, device="cuda"), tiles), t)
    sk = O.step_key(seed, wl.warmup - 1)
    for t in tiles:
        Sref = ref32.state[t][0]
        Sgpu, _ = gw.tile(wcodes, np.zeros((wl.B, wl.H, wl.d_v, 1), np.float32), *t)
        assert rel_l2(Sgpu, Sref) <= 1e-6, "fp32 warmup diverged"
        cfg = tile_cfg(wl, 8)
        rc, rs, _ = O.tile_quantize(cfg, Sref, O.tile_key(sk, t[0] * wl.H + t[1]))
        gc, gs = g.tile(codes, scales, *t)
        assert_parity(cfg, gc, gs, rc, rs, f"load_state tile {t}")
    gw.close()
    g.close()
    # 256 quantized steps free-running from the loaded state, then one full-coverage step
    g = run_free(wl, bits, seed, tiles, wl.steps, check_every=64, start_state=(codes, scales),
                 step0=wl.warmup)
    teacher_forced_all(g, wl, bits, seed, wl.warmup + wl.steps)
    g.close()


def test_mamba2_shaped():
    wl = synth.workload("mamba2")
    bits = [8] * wl.H
    tiles = sample_tiles(wl, bits, 6)
    g = run_free(wl, bits, 3, tiles, wl.steps, check_every=128)
    teacher_forced_all(g, wl, bits, 3, wl.steps)
    g.close()


def test_kda_shaped_mixed_precision():
    wl = synth.workload("kda")
    hp = synth.head_params(wl)
    bits = mixed_bits(wl, hp)
    assert bits.count(8) == 8 and bits.count(4) == 24
    # the promoted heads are the slowest-decaying ones
    md = hp["mean_decay"]
    assert min(md[h] for h in range(wl.H) if bits[h] == 8) > max(
        md[h] for h in range(wl.H) if bits[h] == 4)
    tiles = sample_tiles(wl, bits, 6)
    g = run_free(wl, bits, 4, tiles, wl.steps, check_every=256)
    teacher_forced_all(g, wl, bits, 4, wl.steps)
    g.close()


@pytest.mark.parametrize("variant", ["int8", "mixed", "fp32"])
def test_sweep_layers_in_bench_launch_configuration(variant):
    # The 48-layer sweep point the benchmark times (batch 256, int8), plus the mixed and
    # fp32-state variants at smaller batch.  Sampled (layer, tile) pairs follow the oracle.
    B = {"int8": 256, "mixed": 64, "fp32": 16}[variant]
    wl = synth.workload("sweep", B=B)
    layers = [0, 23, 47]
    steps = 6
    for layer in layers:
        wll = synth.replace(wl, seed=wl.seed * 1000 + layer)
        hp = synth.head_params(wll)
        if variant == "int8":
            bits = [8] * wl.H
        elif variant == "mixed":
            bits = mixed_bits(synth.replace(wll, mixed_frac=0.25), hp)
        else:
            bits = [32] * wl.H
        tiles = sample_tiles(wll, bits, 4, seed=layer)
        g = run_free(wll, bits, 77 + layer, tiles, steps, check_every=3)
        g.close()


# ---------------------------------------------------------------------------------------
# maximum sizes and degenerate inputs
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [[8], [4], [32], [6]])
def test_largest_tile_every_step(bits):
    # the largest tile the library takes: d_k = 256, d_v = 4096 (units split the rows)
    wl = synth.Workload("max", B=1, H=1, d_k=256, d_v=4096, steps=3, delta=1, diag=1,
                        group=64, decay="kda", outliers=4, seed=21)
    g = run_free(wl, bits, seed=3, tiles=[(0, 0)], steps=3, exact=True)
    g.close()


def test_degenerate_inputs_match_oracle():
    # alpha = 1 (no forgetting), beta = 0 (no write), k = q = 0 on some heads, a zero value
    # row: every tile at every step equals the oracle, and nothing is flagged
    wl = synth.Workload("degen", B=2, H=4, d_k=64, d_v=32, steps=4, delta=1, diag=0,
                        group=32, decay="tau", outliers=0, seed=5)
    bits = [8, 4, 6, 32]
    hp = synth.head_params(wl)
    g = GpuRun(wl, bits, seed=9)
    tiles = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    ref = OracleTiles(wl, bits, 9, tiles)
    for step in range(wl.steps):
        q, k, v, a, b = [x.clone() for x in synth.step_inputs(wl, step, hp, device="cuda")]
        a[:, 0] = 1.0                        # head 0: no decay
        b[:, 1] = 0.0                        # head 1: no write (pure decay)
        if step >= 2:
            k[:, 2] = 0.0                    # head 2: k = q = 0 (decay only; readout 0)
            q[:, 2] = 0.0
        v[0, 3, 5] = 0.0
        inp = (q, k, v, a, b)
        o = g.step(inp, step).cpu().numpy()
        oref, flags = ref.step(host_tile_inputs(inp, tiles), step)
        codes, scales = g.export()
        for t in tiles:
            assert flags[t] == 0
            assert rel_l2(o[t], oref[t]) <= 1e-5 or np.abs(o[t] - oref[t]).max() <= 1e-12
            gs, gsc = g.tile(codes, scales, *t)
            rs, rsc = ref.state[t]
            if bits[t[1]] == 32:
                assert np.array_equal(gs, rs)
                continue
            assert assert_parity(ref.cfg[t], gs, gsc, rs, rsc, f"{step} {t}") == 0
            assert np.array_equal(gsc, rsc)
    assert g.check() == lib_ok()
    g.close()


def lib_ok():
    from bit_recurrent_state_lores_b200 import lores
    return lores.LORES_OK


@pytest.mark.parametrize("name,B", [("gdn", 96), ("mamba2", 24), ("kda", 96)])
def test_gpu_step_within_bounds_of_the_plain_definition(name, B):
    """The GPU step against the oracle's plain-definition step (double precision, IEEE
    division, floor of x r/m + (d + 1/2)/256), teacher-forced from the GPU's state on
    sampled tiles over several steps: codes at +-1 on <= 1e-4 of the entries, the
    dequantized state of entries with equal codes and the readout within rel-L2 1e-5.
    (The bit-exact tests above compare with the evaluated step; this one ties the GPU
    to the definition itself.)"""
    wl = synth.workload(name, B=B)
    hp = synth.head_params(wl)
    bits = mixed_bits(wl, hp)
    seed = 17
    g = GpuRun(wl, bits, seed)
    tiles = sample_tiles(wl, bits, 12, seed=3)
    bi = torch.tensor([t[0] for t in tiles])
    hi = torch.tensor([t[1] for t in tiles])
    n_diff = n_total = 0
    try:
        for step in range(5):
            codes, scales = g.export()
            before = {t: g.tile(codes, scales, *t) for t in tiles}
            inp = synth.step_inputs(wl, step, hp, device="cuda")
            og = g.step(inp, step)[bi, hi].cpu().numpy()
            codes, scales = g.export()
            sk = O.step_key(seed, step)
            for m, (t, (q, k, v, a, b)) in enumerate(zip(tiles, host_tile_inputs(inp, tiles))):
                cfg = tile_cfg(wl, bits[t[1]])
                st, sc = (x.copy() for x in before[t])
                o, flag, _ = O.tile_step_plain(cfg, st, sc, q, k, v, a, b,
                                               O.tile_key(sk, t[0] * wl.H + t[1]))
                assert flag == 0
                gs, gsc = g.tile(codes, scales, *t)
                cg, cr = unpack_fast(cfg, gs), unpack_fast(cfg, st)
                d = np.abs(cg - cr)
                assert d.max() <= 1, (step, t)
                n_diff += int((d != 0).sum())
                n_total += d.size
                same = d == 0
                Sg = cg * np.repeat(gsc.astype(np.float64), cfg.group, axis=1) * same
                Sr = cr * np.repeat(sc.astype(np.float64), cfg.group, axis=1) * same
                assert rel_l2(Sg, Sr) <= 1e-5, (step, t)
                assert rel_l2(og[m], o) <= 1e-5, (step, t)
        assert n_diff <= 1e-4 * n_total, (n_diff, n_total)
    finally:
        g.close()


PAIR_WIDTHS = [
    # d_k, d_v, bits, G, delta, diag, sr, B: several scales per row, handles large enough
    # that every row block is full and the batch fills the GPU, so they step with the
    # two-rows-per-lane kernel
    (32, 256, [8, 4], 16, 1, 1, 1, 600),
    (64, 128, [4, 8], 32, 0, 0, 0, 600),
    (128, 128, [8, 4], 64, 1, 0, 1, 400),
    (256, 64, [8, 4], 64, 1, 1, 1, 300),
]


@pytest.mark.parametrize("d_k,d_v,bits,G,delta,diag,sr,B", PAIR_WIDTHS)
def test_two_rows_per_lane_kernel_every_key_width(d_k, d_v, bits, G, delta, diag, sr, B):
    wl = synth.Workload("pair-width", B=B, H=len(bits), d_k=d_k, d_v=d_v, steps=4, delta=delta,
                        diag=diag, group=G, decay="kda" if diag else "tau", outliers=2, seed=13)
    tiles = sample_tiles(wl, bits, 8, seed=1)
    g = run_free(wl, bits, 21, tiles, 4, stochastic=sr, exact=True)
    try:
        assert g.layout.step_kernel == 1
    finally:
        g.close()


MMA_WIDTHS = [
    # d_k, d_v, bits, delta, diag, sr, B: one scale per row (G = d_k), so the tensor-core
    # kernel; d_v = 24 and 40 leave a last strip of 8 rows in every unit
    (16, 24, [8, 4], 1, 0, 1, 40),
    (32, 40, [4, 8], 1, 1, 1, 40),
    (64, 64, [8, 4, 4], 0, 0, 0, 300),
    (128, 128, [8, 4, 8], 1, 1, 1, 200),
    (128, 96, [4, 8], 1, 0, 0, 8),
]


def test_exact_path_at_key_width_256():
    """d_k = 256 heads with one scale per row: beyond the tensor-core kernel's widths, they
    take the general kernel's exact contractions (DP4A on the digit planes); parity with
    the oracle, bit-exact, every step."""
    bits = [8, 4]
    wl = synth.Workload("exact-256", B=96, H=len(bits), d_k=256, d_v=64, steps=4, delta=1,
                        diag=1, group=256, decay="kda", outliers=2, seed=29)
    tiles = sample_tiles(wl, bits, 8, seed=3)
    g = run_free(wl, bits, 27, tiles, 4, stochastic=1, exact=True)
    try:
        assert g.layout.step_kernel == 0
    finally:
        g.close()


@pytest.mark.parametrize("d_k,d_v,bits,delta,diag,sr,B", MMA_WIDTHS)
def test_tensor_core_kernel_every_key_width(d_k, d_v, bits, delta, diag, sr, B):
    wl = synth.Workload("mma-width", B=B, H=len(bits), d_k=d_k, d_v=d_v, steps=4, delta=delta,
                        diag=diag, group=d_k, decay="kda" if diag else "tau", outliers=2, seed=17)
    tiles = sample_tiles(wl, bits, 8, seed=2)
    g = run_free(wl, bits, 23, tiles, 4, stochastic=sr, exact=True)
    try:
        assert g.layout.step_kernel == 3
    finally:
        g.close()


@pytest.mark.parametrize("diag,delta,sr", [(0, 1, 1), (1, 1, 1), (0, 0, 0)])
def test_general_exact_path_equals_tensor_core_kernel(diag, delta, sr):
    """The exact contractions of heads with one scale per row have two implementations:
    the tensor-core kernel, and the general kernel's DP4A path, which a handle takes when it
    also holds an fp32 head.  Heads 0-3 of handle A (last head int8: tensor-core kernel)
    and of handle B (last head fp32: general kernel) get the same inputs and the same tile
    keys, so their readout and state agree bit for bit, step after step."""
    L = lib()
    wl = synth.Workload("cross", B=48, H=5, d_k=128, d_v=128, steps=4, delta=delta, diag=diag,
                        group=128, decay="kda" if diag else "tau", outliers=2, seed=31)
    hp = synth.head_params(wl)
    a = GpuRun(wl, [8, 4, 8, 4, 8], 7, stochastic=sr)
    b = GpuRun(wl, [8, 4, 8, 4, 32], 7, stochastic=sr)
    try:
        assert a.layout.step_kernel == 3 and b.layout.step_kernel == 0
        for t in range(wl.steps):
            inp = synth.step_inputs(wl, t, hp, device="cuda")
            oa = a.step(inp, t).clone()
            ob = b.step(inp, t)
            assert torch.equal(oa[:, :4], ob[:, :4]), t
            assert torch.equal(a.dequant()[:, :4], b.dequant()[:, :4]), t
        assert a.check() == L.LORES_OK and b.check() == L.LORES_OK
    finally:
        a.close()
        b.close()
