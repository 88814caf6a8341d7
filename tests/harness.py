"""Test harness: run the CUDA library and the CPU oracle on the same seeded inputs.

The GPU side goes through the C ABI (bit_recurrent_state_lores_b200.lores); the
oracle side through oracle/.  The two share only the input generators of
bit_recurrent_state_lores_b200.synth.
"""
import numpy as np
import torch

from bit_recurrent_state_lores_b200 import synth
from oracle import oracle as O


def lib():
    from bit_recurrent_state_lores_b200 import lores
    return lores


def mixed_bits(wl, hp):
    """Head bits of a workload; the mixed map comes from the library's policy call."""
    if wl.mixed_frac is None:
        return [wl.bits] * wl.H
    return lib().lores_assign_bits_by_decay(hp["mean_decay"], wl.mixed_frac, 8, 4)


class GpuRun:
    """One handle of the library holding the state of one layer for a batch."""

    def __init__(self, wl, head_bits, seed, stochastic=1, device=0, axis=0, group_bits=None,
                 dense=0):
        """group_bits: None, or per head a list of the key groups' bit widths (then
        head_bits only names the heads' nominal widths for the oracle configs)."""
        L = lib()
        self.wl, self.bits, self.seed, self.axis = wl, list(head_bits), seed, axis
        self.stochastic = stochastic
        self.group_bits = group_bits
        self.dense = dense
        self.h = L.lores_create(wl.B, wl.H, wl.d_k, wl.d_v,
                                group_size=wl.d_k if axis else (wl.group or 0),
                                delta=wl.delta, decay_diag=wl.diag,
                                head_bits=None if group_bits is not None else head_bits,
                                stochastic=stochastic, seed=seed, device=device,
                                scale_axis=axis, group_bits=group_bits, dense_codes=dense)
        self.layout, self.head_off = L.lores_get_layout(self.h, wl.H)
        self.o = torch.empty(wl.B, wl.H, wl.d_v, device="cuda", dtype=torch.float32)

    def step(self, inputs, t):
        q, k, v, a, b = inputs
        lib().lores_decode_step(self.h, q, k, v, a, b, self.o, t)
        return self.o

    def export(self):
        wl = self.wl
        codes = torch.empty(self.layout.code_bytes, dtype=torch.uint8)
        scales = torch.empty(self.layout.scale_count, dtype=torch.float32)
        lib().lores_export_codes(self.h, codes, scales)
        shape = (wl.B, wl.H, wl.d_k) if self.axis else (wl.B, wl.H, wl.d_v, self.layout.n_groups)
        return codes.numpy().reshape(wl.B, -1), scales.numpy().reshape(shape)

    def load(self, codes, scales):
        lib().lores_load_codes(self.h, np.ascontiguousarray(codes), np.ascontiguousarray(scales))

    def dequant(self):
        wl = self.wl
        out = torch.empty(wl.B, wl.H, wl.d_v, wl.d_k, device="cuda", dtype=torch.float32)
        lib().lores_dequant_state(self.h, out)
        torch.cuda.synchronize()
        return out

    def check(self):
        return lib().lores_check_errors(self.h)

    def tile(self, codes, scales, b, hh):
        """(state, scales) of tile (b, hh) from an export, in the oracle's layout."""
        wl, bits = self.wl, self.bits[hh]
        cfg = tile_cfg(wl, bits, axis=self.axis,
                       group_bits=None if self.group_bits is None else self.group_bits[hh],
                       dense=self.dense)
        off = self.head_off[hh]
        raw = codes[b, off:off + cfg.code_bytes()].copy()
        if bits == 32:
            raw = raw.view(np.float32).reshape(wl.d_v, wl.d_k).copy()
        return raw, scales[b, hh].copy()

    def close(self):
        if self.h:
            lib().lores_destroy(self.h)
            self.h = None


def tile_cfg(wl, bits, stochastic=1, axis=0, group_bits=None, dense=0):
    return O.TileCfg(wl.d_k, wl.d_v, group=wl.d_k if axis else wl.G, bits=bits,
                     delta=wl.delta, diag=wl.diag, stochastic=stochastic, axis=axis,
                     group_bits=group_bits, dense=dense)


def host_tile_inputs(inputs, tiles):
    """Host copies of the inputs of the listed (b, h) tiles."""
    q, k, v, a, b = inputs
    bi = torch.tensor([t[0] for t in tiles])
    hi = torch.tensor([t[1] for t in tiles])
    qs = q[bi, hi].cpu().numpy()
    ks = k[bi, hi].cpu().numpy()
    vs = v[bi, hi].cpu().numpy()
    as_ = a[bi, hi].cpu().numpy()
    bs = b[bi, hi].cpu().numpy()
    return [(qs[n], ks[n], vs[n], as_[n], bs[n]) for n in range(len(tiles))]


class OracleTiles:
    """The oracle's own trajectory for a few (b, h) tiles of a workload."""

    def __init__(self, wl, head_bits, seed, tiles, stochastic=1, axis=0, group_bits=None,
                 dense=0):
        self.wl, self.bits, self.seed, self.tiles = wl, list(head_bits), seed, list(tiles)
        self.cfg = {t: tile_cfg(wl, self.bits[t[1]], stochastic, axis,
                                None if group_bits is None else group_bits[t[1]], dense)
                    for t in self.tiles}
        self.state = {t: self.cfg[t].zero_state() for t in self.tiles}

    def load(self, t, state, scales):
        self.state[t] = (state.copy(), scales.copy())

    def step(self, host_inputs, step):
        sk = O.step_key(self.seed, step)
        out, flags = {}, {}
        for t, (q, k, v, a, b) in zip(self.tiles, host_inputs):
            st, sc = self.state[t]
            tk = O.tile_key(sk, t[0] * self.wl.H + t[1])
            o, flag, _ = O.tile_step(self.cfg[t], st, sc, q, k, v, a, b, tk)
            out[t], flags[t] = o, flag
        return out, flags


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def compare_tile(cfg, gpu_state, gpu_scales, ref_state, ref_scales):
    """Returns (n_diff_codes, max_abs_code_diff, dequant_rel_l2, scales_equal)."""
    if cfg.bits == 32:
        return 0, 0, rel_l2(gpu_state, ref_state), True
    small = cfg.d_v * cfg.d_k <= 4096 or cfg.group_bits is not None or cfg.dense
    cg = O.unpack_codes(cfg, gpu_state) if small else unpack_fast(cfg, gpu_state)
    cr = O.unpack_codes(cfg, ref_state) if small else unpack_fast(cfg, ref_state)
    d = np.abs(cg - cr)
    if cfg.axis:                                   # one scale per key column
        Sg = cg * gpu_scales.astype(np.float64)[None, :]
        Sr = cr * ref_scales.astype(np.float64)[None, :]
    else:
        Sg = cg * np.repeat(gpu_scales.astype(np.float64), cfg.group, axis=1)
        Sr = cr * np.repeat(ref_scales.astype(np.float64), cfg.group, axis=1)
    return int((d != 0).sum()), int(d.max()), rel_l2(Sg, Sr), bool((gpu_scales == ref_scales).all())


def unpack_fast(cfg, codes):
    """Vectorised unpack for large tiles; checked against the oracle's unpack in tests."""
    b = np.asarray(codes, np.uint8)
    if cfg.bits != 4:                       # 5- to 8-bit codes: one byte each
        return b.view(np.int8).reshape(cfg.d_v, cfg.d_k).astype(np.int32)
    lo = (b & 0xF).astype(np.int32)
    hi = (b >> 4).astype(np.int32)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((cfg.d_v, cfg.d_k), np.int32)
    out[:, 0::2] = lo.reshape(cfg.d_v, cfg.d_k // 2)
    out[:, 1::2] = hi.reshape(cfg.d_v, cfg.d_k // 2)
    return out


def assert_parity(cfg, gpu_state, gpu_scales, ref_state, ref_scales, where=""):
    """Spec bounds: codes equal except <= 1e-4 of entries at +-1; dequantized
    state within rel-L2 1e-5."""
    n, dmax, rl2, _ = compare_tile(cfg, gpu_state, gpu_scales, ref_state, ref_scales)
    total = cfg.d_v * cfg.d_k
    assert dmax <= 1 and n <= 1e-4 * total, f"{where}: {n} codes differ (max {dmax})"
    assert rl2 <= 1e-5, f"{where}: dequantized state rel-L2 {rl2}"
    return n


def sample_tiles(wl, bits, n, seed=0):
    """n tiles spread over sequences and heads, covering every bit width present."""
    g = np.random.default_rng(seed)
    tiles = [(0, 0), (wl.B - 1, wl.H - 1)]
    for want in sorted(set(bits)):
        hs = [h for h in range(wl.H) if bits[h] == want]
        tiles.append((int(g.integers(wl.B)), int(g.choice(hs))))
    while len(tiles) < n:
        tiles.append((int(g.integers(wl.B)), int(g.integers(wl.H))))
    out = []
    for t in tiles:
        if t not in out:
            out.append(t)
    return out
