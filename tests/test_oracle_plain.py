"""The oracle's evaluation scheme pinned to the plain definition of the step.

The oracle's decode step (lo_tile_step) evaluates the method with fixed choices that
make two implementations agree bit for bit: a fixed fp32 order for the dot product S'k,
a Newton reciprocal in place of r/m, and a quantizer that rounds x r/m to a 1/256 grid
before adding the dither.  None of these is the method itself.  These tests tie them to
the plain definition ("Quantizing Recurrent Language Models Is Easier Than You Think",
summary page: General recurrence form; Proposition 1, s = max|S_G| / r; Proposition 3,
stochastic rounding):

* every stochastically rounded code equals floor(x r / m + d / 256), computed exactly
  with rationals, except where that sum lies so close to an integer that the 1/256-grid
  rounding may cross it;
* one step of the evaluated oracle and one step of the plain-definition oracle
  (lo_tile_step_plain: double precision, IEEE division, floor), started from the same
  state with the same inputs and dither, agree within the parity bounds (codes equal
  except <= 1e-4 of entries at +-1, dequantized state and readout within rel-L2 1e-5) on
  the five workload shapes.
"""
from fractions import Fraction

import numpy as np
import pytest

from bit_recurrent_state_lores_b200 import synth
from oracle import oracle as O


def _exact_codes(X, r, G, tkey, d_k, stochastic):
    """floor(x r / m + u) per entry in exact rational arithmetic (u = d/256, or 1/2 for
    round to nearest), and the distance of that sum from the nearest integer."""
    d_v = X.shape[0]
    codes = np.zeros(X.shape, np.int64)
    dist = np.ones(X.shape)
    for i in range(d_v):
        for g0 in range(0, d_k, G):
            grp = [Fraction(float(x)) for x in X[i, g0:g0 + G]]
            m = max(abs(x) for x in grp)
            if m == 0:
                continue
            for jj, x in enumerate(grp):
                j = g0 + jj
                u = Fraction(O.dither(tkey, d_k, i, j), 256) if stochastic else Fraction(1, 2)
                y = x * r / m + u
                fl = y.numerator // y.denominator
                codes[i, j] = fl
                frac = y - fl
                dist[i, j] = float(min(frac, 1 - frac))
    return codes, dist


@pytest.mark.parametrize("bits,G,stochastic", [(8, 16, 1), (8, 32, 1), (4, 16, 1), (6, 32, 1),
                                               (8, 32, 0)])
def test_codes_equal_exact_floor(bits, G, stochastic):
    d_k, d_v = 64, 24
    cfg = O.TileCfg(d_k, d_v, group=G, bits=bits, stochastic=stochastic)
    g = np.random.default_rng(100 + bits + G)
    X = (g.standard_normal((d_v, d_k)) * np.exp(g.uniform(-3, 3, (d_v, 1)))).astype(np.float32)
    tkey = O.tile_key(O.step_key(11, 3), 5)
    codes, scales, flag = O.tile_quantize(cfg, X, tkey)
    assert flag == 0
    got = O.unpack_codes(cfg, codes)
    r = (1 << (bits - 1)) - 1
    want, dist = _exact_codes(X, r, G, tkey, d_k, stochastic)
    # the grid rounds x r/m by at most 2^-9 and the reciprocal errs by < 2^-21 relative
    # (below 2^-14 of a step for |x r/m| <= 127): only sums that close to an integer may
    # land on the other side
    band = 2.0 ** -9 + 2.0 ** -12
    near = dist < band
    assert near.mean() < 0.01
    assert (got[~near] == want[~near]).all(), np.argwhere((got != want) & ~near)[:5]
    assert (np.abs(got - want) <= 1).all()


def _tile_inputs(wl, hp, t, tiles):
    q, k, v, a, b = [x.numpy() for x in synth.step_inputs(wl, t, hp, device="cpu")]
    return [(q[bb, hh], k[bb, hh], v[bb, hh], a[bb, hh], b[bb, hh]) for (bb, hh) in tiles]


def _case_workloads():
    """The five workload shapes at a reduced batch: (workload, head bits, tiles)."""
    out = []
    tiny = synth.workload("tiny")
    out.append((tiny, [8] * tiny.H, [(0, 0), (0, 1)]))
    gdn = synth.workload("gdn", B=2)
    out.append((gdn, [8] * gdn.H, [(0, 0), (1, 7), (0, 19), (1, 31)]))
    m2 = synth.workload("mamba2", B=2)
    out.append((m2, [8] * m2.H, [(0, 0), (1, 50), (0, 101), (1, 127)]))
    kda = synth.workload("kda", B=2)
    hp = synth.head_params(kda)
    kbits = list(O.assign_bits_by_decay(hp["mean_decay"], 0.25, 8, 4))
    hi = [h for h in range(kda.H) if kbits[h] == 8][:2]
    lo = [h for h in range(kda.H) if kbits[h] == 4][:2]
    out.append((kda, kbits, [(0, hi[0]), (1, hi[1]), (0, lo[0]), (1, lo[1])]))
    sw = synth.workload("sweep", B=2, layers=1)
    out.append((sw, [8] * sw.H, [(0, 0), (1, 9), (0, 22), (1, 31)]))
    return out


def test_plain_definition_matches_evaluated_step_teacher_forced():
    """From the same state, one step of each oracle; codes +-1 on <= 1e-4 of all entries,
    dequantized state (entries with equal codes) and readout within rel-L2 1e-5 per
    workload.  A single code at +-1 moves the dequantized state by a full step s, about
    1/40 of a typical entry, so rel-L2 1e-5 over all entries would allow no flip at all
    (a flip rate f gives about sqrt(f)/40): the two bounds are read as one budget for the
    codes and one for the scales and the readout."""
    n_diff = n_total = 0
    for wl, bits, tiles in _case_workloads():
        hp = synth.head_params(wl)
        cfgs = {t: O.TileCfg(wl.d_k, wl.d_v, group=wl.G, bits=bits[t[1]], delta=wl.delta,
                             diag=wl.diag) for t in tiles}
        state = {t: cfgs[t].zero_state() for t in tiles}
        o_err_num = o_err_den = s_err_num = s_err_den = 0.0
        for step in range(6):
            inp = _tile_inputs(wl, hp, step, tiles)
            sk = O.step_key(wl.seed, step)
            for t, (q, k, v, a, b) in zip(tiles, inp):
                cfg = cfgs[t]
                tk = O.tile_key(sk, t[0] * wl.H + t[1])
                st, sc = state[t]
                st2, sc2 = st.copy(), sc.copy()
                o1, f1, _ = O.tile_step(cfg, st, sc, q, k, v, a, b, tk)
                o2, f2, _ = O.tile_step_plain(cfg, st2, sc2, q, k, v, a, b, tk)
                assert f1 == f2 == 0
                c1 = O.unpack_codes(cfg, st)
                c2 = O.unpack_codes(cfg, st2)
                d = np.abs(c1 - c2)
                assert d.max() <= 1, (wl.name, step, t)
                n_diff += int((d != 0).sum())
                n_total += d.size
                # dequantized state over the entries whose codes agree (the scales'
                # agreement); the entries at +-1 are bounded by the code budget above
                same = d == 0
                S1 = c1 * np.repeat(sc.astype(np.float64), cfg.group, axis=1)
                S2 = c2 * np.repeat(sc2.astype(np.float64), cfg.group, axis=1)
                s_err_num += float((((S1 - S2) * same) ** 2).sum())
                s_err_den += float(((S2 * same) ** 2).sum())
                o_err_num += float(((o1 - o2) ** 2).sum())
                o_err_den += float((o2 ** 2).sum())
                # the evaluated trajectory continues (teacher forcing of the next step)
        assert np.sqrt(s_err_num / s_err_den) <= 1e-5, wl.name
        assert np.sqrt(o_err_num / o_err_den) <= 1e-5, wl.name
    print("codes at +-1:", n_diff, "of", n_total)
    assert n_diff <= 1e-4 * n_total, (n_diff, n_total)


def test_plain_definition_fp32_state_matches():
    """fp32 heads: the plain step and the evaluated step differ only by fp32 rounding."""
    wl = synth.workload("sweep", B=1, layers=1)
    hp = synth.head_params(wl)
    cfg = O.TileCfg(wl.d_k, wl.d_v, bits=32, delta=1)
    st, sc = cfg.zero_state()
    for step in range(5):
        (q, k, v, a, b), = _tile_inputs(wl, hp, step, [(0, 3)])
        st2, sc2 = st.copy(), sc.copy()
        o1, _, _ = O.tile_step(cfg, st, sc, q, k, v, a, b, 0)
        o2, _, _ = O.tile_step_plain(cfg, st2, sc2, q, k, v, a, b, 0)
        assert np.linalg.norm(st - st2) <= 1e-6 * np.linalg.norm(st2)
        assert np.linalg.norm(o1 - o2) <= 1e-6 * np.linalg.norm(o2)


def test_plain_step_catches_a_planted_mistake():
    """The comparison has teeth: a plain step whose dither is shifted by one grid step
    (d + 1 in place of d) disagrees with the evaluated step far beyond the bound."""
    wl = synth.workload("sweep", B=1, layers=1)
    hp = synth.head_params(wl)
    cfg = O.TileCfg(wl.d_k, wl.d_v, bits=8, delta=1)
    st, sc = cfg.zero_state()
    for step in range(3):
        (q, k, v, a, b), = _tile_inputs(wl, hp, step, [(0, 5)])
        O.tile_step(cfg, st, sc, q, k, v, a, b, O.tile_key(O.step_key(1, step), 5))
    # one more step, quantized exactly by hand from the evaluated x with a shifted dither
    tk = O.tile_key(O.step_key(1, 3), 5)
    (q, k, v, a, b), = _tile_inputs(wl, hp, 3, [(0, 5)])
    st1, sc1 = st.copy(), sc.copy()
    _, _, X = O.tile_step(cfg, st1, sc1, q, k, v, a, b, tk, want_x=True)
    good = O.unpack_codes(cfg, st1)
    m = np.abs(X.astype(np.float64)).max(axis=1, keepdims=True)
    d = np.array([[O.dither(tk, cfg.d_k, i, j) for j in range(cfg.d_k)] for i in range(cfg.d_v)])
    shifted = np.floor(X * 127.0 / m + (d + 1 + 0.5) / 256.0)
    assert (shifted != good).mean() > 10 * 1e-4


def test_all_cores_loop_equals_the_single_thread_step():
    """The OpenMP tile loop of the CPU baseline computes what lo_tile_step computes, tile
    by tile (mixed int8 / int4 heads, diagonal decay)."""
    wl = synth.workload("kda", B=3, H=8)
    hp = synth.head_params(wl)
    bits = [8 if h % 3 == 0 else 4 for h in range(wl.H)]
    cfgs = [O.TileCfg(wl.d_k, wl.d_v, bits=b, delta=1, diag=1) for b in bits]
    n = wl.B * wl.H
    cfg_of = [i % wl.H for i in range(n)]
    one = [cfgs[c].zero_state() for c in cfg_of]
    many = [(a.copy(), b.copy()) for a, b in one]
    for t in range(3):
        q, k, v, a, b = [x.numpy() for x in synth.step_inputs(wl, t, hp)]
        sk = O.step_key(9, t)
        keys = [O.tile_key(sk, i) for i in range(n)]
        o1 = np.stack([O.tile_step(cfgs[cfg_of[i]], one[i][0], one[i][1], q.reshape(n, -1)[i],
                                   k.reshape(n, -1)[i], v.reshape(n, -1)[i], a.reshape(n, -1)[i],
                                   b.reshape(n)[i], keys[i])[0] for i in range(n)])
        o2, flags, used = O.batch_step(cfgs, cfg_of, [m[0] for m in many], [m[1] for m in many],
                                       q.reshape(n, -1), k.reshape(n, -1), v.reshape(n, -1),
                                       a.reshape(n, -1), b.reshape(n), keys)
        assert used >= 1 and not flags.any()
        assert np.array_equal(o1, o2)
        for x, y in zip(one, many):
            assert np.array_equal(x[0], y[0]) and np.array_equal(x[1], y[1])
