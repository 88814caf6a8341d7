"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: every expected value is a closed
form of the recurrence, an fp64 brute-force product, an invariant the pages
state (delta-rule projection, Propositions 1-3, the absmax scale), a
published known-answer vector, or a hand-derived worked example of the state
format.  Page references are to "Quantizing Recurrent Language Models Is
Easier Than You Think" (summary page).
"""
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed):
    return np.random.default_rng(seed)


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def draw(T, d_k, d_v, seed, diag=False, alpha_lo=0.5, beta_hi=2.0):
    """Seeded inputs inside the recurrence's domain (General recurrence form):
    unit q, k; beta in (0, 2); alpha in (0, 1]."""
    g = rng(seed)
    q = unit(g.standard_normal((T, d_k))).astype(np.float32)
    k = unit(g.standard_normal((T, d_k))).astype(np.float32)
    v = g.standard_normal((T, d_v)).astype(np.float32)
    beta = g.uniform(0.05, beta_hi * 0.95, T).astype(np.float32)
    shape = (T, d_k) if diag else (T, 1)
    alpha = g.uniform(alpha_lo, 1.0, shape).astype(np.float32)
    return q, k, v, alpha, beta


def run_fp32(cfg, q, k, v, alpha, beta, S0=None):
    S = np.zeros((cfg.d_v, cfg.d_k), np.float32) if S0 is None else S0.astype(np.float32).copy()
    sc = np.zeros((cfg.d_v, cfg.n_groups), np.float32)
    Ss, os_ = [], []
    for t in range(q.shape[0]):
        o, flag, _ = O.tile_step(cfg, S, sc, q[t], k[t], v[t], alpha[t], beta[t], 0)
        assert flag == 0
        Ss.append(S.copy())
        os_.append(o)
    return Ss, os_


def recur64(S, a, k, v, beta, delta):
    """fp64 brute force: S diag(a) (I - delta beta k k^T) + beta v k^T."""
    d_k = S.shape[1]
    a = np.broadcast_to(np.asarray(a, np.float64), (d_k,))
    k = k.astype(np.float64)
    A = np.diag(a) @ (np.eye(d_k) - delta * float(beta) * np.outer(k, k))
    return S.astype(np.float64) @ A + float(beta) * np.outer(v.astype(np.float64), k)


# --------------------------------------------------------------------------
# Random bits: published known-answer vectors and uniformity
# --------------------------------------------------------------------------

def test_rng_known_answers():
    n = 0
    for line in open(os.path.join(GOLDEN, "rng_kat.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        fn, arg, want = line.split()
        if fn == "splitmix64":
            z = (int(arg) * 0x9E3779B97F4A7C15) % 2**64
            assert O.splitmix64(z) == int(want, 16)
        else:
            assert O.fmix32(int(arg, 16)) == int(want, 16)
        n += 1
    assert n == 7


def test_dither_bytes_uniform_and_keyed():
    # chi-square over 256 bins on 2^17 dithers from many tiles, steps and elements
    counts = np.zeros(256)
    for step in range(8):
        sk = O.step_key(11, step)
        for tile in range(4):
            tk = O.tile_key(sk, tile)
            for i in range(32):
                for j in range(128):
                    counts[O.dither(tk, 128, i, j)] += 1
    n = counts.sum()
    chi2 = ((counts - n / 256) ** 2 / (n / 256)).sum()
    # 255 dof: mean 255, sd ~22.6; 6 sd bound
    assert chi2 < 255 + 6 * 22.6, chi2
    # different steps / tiles / seeds give different keys
    keys = {O.tile_key(O.step_key(s, t), b) for s in range(3) for t in range(50) for b in range(40)}
    assert len(keys) == 3 * 50 * 40


def test_dither_adjacent_columns_independent():
    # the four bytes of one hash feed four columns: their pairwise correlation is ~0
    sk = O.step_key(5, 9)
    tk = O.tile_key(sk, 3)
    d = np.array([[O.dither(tk, 128, i, j) for j in range(128)] for i in range(128)], float)
    for off in (1, 2, 3, 4):
        c = np.corrcoef(d[:, :-off].ravel(), d[:, off:].ravel())[0, 1]
        assert abs(c) < 0.03, (off, c)


def test_mulfold_is_the_folded_64_bit_product():
    # the words of the dither stream: (low half XOR high half) of 32 x 32 -> 64-bit
    # products, checked against Python's exact integer product
    g = rng(4)
    for a, b in zip(g.integers(0, 2**32, 200, dtype=np.uint64), g.integers(0, 2**32, 200, dtype=np.uint64)):
        p = int(a) * int(b)
        assert O.mulfold(int(a), int(b)) == (p & 0xFFFFFFFF) ^ (p >> 32)
    mul = (0x846CA68B, 0xCC9E2D51, 0x1B873593, 0xE6546B65)
    for c in (0, 1, 0xFFFFFFFF, 0x9E3779B9, 123456789):
        for q in range(4):
            assert O.dither_word(c, q) == O.mulfold(O.mulfold(c, 0x7FEB352D), mul[q])
    # lo_dither: block n4 = (row, 16 columns) has counter tile key + golden (4 n4 + 1);
    # column j takes byte j mod 4 of word (j mod 16) / 4 of its block
    tk = O.tile_key(O.step_key(3, 1), 7)
    w = O.dither_words(tk, 0, 64)
    for i in range(2):
        for j in range(128):
            n4 = i * 8 + j // 16
            c = (tk + 0x9E3779B9 * (4 * n4 + 1)) & 0xFFFFFFFF
            want = (O.dither_word(c, (j % 16) // 4) >> (8 * (j % 4))) & 0xFF
            assert O.dither(tk, 128, i, j) == want
            assert (int(w[i * 32 + j // 4]) >> (8 * (j % 4))) & 0xFF == want


def _dither_stream(tk, quads):
    w = O.dither_words(tk, 0, quads).astype(np.uint64)
    return np.stack([(w >> np.uint64(8 * j)) & np.uint64(255) for j in range(4)], 1).reshape(-1).astype(np.int64)


def test_dither_stream_byte_pairs_uniform():
    # 2^22 consecutive dither bytes of one tile (a tile's entries in row order): every
    # pair (d_e, d_e+lag) is uniform over the 65536 cells, for lags inside a word (1-3),
    # between the words of a 16-column block (4, 8, 12), across blocks (5, 16, 32) and
    # to the same column of the next row (128 at d_k = 128).  A hash that dropped a
    # fold, or kept one half of a product, fails this by orders of magnitude.
    for key in (0x12345678, O.tile_key(O.step_key(9, 2), 5)):
        d = _dither_stream(key, 2 ** 20)
        for lag in (1, 2, 3, 4, 5, 8, 12, 16, 32, 128):
            a = d[:-lag] * 256 + d[lag:]
            cnt = np.bincount(a, minlength=65536)
            e = len(a) / 65536
            chi = ((cnt - e) ** 2 / e).sum() / 65535
            # chi2 / dof has sd sqrt(2 / 65535) = 0.0055: 6 sd
            assert abs(chi - 1.0) < 6 * 0.0055, (key, lag, chi)


def test_dither_stream_gives_independent_rounding_errors():
    # Proposition 3's unbiasedness and the variance of a row's rounding error: with
    # independent uniform dither, floor(x + (d + 1/2)/256) - x has mean ~0 and the sum
    # over 128 entries has variance sum p(1 - p) (p = frac(x) on the 1/256 grid)
    d = _dither_stream(O.tile_key(O.step_key(1, 1), 0), 2 ** 20)
    x = 0.3 + (np.arange(d.size) % 7) * 0.05
    fr = x - np.floor(x)
    code = np.floor(x + (d + 0.5) / 256.0)
    err = code - x
    rows = err.reshape(-1, 128).sum(1)
    pv = (fr * (1 - fr)).reshape(-1, 128).sum(1).mean()
    # the 1/256 grid rounds fr to the nearest 1/256 (here fr is on a 1/20 grid: bias below
    # 1/512 per entry at most); the row-sum variance of independent Bernoulli errors is pv
    assert abs(rows.var() / pv - 1.0) < 0.03, rows.var() / pv
    assert abs(err.mean()) < 2.5e-3, err.mean()


# --------------------------------------------------------------------------
# Fixed-order dot product
# --------------------------------------------------------------------------

def test_dot_exact_on_integers():
    g = rng(1)
    for n in (16, 32, 64, 128, 256):
        a = g.integers(-50, 50, n).astype(np.float32)
        b = g.integers(-50, 50, n).astype(np.float32)
        assert O.dot_b16(a, b) == float(np.dot(a.astype(np.int64), b.astype(np.int64)))


def test_dot_error_bound():
    # |fl(a.b) - a.b| <= gamma_n sum|a_j b_j| (Higham, Accuracy and Stability, 3.1)
    g = rng(2)
    for n in (16, 64, 128, 256):
        a = g.standard_normal(n).astype(np.float32)
        b = g.standard_normal(n).astype(np.float32)
        exact = sum(Fraction(float(x)) * Fraction(float(y)) for x, y in zip(a, b))
        u = 2.0 ** -24
        bound = n * u / (1 - n * u) * float(np.sum(np.abs(a.astype(np.float64) * b)))
        assert abs(float(Fraction(O.dot_b16(a, b)) - exact)) <= bound


def test_dot_combine_order_worked_example():
    # Block sums p = [1, 2^24, 1, -2^24] (one nonzero term per 16-column block).
    # Nearest partner first: [p0+p1, p2+p3] = [2^24 (the 1 is lost: tie to even),
    # 1 - 2^24 (exact)], then 2^24 + (1 - 2^24) = 1.  (Left to right would give 0;
    # the far partner first would give [p0+p2, p1+p3] = [2, 0] -> 2.)
    a = np.zeros(64, np.float32)
    b = np.ones(64, np.float32)
    a[0], a[16], a[32], a[48] = 1.0, 2.0 ** 24, 1.0, -(2.0 ** 24)
    assert O.dot_b16(a, b) == 1.0


def test_dot_block_chains_worked_examples():
    b = np.ones(16, np.float32)
    # Chains by half and parity: c00 = col 0, c10 = col 8, c01 = col 1, c11 = col 9.
    # (c00 + c10) + (c01 + c11) = (1 + 2^24 -> 2^24) + (1 - 2^24) = 1; pairing by
    # parity first, (c00 + c01) + (c10 + c11), would give 2 + 0 = 2.
    a = np.zeros(16, np.float32)
    a[0], a[8], a[1], a[9] = 1.0, 2.0 ** 24, 1.0, -(2.0 ** 24)
    assert O.dot_b16(a, b) == 1.0
    # Columns 1 and 3 share chain (0, 1), away from column 0: 2^24 + (1 + 1) = 2^24 + 2
    # exactly; one chain over columns 0..3 would lose both ones (2^24 + 1 -> 2^24).
    a = np.zeros(16, np.float32)
    a[0], a[1], a[3] = 2.0 ** 24, 1.0, 1.0
    assert O.dot_b16(a, b) == 2.0 ** 24 + 2
    # Inside a chain the order is ascending: 2^24 at column 0 absorbs the ones at
    # columns 2 and 4 one at a time (ties to even); descending would give 2^24 + 2.
    a = np.zeros(16, np.float32)
    a[0], a[2], a[4] = 2.0 ** 24, 1.0, 1.0
    assert O.dot_b16(a, b) == 2.0 ** 24


def test_newton_reciprocal_error_bound():
    # three Newton-Raphson steps from the exponent-reflected seed: |m y - 1| <= 2^-21
    g = rng(60)
    ms = np.concatenate([2.0 ** g.uniform(-100, 100, 20000), 1 + np.arange(0, 1, 1 / 4096),
                         [2.0 ** -100, 2.0 ** 100, 1.5, 1.9999999]]).astype(np.float32)
    worst = 0.0
    for m in ms:
        y = O.recip_nr(m)
        worst = max(worst, abs(float(m) * y - 1.0))
    assert worst <= 2.0 ** -21, worst
    for k in range(-100, 101, 7):                     # exact on powers of two
        assert O.recip_nr(2.0 ** k) == 2.0 ** -k


# --------------------------------------------------------------------------
# The recurrence (General recurrence form), quantization off (fp32 state)
# --------------------------------------------------------------------------

# --------------------------------------------------------------------------
# Exact projection u = S'k for integer codes with one scale per row
# --------------------------------------------------------------------------

def test_fixed_point_grid_is_exact_rounding():
    # Y_j = alpha_j k_j 2^E rounded to the nearest integer (ties to even), with
    # max |alpha k| 2^E in [2^29, 2^30): checked with exact rationals
    g = rng(21)
    for trial in range(12):
        n = int(g.choice([16, 32, 128, 256]))
        diag = trial % 2 == 1
        mag = 10.0 ** g.uniform(-30, 30)
        k = (g.standard_normal(n) * mag).astype(np.float32)
        k[g.integers(0, n, 3)] = 0.0
        alpha = g.uniform(0.1, 1.0, n if diag else 1).astype(np.float32)
        ok, Y, E = O.fixed_point(alpha, k, diag)
        assert ok
        p = [Fraction(float(alpha[j if diag else 0])) * Fraction(float(k[j])) for j in range(n)]
        m = max(abs(x) for x in p)
        assert Fraction(2) ** 29 <= m * Fraction(2) ** E < Fraction(2) ** 30, (E, float(m))
        for j in range(n):
            assert int(Y[j]) == round(p[j] * Fraction(2) ** E), (j, int(Y[j]))
    # a tie rounds to even: alpha k 2^E = 2^29 + 1/2 has neighbours 2^29 and 2^29 + 1
    k = np.array([2.0 ** 29 + 0.5, 1.5, 2.5, -2.5], np.float32)
    ok, Y, E = O.fixed_point(np.ones(1, np.float32), k, False)
    assert ok and E == 0 and list(Y) == [2 ** 29, 2, 2, -2]
    # all zero: E = 0 and Y = 0; a non-finite product is refused
    ok, Y, E = O.fixed_point(np.ones(1, np.float32), np.zeros(8, np.float32), False)
    assert ok and E == 0 and not Y.any()
    assert not O.fixed_point(np.ones(1, np.float32), np.array([1.0, np.inf], np.float32), False)[0]
    assert not O.fixed_point(np.array([np.nan], np.float32), np.ones(4, np.float32), False)[0]


@pytest.mark.parametrize("bits,d_k,diag", [(8, 128, 0), (8, 32, 1), (4, 128, 1), (6, 64, 0)])
def test_exact_projection_error_bound(bits, d_k, diag):
    # u_i against the exact rational sum_j c_ij s_i alpha_j k_j: the only errors are the
    # fixed-point grid (half a step per term), one double rounding and one fp32 rounding
    g = rng(22 + bits + d_k)
    cfg, ints, codes, scales = quantized_case(bits, d_k, d_k=d_k, d_v=8, seed=23, diag=diag)
    k = unit(g.standard_normal(d_k)).astype(np.float32)
    alpha = g.uniform(0.3, 1.0, d_k if diag else 1).astype(np.float32)
    ok, Y, E = O.fixed_point(alpha, k, bool(diag))
    assert ok
    for i in range(cfg.d_v):
        s = Fraction(float(scales[i, 0]))
        u = O.exact_projection(cfg, codes, scales[i, 0], i, Y, E)
        t = s * sum(int(ints[i, j]) * Fraction(float(alpha[j if diag else 0])) * Fraction(float(k[j]))
                    for j in range(d_k))
        grid = s * sum(abs(int(c)) for c in ints[i]) * Fraction(1, 2 ** (E + 1))
        bound = grid + (abs(t) + grid) * Fraction(1, 2 ** 53) + Fraction(abs(u)) * Fraction(1, 2 ** 24) \
            + Fraction(1, 2 ** 149)
        assert abs(Fraction(u) - t) <= bound, (i, u, float(t))
        # and it is the integer sum itself, rounded: U exact, then fl64, then fl32
        U = sum(int(ints[i, j]) * int(Y[j]) for j in range(d_k))
        assert u == float(np.float32(np.ldexp(float(scales[i, 0]) * float(U), -E)))


def test_exact_projection_is_what_the_step_uses():
    # one step of an int8 head with one scale per row: w_i = beta (v_i - u_i) with u the
    # exact projection (not the fp32 block-order dot); a head with two scales per row keeps
    # the block order
    g = rng(24)
    q, k, v, alpha, beta = draw(1, 128, 8, 25)
    for group, exact in ((128, True), (64, False)):
        cfg, ints, codes, scales = quantized_case(8, group, d_k=128, d_v=8, seed=26, diag=0)
        _, _, x = O.tile_step(cfg, codes.copy(), scales.copy(), q[0], k[0], v[0], alpha[0], beta[0], 7,
                              want_x=True)
        ok, Y, E = O.fixed_point(alpha[0], k[0], False)
        for i in range(cfg.d_v):
            Sp = (ints[i].astype(np.float32) * np.repeat(scales[i] * alpha[0, 0], group)).astype(np.float32)
            if exact:
                u = np.float32(O.exact_projection(cfg, codes, scales[i, 0], i, Y, E))
            else:
                u = np.float32(O.dot_b16(Sp, k[0]))
            w = np.float32(beta[0] * np.float32(v[0, i] - u))
            xi = (Sp.astype(np.float64) + np.float64(w) * k[0]).astype(np.float32)   # fma: one rounding
            np.testing.assert_array_equal(x[i], xi)


def test_closed_form_no_decay_no_delta():
    # alpha = 1, delta = 0: S_T = sum_t beta_t v_t k_t^T and o_t = S_t q_t
    T, d = 40, 32
    cfg = O.TileCfg(d, d, bits=32, delta=0)
    q, k, v, _, beta = draw(T, d, d, 3)
    alpha = np.ones((T, 1), np.float32)
    Ss, os_ = run_fp32(cfg, q, k, v, alpha, beta)
    S = np.zeros((d, d))
    for t in range(T):
        S += float(beta[t]) * np.outer(v[t].astype(np.float64), k[t].astype(np.float64))
        np.testing.assert_allclose(Ss[t], S, rtol=0, atol=1e-5 * np.abs(S).max())
        o = S @ q[t].astype(np.float64)
        assert np.linalg.norm(os_[t] - o) <= 1e-5 * np.linalg.norm(o)


@pytest.mark.parametrize("diag", [0, 1])
def test_closed_form_decayed_linear_attention(diag):
    # delta = 0: S_T[:, j] = sum_t (prod_{tau > t} alpha_tau,j) beta_t v_t k_t,j
    T, dk, dv = 30, 32, 16
    cfg = O.TileCfg(dk, dv, bits=32, delta=0, diag=diag)
    q, k, v, alpha, beta = draw(T, dk, dv, 4 + diag, diag=bool(diag), alpha_lo=0.7)
    Ss, _ = run_fp32(cfg, q, k, v, alpha, beta)
    a = np.broadcast_to(alpha.astype(np.float64), (T, dk))
    S = np.zeros((dv, dk))
    for t in range(T):
        w = np.prod(a[t + 1:], axis=0)
        S += float(beta[t]) * np.outer(v[t].astype(np.float64), k[t] * w)
    np.testing.assert_allclose(Ss[-1], S, rtol=0, atol=2e-6 * np.abs(S).max() * T)


def test_delta_rule_projection_invariant():
    # delta = 1, beta = 1, unit k: (I - k k^T) annihilates k, so S_t k_t = v_t
    T, d = 40, 64
    cfg = O.TileCfg(d, d, bits=32, delta=1, diag=1)
    q, k, v, alpha, _ = draw(T, d, d, 6, diag=True)
    beta = np.ones(T, np.float32)
    Ss, _ = run_fp32(cfg, q, k, v, alpha, beta)
    for t in range(T):
        r = Ss[t].astype(np.float64) @ k[t].astype(np.float64) - v[t]
        assert np.linalg.norm(r) <= 1e-5 * np.linalg.norm(v[t])


@pytest.mark.parametrize("delta,diag", [(1, 0), (1, 1), (0, 1)])
def test_brute_force_recurrence_fp32_state(delta, diag):
    T, d = 24, 16
    cfg = O.TileCfg(d, d, bits=32, delta=delta, diag=diag)
    q, k, v, alpha, beta = draw(T, d, d, 7 + delta + 2 * diag, diag=bool(diag))
    S0 = rng(8).standard_normal((d, d)).astype(np.float32)
    Ss, os_ = run_fp32(cfg, q, k, v, alpha, beta, S0=S0)
    S = S0.astype(np.float64)
    for t in range(T):
        S = recur64(S, alpha[t], k[t], v[t], beta[t], delta)
        np.testing.assert_allclose(Ss[t], S, rtol=0, atol=1e-5 * max(1.0, np.abs(S).max()))
        np.testing.assert_allclose(os_[t], S @ q[t].astype(np.float64), rtol=0,
                                   atol=1e-5 * max(1.0, np.abs(S).max()))


# --------------------------------------------------------------------------
# Quantized step: dequantize -> update -> requantize (Key properties, item 3)
# --------------------------------------------------------------------------

def quantized_case(bits, group, d_k=32, d_v=16, seed=9, delta=1, diag=1):
    g = rng(seed)
    cfg = O.TileCfg(d_k, d_v, group=group, bits=bits, delta=delta, diag=diag)
    r = (1 << (bits - 1)) - 1
    ints = g.integers(-r, r + 1, (d_v, d_k))
    codes = O.pack_codes(cfg, ints)
    scales = g.uniform(0.01, 0.1, (d_v, cfg.n_groups)).astype(np.float32)
    return cfg, ints, codes, scales


@pytest.mark.parametrize("bits,group,delta,diag", [(8, 32, 1, 1), (8, 16, 0, 0), (4, 32, 1, 0),
                                                    (4, 16, 1, 1), (8, 8, 1, 1)])
def test_quantized_step_matches_fp64_update(bits, group, delta, diag):
    d_k = 32
    if d_k % group:
        pytest.skip()
    cfg, ints, codes, scales = quantized_case(bits, group, delta=delta, diag=diag)
    q, k, v, alpha, beta = draw(1, cfg.d_k, cfg.d_v, 10, diag=bool(diag))
    # fp64 reference: dequantize with the scale of each entry's group, then update
    S_hat = ints * np.repeat(scales.astype(np.float64), group, axis=1)
    X = recur64(S_hat, alpha[0], k[0], v[0], beta[0], delta)
    o, flag, x = O.tile_step(cfg, codes, scales, q[0], k[0], v[0], alpha[0], beta[0],
                             O.tile_key(O.step_key(1, 2), 3), want_x=True)
    assert flag == 0
    np.testing.assert_allclose(x, X, rtol=0, atol=1e-5 * np.abs(X).max())
    np.testing.assert_allclose(o, X @ q[0].astype(np.float64), rtol=0, atol=1e-5 * np.abs(X).max())


@pytest.mark.parametrize("bits,group,sr", [(8, 128, 1), (8, 32, 1), (4, 128, 1), (4, 16, 1),
                                            (8, 128, 0), (4, 32, 0), (6, 128, 1), (5, 32, 1),
                                            (7, 64, 0), (6, 16, 0)])
def test_absmax_quantizer_invariants(bits, group, sr):
    # Proposition 1's scale: s_G = max|S_G| / r, r = 2^(b-1) - 1, codes in [-r, r]
    d_k, d_v = 128, 64
    cfg = O.TileCfg(d_k, d_v, group=group, bits=bits, stochastic=sr)
    r = (1 << (bits - 1)) - 1
    g = rng(12 + bits + group)
    X = (g.standard_normal((d_v, d_k)) * np.exp(g.uniform(-8, 8, (d_v, 1)))).astype(np.float32)
    X[3, :] = 0.0                                # an all-zero row
    X[5, :group] = 0.0                           # an all-zero group
    codes, scales, flag = O.tile_quantize(cfg, X, O.tile_key(O.step_key(2, 7), 1))
    assert flag == 0
    C_ = O.unpack_codes(cfg, codes)
    assert C_.min() >= -r and C_.max() <= r
    for i in range(d_v):
        for gi in range(cfg.n_groups):
            xs = X[i, gi * group:(gi + 1) * group]
            cs = C_[i, gi * group:(gi + 1) * group]
            m = np.float32(np.abs(xs).max())
            s = scales[i, gi]
            if m == 0:
                assert s == 0 and not cs.any()
                continue
            # s = m * fl(1/r): two roundings, so |s r / m - 1| <= 2^-24 + 2^-24 (+ tiny)
            assert s == np.float32(m * (np.float32(1) / np.float32(r)))
            assert r == 2 ** (bits - 1) - 1                  # Proposition 1: r = 2^(b-1) - 1
            assert abs(float(s) * r / float(m) - 1.0) <= 2.0 ** -23 * (1 + 1e-6)
            assert np.abs(cs).max() == r            # the group's max code is r exactly
            err = np.abs(cs * np.float64(s) - xs)
            lim = (1.0 if sr else 0.5 + 2.0 ** -8) * float(s) * (1 + 1e-6)
            assert err.max() <= lim


def test_int6_codes_one_byte_each():
    # 5 to 7-bit codes are stored one per byte (two's complement), like int8
    cfg = O.TileCfg(16, 2, bits=6)
    ints = np.array([list(range(-31, -15)), list(range(16, 32))])
    b = O.pack_codes(cfg, ints)
    assert b.size == 32 and b.view(np.int8).reshape(2, 16).tolist() == ints.tolist()


def test_int4_and_int8_packing_worked_example():
    # int4: even column in the low nibble, odd in the high one, two's complement.
    cfg4 = O.TileCfg(16, 1, bits=4)
    ints = np.array([[1, -1, 7, -7, 0, 3, -3, 2, 5, -5, 6, -6, 4, -4, 1, 0]])
    b = O.pack_codes(cfg4, ints)
    assert b[0] == 0xF1 and b[1] == 0x97 and b[2] == 0x30 and b[3] == 0x2D
    assert (O.unpack_codes(cfg4, b) == ints).all()
    cfg8 = O.TileCfg(16, 16, bits=8)
    allc = np.arange(-127, 129)[:256].reshape(16, 16).clip(-127, 127)
    b8 = O.pack_codes(cfg8, allc)
    assert b8.view(np.int8).reshape(16, 16).tolist() == allc.tolist()
    assert (O.unpack_codes(cfg8, b8) == allc).all()
    all4 = np.tile(np.arange(-7, 8), 2)[:16].reshape(1, 16)
    assert (O.unpack_codes(cfg4, O.pack_codes(cfg4, all4)) == all4).all()


def test_stochastic_rounding_unbiased_and_variance():
    # mean over 10^4 keys of code*s converges to x (Proposition 3's premise);
    # per-element variance is f(1-f) s^2 for fractional part f
    d_k, d_v = 16, 4
    cfg = O.TileCfg(d_k, d_v, bits=8)
    g = rng(13)
    X = g.standard_normal((d_v, d_k)).astype(np.float32)
    N = 10000
    acc = np.zeros((d_v, d_k))
    acc2 = np.zeros((d_v, d_k))
    for n in range(N):
        codes, scales, _ = O.tile_quantize(cfg, X, O.tile_key(O.step_key(n, 0), 0))
        Y = O.unpack_codes(cfg, codes) * scales.astype(np.float64)
        acc += Y
        acc2 += Y * Y
    mean = acc / N
    var = acc2 / N - mean ** 2
    s = (np.abs(X).max(axis=1, keepdims=True) / 127.0)
    f = (X / s) - np.floor(X / s)
    sd = np.sqrt(f * (1 - f)) * s
    bias_bound = s * 2.0 ** -9                      # the 1/256 grid rounds by <= 1/512 step
    assert (np.abs(mean - X) <= 4.5 * sd / np.sqrt(N) + bias_bound + 1e-12).all()
    np.testing.assert_allclose(var, (f * (1 - f)) * s ** 2, rtol=0, atol=0.08 * float(s.max()) ** 2)


def test_round_to_nearest_mode_is_deterministic_nearest():
    d_k, d_v = 32, 8
    cfg = O.TileCfg(d_k, d_v, bits=8, stochastic=0)
    X = rng(14).standard_normal((d_v, d_k)).astype(np.float32)
    c1, s1, _ = O.tile_quantize(cfg, X, 1)
    c2, s2, _ = O.tile_quantize(cfg, X, 999)
    assert (c1 == c2).all() and (s1 == s2).all()
    Y = O.unpack_codes(cfg, c1)
    nearest = np.rint(X.astype(np.float64) / s1.astype(np.float64))
    # equal except where x/s sits within 1/512 of a half step
    frac = np.abs(X / s1 - np.floor(X / s1) - 0.5)
    assert ((Y == nearest) | (frac < 2.0 ** -8)).all()


def test_scale_range_rules():
    # group maxima below 2^-100 are stored as zero; above 2^100 the row is overflow
    d_k, d_v = 32, 4
    cfg = O.TileCfg(d_k, d_v, group=16, bits=8)
    X = rng(16).standard_normal((d_v, d_k)).astype(np.float32)
    X[0, :16] *= np.float32(2.0 ** -104)              # tiny group, rest of the row normal
    X[1, 3] = np.float32(2.0 ** 101)                  # overflow row
    codes, scales, flag = O.tile_quantize(cfg, X, 3)
    C_ = O.unpack_codes(cfg, codes)
    assert flag == 1
    assert scales[0, 0] == 0 and not C_[0, :16].any() and np.abs(C_[0, 16:]).max() == 127
    assert not C_[1].any() and not scales[1].any()
    assert np.abs(C_[2:]).max() == 127


def test_nonfinite_row_is_zeroed_and_flagged():
    d_k, d_v = 32, 8
    cfg = O.TileCfg(d_k, d_v, bits=8)
    X = rng(15).standard_normal((d_v, d_k)).astype(np.float32)
    X[2, 5] = np.nan
    X[6, 0] = np.inf
    codes, scales, flag = O.tile_quantize(cfg, X, 7)
    assert flag == 1
    C_ = O.unpack_codes(cfg, codes)
    assert not C_[2].any() and not C_[6].any() and scales[2, 0] == 0 and scales[6, 0] == 0
    assert C_[[0, 1, 3, 4, 5, 7]].any(axis=1).all()


def test_step_requantization_equals_quantizer():
    # the step's requantization is the same quantizer as the state loader
    cfg, ints, codes, scales = quantized_case(8, 32, d_k=64, d_v=8, seed=16)
    q, k, v, alpha, beta = draw(1, 64, 8, 17, diag=True)
    tk = O.tile_key(O.step_key(3, 4), 5)
    c1, s1 = codes.copy(), scales.copy()
    _, _, x = O.tile_step(cfg, c1, s1, q[0], k[0], v[0], alpha[0], beta[0], tk, want_x=True)
    c2, s2, _ = O.tile_quantize(cfg, x, tk)
    assert (c1 == c2).all() and (s1 == s2).all()


# --------------------------------------------------------------------------
# Error recursion and Propositions 1-3
# --------------------------------------------------------------------------

def trajectories(bits, T, d, seed, delta, diag, alpha_lo=0.8, sr=1):
    """Quantized and fp32 trajectories from the same inputs and zero state.
    Returns lists of S_hat_t (dequantized), X_t (pre-quantization), S_fp_t."""
    q, k, v, alpha, beta = draw(T, d, d, seed, diag=bool(diag), alpha_lo=alpha_lo)
    cq = O.TileCfg(d, d, bits=bits, delta=delta, diag=diag, stochastic=sr)
    cf = O.TileCfg(d, d, bits=32, delta=delta, diag=diag)
    codes, sc = cq.zero_state()
    Sf = np.zeros((d, d), np.float32)
    scf = np.zeros((d, 1), np.float32)
    S_hat, X, S_fp = [], [], []
    for t in range(T):
        tk = O.tile_key(O.step_key(seed, t), 0)
        _, _, x = O.tile_step(cq, codes, sc, q[t], k[t], v[t], alpha[t], beta[t], tk, want_x=True)
        O.tile_step(cf, Sf, scf, q[t], k[t], v[t], alpha[t], beta[t], 0)
        S_hat.append(O.tile_dequant(cq, codes, sc).astype(np.float64))
        X.append(x.astype(np.float64))
        S_fp.append(Sf.astype(np.float64).copy())
    return (q, k, v, alpha, beta), S_hat, X, S_fp


@pytest.mark.parametrize("delta,diag", [(1, 0), (1, 1), (0, 0)])
def test_error_recursion_identity(delta, diag):
    # E_t = E_{t-1} diag(alpha_t)(I - delta beta_t k_t k_t^T) + eps_t with
    # E_t = S_hat_t - S_fp_t and eps_t = S_hat_t - X_t (this step's rounding)
    T, d = 30, 32
    (q, k, v, alpha, beta), S_hat, X, S_fp = trajectories(8, T, d, 20 + delta + diag, delta, diag)
    E_prev = np.zeros((d, d))
    for t in range(T):
        eps = S_hat[t] - X[t]
        a = np.broadcast_to(alpha[t].astype(np.float64), (d,))
        A = np.diag(a) @ (np.eye(d) - delta * float(beta[t]) * np.outer(k[t], k[t]))
        E = S_hat[t] - S_fp[t]
        pred = E_prev @ A + eps
        scale = max(np.abs(S_fp[t]).max(), 1e-30)
        assert np.abs(E - pred).max() <= 1e-5 * scale, t
        E_prev = E


def test_proposition2_decaying_error_bound():
    # ||E_t||_F <= sum_tau alpha^(t - tau) ||eps_tau||_F for alpha < 1 bounding the decay
    T, d = 60, 32
    (q, k, v, alpha, beta), S_hat, X, S_fp = trajectories(4, T, d, 30, 1, 1, alpha_lo=0.6)
    amax = float(alpha.max())
    assert amax < 1.0
    bound = 0.0
    for t in range(T):
        eps = np.linalg.norm(S_hat[t] - X[t])
        bound = amax * bound + eps
        E = np.linalg.norm(S_hat[t] - S_fp[t])
        assert E <= bound * (1 + 1e-4) + 1e-5 * np.abs(S_fp[t]).max(), t


def test_proposition1_value_axis_readout_error():
    # RTN with one scale per value row: E[e_i^2] = M_i^2 / (12 r^2) for the readout
    # error e = (S_hat - S) q with unit q (uniform rounding-error model)
    d_k, d_v, n = 128, 32, 400
    cfg = O.TileCfg(d_k, d_v, bits=4, stochastic=0)
    g = rng(40)
    num = np.zeros(d_v)
    den = np.zeros(d_v)
    for it in range(n):
        S = (g.standard_normal((d_v, d_k)) * g.uniform(0.1, 10, (d_v, 1))).astype(np.float32)
        q = unit(g.standard_normal(d_k))
        codes, sc, _ = O.tile_quantize(cfg, S, 0)
        e = (O.tile_dequant(cfg, codes, sc).astype(np.float64) - S) @ q
        M = np.abs(S).max(axis=1).astype(np.float64)
        num += e ** 2
        den += M ** 2 / (12 * 7 ** 2)
    ratio = num.sum() / den.sum()
    assert 0.9 < ratio < 1.1, ratio


def test_proposition3_sr_cross_terms_vanish():
    # delta = 0, scalar decay: E||E_t^SR||^2 = sum gamma^2 E||eps||^2 (no cross terms),
    # while RTN's cross terms reinforce.  A repeated token with a small write makes
    # consecutive RTN rounding errors nearly identical, the case the proposition targets.
    T, d, a, b = 40, 16, 0.97, 0.05
    g = rng(50)
    k = unit(g.standard_normal(d)).astype(np.float32)
    v = g.standard_normal(d).astype(np.float32)
    q = k.copy()
    S0 = g.standard_normal((d, d)).astype(np.float32)
    cf = O.TileCfg(d, d, bits=32, delta=0)

    def run(sr, seed):
        cq = O.TileCfg(d, d, bits=4, delta=0, stochastic=sr)
        codes, sc, _ = O.tile_quantize(cq, S0, O.tile_key(O.step_key(seed, 10 ** 6), 0))
        Sf = O.tile_dequant(cq, codes, sc)
        scf = np.zeros((d, 1), np.float32)
        eps = []
        for t in range(T):
            tk = O.tile_key(O.step_key(seed, t), 0)
            _, _, x = O.tile_step(cq, codes, sc, q, k, v, a, b, tk, want_x=True)
            O.tile_step(cf, Sf, scf, q, k, v, a, b, 0)
            eps.append(O.tile_dequant(cq, codes, sc).astype(np.float64) - x)
        E = O.tile_dequant(cq, codes, sc).astype(np.float64) - Sf
        gam = [np.float64(a) ** (T - 1 - t) for t in range(T)]
        return np.sum(E * E), sum(gm ** 2 * np.sum(e * e) for gm, e in zip(gam, eps))

    ratios = []
    for s in range(60):
        e, dsum = run(1, s)
        ratios.append(e / dsum)
    # SR: ratio 1 in expectation (spread ~0.15 per run, so test the mean of 60)
    assert 0.85 < np.mean(ratios) < 1.15, np.mean(ratios)
    e_rtn, d_rtn = run(0, 0)
    assert e_rtn / d_rtn > 5.0, e_rtn / d_rtn


# --------------------------------------------------------------------------
# Decay-based mixed precision (Table 5 text)
# --------------------------------------------------------------------------

def test_assign_bits_by_decay_worked_examples():
    # slowest-decaying (largest mean decay) heads are promoted
    assert O.assign_bits_by_decay([0.5, 0.9, 0.99, 0.7], 0.5).tolist() == [4, 8, 8, 4]
    # ties go to the lower head index
    assert O.assign_bits_by_decay([0.9, 0.9, 0.9, 0.1], 0.5).tolist() == [8, 8, 4, 4]
    # 25% of 32 heads -> 8 heads
    d = np.linspace(0.5, 0.9999, 32).astype(np.float32)
    b = O.assign_bits_by_decay(d, 0.25)
    assert (b[24:] == 8).all() and (b[:24] == 4).all()
    assert O.assign_bits_by_decay([0.3, 0.2], 0.0).tolist() == [4, 4]
    assert O.assign_bits_by_decay([0.3, 0.2], 1.0).tolist() == [8, 8]


# --------------------------------------------------------------------------
# Key-axis grouping (Scale Grouping paragraph; Proposition 1's column ranges)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits,sr", [(8, 1), (8, 0), (4, 1), (6, 0)])
def test_key_axis_quantizer_invariants(bits, sr):
    # one scale per key column: s_j = C_j / r with C_j = max_i |S_ij|; each column's
    # largest code is r; codes in [-r, r]
    d_k, d_v = 64, 48
    cfg = O.TileCfg(d_k, d_v, bits=bits, stochastic=sr, axis=1)
    r = 2 ** (bits - 1) - 1
    g = rng(70 + bits + sr)
    X = (g.standard_normal((d_v, d_k)) * np.exp(g.uniform(-6, 6, (1, d_k)))).astype(np.float32)
    X[:, 7] = 0.0                                     # an all-zero column
    codes, scales, flag = O.tile_quantize(cfg, X, O.tile_key(O.step_key(4, 1), 2))
    assert flag == 0 and scales.shape == (d_k,)
    C_ = O.unpack_codes(cfg, codes)
    assert C_.min() >= -r and C_.max() <= r
    for j in range(d_k):
        m = np.float32(np.abs(X[:, j]).max())
        if m == 0:
            assert scales[j] == 0 and not C_[:, j].any()
            continue
        assert scales[j] == np.float32(m * (np.float32(1) / np.float32(r)))
        assert np.abs(C_[:, j]).max() == r
        err = np.abs(C_[:, j] * np.float64(scales[j]) - X[:, j])
        assert err.max() <= (1.0 if sr else 0.5 + 2.0 ** -8) * float(scales[j]) * (1 + 1e-6)


def test_key_axis_quantized_step_matches_fp64_update():
    d_k, d_v, r = 32, 16, 127
    cfg = O.TileCfg(d_k, d_v, bits=8, delta=1, diag=1, axis=1)
    g = rng(71)
    ints = g.integers(-r, r + 1, (d_v, d_k))
    codes = O.pack_codes(cfg, ints)
    scales = g.uniform(0.01, 0.1, d_k).astype(np.float32)
    q, k, v, alpha, beta = draw(1, d_k, d_v, 72, diag=True)
    X = recur64(ints * scales.astype(np.float64)[None, :], alpha[0], k[0], v[0], beta[0], 1)
    o, flag, x = O.tile_step(cfg, codes, scales, q[0], k[0], v[0], alpha[0], beta[0], 5,
                             want_x=True)
    assert flag == 0
    np.testing.assert_allclose(x, X, rtol=0, atol=1e-5 * np.abs(X).max())
    np.testing.assert_allclose(o, X @ q[0].astype(np.float64), rtol=0, atol=1e-5 * np.abs(X).max())
    # and the stored state is the key-axis quantization of x
    c2, s2, _ = O.tile_quantize(cfg, x, 5)
    assert (c2 == codes).all() and (s2 == scales).all()


def test_key_axis_nonfinite_column_is_zeroed_and_flagged():
    cfg = O.TileCfg(32, 8, bits=8, axis=1)
    X = rng(73).standard_normal((8, 32)).astype(np.float32)
    X[3, 9] = np.nan
    X[5, 20] = np.float32(2.0 ** 101)
    codes, scales, flag = O.tile_quantize(cfg, X, 9)
    C_ = O.unpack_codes(cfg, codes)
    assert flag == 1
    for j in (9, 20):
        assert scales[j] == 0 and not C_[:, j].any()
    keep = [j for j in range(32) if j not in (9, 20)]
    assert (np.abs(C_[:, keep]).max(axis=0) == 127).all()


def test_proposition1_key_axis_readout_error():
    # RTN with one scale per key column: E[e_i^2] = sum_j q_j^2 C_j^2 / (12 r^2)
    d_k, d_v, n = 128, 32, 400
    cfg = O.TileCfg(d_k, d_v, bits=4, stochastic=0, axis=1)
    g = rng(74)
    num = 0.0
    den = 0.0
    for it in range(n):
        S = (g.standard_normal((d_v, d_k)) * g.uniform(0.1, 10, (1, d_k))).astype(np.float32)
        q = unit(g.standard_normal(d_k))
        codes, sc, _ = O.tile_quantize(cfg, S, 0)
        e = (O.tile_dequant(cfg, codes, sc).astype(np.float64) - S) @ q
        Cj = np.abs(S).max(axis=0).astype(np.float64)
        num += np.sum(e ** 2)
        den += d_v * np.sum(q ** 2 * Cj ** 2) / (12 * 7 ** 2)
    ratio = num / den
    assert 0.9 < ratio < 1.1, ratio


def test_value_axis_beats_key_axis_with_outlier_value_rows():
    # Scale Grouping paragraph: value-axis grouping is preferred at INT8; with a few large
    # value rows (outlier channels of v) a per-row scale keeps the other rows fine
    d_k, d_v = 64, 64
    g = rng(75)
    errs = {0: 0.0, 1: 0.0}
    for it in range(50):
        S = g.standard_normal((d_v, d_k)).astype(np.float32)
        S[g.choice(d_v, 4, replace=False)] *= 50.0
        q = unit(g.standard_normal(d_k))
        for axis in (0, 1):
            cfg = O.TileCfg(d_k, d_v, bits=8, stochastic=1, axis=axis)
            codes, sc, _ = O.tile_quantize(cfg, S, O.tile_key(O.step_key(it, 0), axis))
            e = (O.tile_dequant(cfg, codes, sc).astype(np.float64) - S) @ q
            errs[axis] += float(np.sum(e ** 2))
    assert errs[0] < 0.5 * errs[1], errs


# --------------------------------------------------------------------------
# Per-channel precision: a bit width per key group (the abstract's decay-based
# mixed precision across channels; value-axis scale groups of G columns)
# --------------------------------------------------------------------------

def test_group_bits_layout_worked_example():
    # d_k = 32, G = 16, groups at 8 and 4 bits: a row is 16 code bytes then 8 nibble bytes
    cfg = O.TileCfg(32, 1, group=16, group_bits=[8, 4])
    assert cfg.row_bytes() == 24 and cfg.code_bytes() == 24
    ints = np.array([[j - 10 for j in range(16)] + [1, -1, 7, -7, 0, 3, -3, 2, 5, -5, 6, -6, 4, -4, 1, 0]])
    b = O.pack_codes(cfg, ints)
    assert b[:16].view(np.int8).tolist() == list(range(-10, 6))
    # the int4 group packs like a 16-column int4 row (same worked bytes as the plain layout)
    assert b[16] == 0xF1 and b[17] == 0x97 and b[18] == 0x30 and b[19] == 0x2D
    assert (O.unpack_codes(cfg, b) == ints).all()
    # the other order: the nibble group first
    cfg2 = O.TileCfg(32, 1, group=16, group_bits=[4, 8])
    ints2 = np.concatenate([ints[:, 16:], ints[:, :16]], axis=1)
    b2 = O.pack_codes(cfg2, ints2)
    assert b2[:4].tolist() == [0xF1, 0x97, 0x30, 0x2D] and b2[8:].view(np.int8).tolist() == list(range(-10, 6))


@pytest.mark.parametrize("bits", [4, 5, 6, 8])
def test_uniform_group_bits_equal_plain_bits(bits):
    # every group at the same width gives exactly the plain layout and the same step
    d_k, d_v, G = 64, 8, 16
    plain = O.TileCfg(d_k, d_v, group=G, bits=bits, delta=1, diag=1)
    grp = O.TileCfg(d_k, d_v, group=G, group_bits=[bits] * (d_k // G), delta=1, diag=1)
    assert plain.code_bytes() == grp.code_bytes()
    g = rng(70 + bits)
    S = g.standard_normal((d_v, d_k)).astype(np.float32)
    tk = O.tile_key(O.step_key(5, 1), 2)
    c1, s1, _ = O.tile_quantize(plain, S, tk)
    c2, s2, _ = O.tile_quantize(grp, S, tk)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    q, k, v, alpha, beta = draw(1, d_k, d_v, 71, diag=True)
    o1, f1, _ = O.tile_step(plain, c1, s1, q[0], k[0], v[0], alpha[0], beta[0], tk)
    o2, f2, _ = O.tile_step(grp, c2, s2, q[0], k[0], v[0], alpha[0], beta[0], tk)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2) and np.array_equal(o1, o2)


@pytest.mark.parametrize("sr", [1, 0])
def test_group_bits_quantizer_invariants(sr):
    # each group follows Proposition 1 with its own r = 2^(b_g - 1) - 1
    d_k, d_v, G = 64, 32, 16
    gb = [8, 4, 6, 5]
    cfg = O.TileCfg(d_k, d_v, group=G, group_bits=gb, stochastic=sr)
    g = rng(73 + sr)
    X = (g.standard_normal((d_v, d_k)) * np.exp(g.uniform(-6, 6, (d_v, 1)))).astype(np.float32)
    X[2, 16:32] = 0.0                            # an all-zero int4 group
    codes, scales, flag = O.tile_quantize(cfg, X, O.tile_key(O.step_key(3, 9), 4))
    assert flag == 0
    C_ = O.unpack_codes(cfg, codes)
    for gi, b in enumerate(gb):
        r = (1 << (b - 1)) - 1
        for i in range(d_v):
            xs = X[i, gi * G:(gi + 1) * G]
            cs = C_[i, gi * G:(gi + 1) * G]
            m = np.float32(np.abs(xs).max())
            s = scales[i, gi]
            assert np.abs(cs).max() <= r
            if m == 0:
                assert s == 0 and not cs.any()
                continue
            assert s == np.float32(m * (np.float32(1) / np.float32(r)))
            assert np.abs(cs).max() == r
            err = np.abs(cs * np.float64(s) - xs)
            assert err.max() <= (1.0 if sr else 0.5 + 2.0 ** -8) * float(s) * (1 + 1e-6)
    # the dequantized tile is code times its group's scale
    D = O.tile_dequant(cfg, codes, scales)
    assert np.array_equal(D, (C_ * np.repeat(scales, G, axis=1)).astype(np.float32))


def test_group_bits_step_matches_fp64_update():
    d_k, d_v, G = 32, 12, 16
    gb = [4, 8]
    cfg = O.TileCfg(d_k, d_v, group=G, group_bits=gb, delta=1, diag=1)
    g = rng(75)
    ints = np.concatenate([g.integers(-7, 8, (d_v, 16)), g.integers(-127, 128, (d_v, 16))], axis=1)
    codes = O.pack_codes(cfg, ints)
    scales = g.uniform(0.01, 0.1, (d_v, 2)).astype(np.float32)
    q, k, v, alpha, beta = draw(1, d_k, d_v, 76, diag=True)
    S_hat = ints * np.repeat(scales.astype(np.float64), G, axis=1)
    X = recur64(S_hat, alpha[0], k[0], v[0], beta[0], 1)
    o, flag, x = O.tile_step(cfg, codes, scales, q[0], k[0], v[0], alpha[0], beta[0],
                             O.tile_key(O.step_key(1, 2), 3), want_x=True)
    assert flag == 0
    np.testing.assert_allclose(x, X, rtol=0, atol=1e-5 * np.abs(X).max())
    np.testing.assert_allclose(o, X @ q[0].astype(np.float64), rtol=0, atol=1e-5 * np.abs(X).max())
    # requantized: every entry within one step of its group's new scale
    C_ = O.unpack_codes(cfg, codes)
    err = np.abs(C_ * np.repeat(scales.astype(np.float64), G, axis=1) - x)
    assert (err <= np.repeat(scales.astype(np.float64), G, axis=1) * (1 + 1e-6)).all()


# --------------------------------------------------------------------------
# Dense 5- to 7-bit codes: offset binary split into 4-, 2- and 1-bit planes
# --------------------------------------------------------------------------

def test_dense_layout_worked_examples():
    # bytes written out by hand from the plane layout (16 columns, one row, padded to 16)
    cases = {
        6: ([-31, 31, 0, 1, -1, 15, -16, 16, 7, -7, 30, -30, 2, -2, 5, -5],
            [0xF1, 0x10, 0xFF, 0x00, 0x97, 0x2E, 0xE2, 0xB5, 0xC6, 0xA3, 0x96, 0xD6, 0, 0, 0, 0]),
        5: ([-15, 15, 0, 1, -1, 7, -8, 8, 3, -3, 14, -14, 2, -2, 5, -5],
            [0xF1, 0x10, 0x7F, 0x88, 0xD3, 0x2E, 0xE2, 0xB5, 0xF2, 0x0F, 0, 0, 0, 0, 0, 0]),
        7: ([-63, 63, 0, 1, -1, 31, -32, 32, 7, -7, 62, -62, 2, -2, 45, -45],
            [0xF1, 0x10, 0xFF, 0x00, 0x97, 0x2E, 0xE2, 0x3D, 0xCC, 0x03, 0x7C, 0xA6, 0xF2, 0x0F,
             0, 0]),
    }
    for bits, (ints, want) in cases.items():
        cfg = O.TileCfg(16, 1, bits=bits, dense=1)
        assert cfg.code_bytes() == 16
        b = O.pack_codes(cfg, np.array([ints]))
        assert b.tolist() == want, (bits, [hex(x) for x in b])
        assert (O.unpack_codes(cfg, b) == np.array([ints])).all()


@pytest.mark.parametrize("bits", [5, 6, 7])
def test_dense_round_trip_and_row_sizes(bits):
    r = (1 << (bits - 1)) - 1
    for d_k, row in ((16, 16), (32, {5: 24, 6: 24, 7: 32}[bits]), (128, 16 * bits)):
        cfg = O.TileCfg(d_k, 3, bits=bits, dense=1)
        assert cfg.code_bytes() == 3 * row
        ints = np.tile(np.arange(-r, r + 1), 3 * d_k)[:3 * d_k].reshape(3, d_k)
        assert (O.unpack_codes(cfg, O.pack_codes(cfg, ints)) == ints).all()


@pytest.mark.parametrize("bits", [5, 6, 7])
def test_dense_codes_equal_byte_codes(bits):
    # the layout does not change the arithmetic: the same state, step and dither give the
    # same codes and scales in either layout
    d_k, d_v, G = 64, 12, 32
    dense = O.TileCfg(d_k, d_v, group=G, bits=bits, dense=1, delta=1, diag=1)
    plain = O.TileCfg(d_k, d_v, group=G, bits=bits, delta=1, diag=1)
    g = rng(90 + bits)
    S = (g.standard_normal((d_v, d_k)) * np.exp(g.uniform(-3, 3, (d_v, 1)))).astype(np.float32)
    tk = O.tile_key(O.step_key(8, 2), 5)
    cd, sd, _ = O.tile_quantize(dense, S, tk)
    cp, sp, _ = O.tile_quantize(plain, S, tk)
    assert np.array_equal(sd, sp)
    assert np.array_equal(O.unpack_codes(dense, cd), O.unpack_codes(plain, cp))
    q, k, v, alpha, beta = draw(1, d_k, d_v, 91, diag=True)
    od, _, _ = O.tile_step(dense, cd, sd, q[0], k[0], v[0], alpha[0], beta[0], tk)
    op, _, _ = O.tile_step(plain, cp, sp, q[0], k[0], v[0], alpha[0], beta[0], tk)
    assert np.array_equal(od, op) and np.array_equal(sd, sp)
    assert np.array_equal(O.unpack_codes(dense, cd), O.unpack_codes(plain, cp))
