"""ctypes front end of the CPU oracle (test infrastructure only).

Every arithmetic step lives in lores_oracle.c; this module only moves numpy
arrays in and out and loops over tiles and steps.  Layouts follow the state
format: codes of one (sequence, head) tile are row-major [d_v][d_k] (int8) or
[d_v][d_k/2] bytes (int4, even column in the low nibble); scales are
[d_v][d_k/G] fp32; the fp32 state is [d_v][d_k].
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


class LoCfg(C.Structure):
    _fields_ = [("d_k", C.c_int), ("d_v", C.c_int), ("group", C.c_int), ("bits", C.c_int),
                ("delta", C.c_int), ("diag", C.c_int), ("stochastic", C.c_int),
                ("axis", C.c_int), ("group_bits", C.c_void_p), ("dense", C.c_int)]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        L.lo_splitmix64.restype = C.c_uint64
        L.lo_splitmix64.argtypes = [C.c_uint64]
        L.lo_fmix32.restype = C.c_uint32
        L.lo_fmix32.argtypes = [C.c_uint32]
        L.lo_step_key.restype = C.c_uint32
        L.lo_step_key.argtypes = [C.c_uint64, C.c_uint64]
        L.lo_tile_key.restype = C.c_uint32
        L.lo_tile_key.argtypes = [C.c_uint32, C.c_uint32]
        L.lo_mulfold.restype = C.c_uint32
        L.lo_mulfold.argtypes = [C.c_uint32, C.c_uint32]
        L.lo_dither_word.restype = C.c_uint32
        L.lo_dither_word.argtypes = [C.c_uint32, C.c_int]
        L.lo_dither_words.restype = None
        L.lo_dither_words.argtypes = [C.c_uint32, C.c_uint32, C.c_int, C.c_void_p]
        L.lo_dither.restype = C.c_uint32
        L.lo_dither.argtypes = [C.c_uint32, C.c_int, C.c_int, C.c_int]
        L.lo_dot_b16.restype = C.c_float
        L.lo_dot_b16.argtypes = [C.c_void_p, C.c_void_p, C.c_int]
        L.lo_fixed_point.restype = C.c_int
        L.lo_fixed_point.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_void_p,
                                     C.POINTER(C.c_int)]
        L.lo_exact_projection.restype = C.c_float
        L.lo_exact_projection.argtypes = [C.POINTER(LoCfg), C.c_void_p, C.c_float, C.c_int,
                                          C.c_void_p, C.c_int]
        L.lo_recip_nr.restype = C.c_float
        L.lo_recip_nr.argtypes = [C.c_float]
        L.lo_get_code.restype = C.c_int
        L.lo_get_code.argtypes = [C.POINTER(LoCfg), C.c_void_p, C.c_int, C.c_int]
        L.lo_put_code.restype = None
        L.lo_put_code.argtypes = [C.POINTER(LoCfg), C.c_void_p, C.c_int, C.c_int, C.c_int]
        L.lo_tile_step.restype = C.c_int
        L.lo_tile_step.argtypes = [C.POINTER(LoCfg), C.c_void_p, C.c_void_p, C.c_void_p,
                                   C.c_void_p, C.c_void_p, C.c_void_p, C.c_float, C.c_uint32,
                                   C.c_void_p, C.c_void_p]
        L.lo_tile_step_plain.restype = C.c_int
        L.lo_tile_step_plain.argtypes = L.lo_tile_step.argtypes
        L.lo_tile_quantize.restype = C.c_int
        L.lo_tile_quantize.argtypes = [C.POINTER(LoCfg), C.c_void_p, C.c_void_p, C.c_void_p,
                                       C.c_uint32]
        L.lo_tile_dequant.restype = None
        L.lo_tile_dequant.argtypes = [C.POINTER(LoCfg), C.c_void_p, C.c_void_p, C.c_void_p]
        L.lo_assign_bits_by_decay.restype = None
        L.lo_assign_bits_by_decay.argtypes = [C.c_void_p, C.c_int, C.c_float, C.c_int, C.c_int,
                                              C.c_void_p]
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p)


def _f32(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a


class TileCfg:
    """Shape and recipe of one (sequence, head) tile."""

    def __init__(self, d_k, d_v, group=None, bits=8, delta=1, diag=0, stochastic=1, axis=0,
                 group_bits=None, dense=0):
        self.d_k, self.d_v = int(d_k), int(d_v)
        self.group = int(group if group else d_k)
        self.bits, self.delta, self.diag, self.stochastic = int(bits), int(delta), int(diag), int(stochastic)
        self.axis = int(axis)
        # per-channel precision: bits of each key group (the `bits` field is then unused)
        self.group_bits = None
        gb = None
        if group_bits is not None:
            self.group_bits = np.ascontiguousarray(group_bits, dtype=np.int32)
            assert self.group_bits.shape == (self.d_k // self.group,) and not self.axis
            self.bits = 0
            gb = self.group_bits.ctypes.data_as(C.c_void_p)
        # dense: 5- to 7-bit codes in bit planes instead of one byte each
        self.dense = int(bool(dense) and group_bits is None and 5 <= self.bits <= 7)
        self.c = LoCfg(self.d_k, self.d_v, self.group, self.bits, self.delta, self.diag,
                       self.stochastic, self.axis, gb, self.dense)

    @property
    def n_groups(self):
        return self.d_k // self.group

    def scale_shape(self):
        """value axis: [d_v, d_k/G]; key axis: [d_k] (one scale per key column)."""
        return (self.d_k,) if self.axis else (self.d_v, self.n_groups)

    def row_bytes(self):
        """Bytes of one quantized row: key groups back to back, each G * storage / 8."""
        if self.group_bits is not None:
            return sum(self.group * (4 if b == 4 else 8) // 8 for b in self.group_bits)
        return self.code_bytes() // self.d_v

    def code_bytes(self):
        if self.group_bits is not None:
            return self.d_v * self.row_bytes()
        if self.dense:
            return self.d_v * ((self.d_k * self.bits // 8 + 7) // 8 * 8)
        if self.bits == 32:
            return self.d_v * self.d_k * 4
        if self.bits == 4:
            return self.d_v * self.d_k // 2
        return self.d_v * self.d_k          # 5 to 8 bits: one byte per code

    def zero_state(self):
        """(state, scales) of an all-zero tile."""
        if self.bits == 32:
            return np.zeros((self.d_v, self.d_k), np.float32), np.zeros(self.scale_shape(), np.float32)
        return (np.zeros(self.code_bytes(), np.uint8), np.zeros(self.scale_shape(), np.float32))


# --- random bits ------------------------------------------------------------

def splitmix64(z):
    return int(lib().lo_splitmix64(z & (2**64 - 1)))


def fmix32(h):
    return int(lib().lo_fmix32(h & 0xFFFFFFFF))


def step_key(seed, step):
    return int(lib().lo_step_key(seed & (2**64 - 1), step & (2**64 - 1)))


def tile_key(skey, tile_index):
    return int(lib().lo_tile_key(skey, tile_index & 0xFFFFFFFF))


def mulfold(a, b):
    return int(lib().lo_mulfold(a & 0xFFFFFFFF, b & 0xFFFFFFFF))


def dither_word(c, q):
    """Word q of the 16-column block whose counter is c."""
    return int(lib().lo_dither_word(c & 0xFFFFFFFF, int(q)))


def dither_words(tkey, n0, count):
    """Dither words of quads n0 .. n0 + count - 1 of a tile (uint32 array)."""
    out = np.empty(count, np.uint32)
    lib().lo_dither_words(tkey & 0xFFFFFFFF, n0 & 0xFFFFFFFF, count, _p(out))
    return out


def dither(tkey, d_k, i, j):
    return int(lib().lo_dither(tkey, d_k, i, j))


def dot_b16(a, b):
    a, b = _f32(a), _f32(b)
    return float(lib().lo_dot_b16(_p(a), _p(b), a.size))


def fixed_point(alpha, y, diag):
    """(ok, Y, E): the fixed-point copy Y_j = rint(alpha_j y_j 2^E) of the exact projection."""
    a, yy = _f32(np.atleast_1d(alpha)), _f32(y)
    Y = np.zeros(yy.size, np.int32)
    E = C.c_int(0)
    ok = lib().lo_fixed_point(_p(a), int(diag), _p(yy), yy.size, _p(Y), C.byref(E))
    return bool(ok), Y, int(E.value)


def exact_projection(cfg, codes, s, i, Y, E):
    """u_i of the exact projection for row i of a head's codes (one scale s per row)."""
    Y = np.ascontiguousarray(Y, np.int32)
    return float(np.float32(lib().lo_exact_projection(C.byref(cfg.c), _p(codes), float(np.float32(s)),
                                                      int(i), _p(Y), int(E))))


def recip_nr(m):
    return float(np.float32(lib().lo_recip_nr(float(np.float32(m)))))


# --- codes ------------------------------------------------------------------

def unpack_codes(cfg: TileCfg, codes):
    """Packed tile bytes -> int array [d_v, d_k] (int8 or int4 layouts)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty((cfg.d_v, cfg.d_k), np.int32)
    L = lib()
    for i in range(cfg.d_v):
        for j in range(cfg.d_k):
            out[i, j] = L.lo_get_code(C.byref(cfg.c), _p(codes), i, j)
    return out


def pack_codes(cfg: TileCfg, ints):
    """int array [d_v, d_k] -> packed tile bytes."""
    codes = np.zeros(cfg.code_bytes(), np.uint8)
    L = lib()
    for i in range(cfg.d_v):
        for j in range(cfg.d_k):
            L.lo_put_code(C.byref(cfg.c), _p(codes), i, j, int(ints[i, j]))
    return codes


# --- steps ------------------------------------------------------------------

def tile_step(cfg: TileCfg, state, scales, q, k, v, alpha, beta, tkey, want_x=False):
    """One decode step of one tile, in place on (state, scales).

    Returns (o [d_v] float64, flag, x or None)."""
    assert state.flags.c_contiguous and scales.flags.c_contiguous
    q, k, v = _f32(q), _f32(k), _f32(v)
    alpha = _f32(np.atleast_1d(alpha))
    o = np.empty(cfg.d_v, np.float64)
    x = np.empty((cfg.d_v, cfg.d_k), np.float32) if want_x else None
    flag = lib().lo_tile_step(C.byref(cfg.c), _p(state), _p(scales), _p(q), _p(k), _p(v),
                              _p(alpha), float(np.float32(beta)), tkey, _p(o),
                              _p(x) if want_x else None)
    return o, int(flag), x


def tile_step_plain(cfg: TileCfg, state, scales, q, k, v, alpha, beta, tkey, want_x=False):
    """The plain definition of the same step (double precision, plain division and
    floor; see lo_tile_step_plain).  Same arguments and results as tile_step."""
    assert state.flags.c_contiguous and scales.flags.c_contiguous
    q, k, v = _f32(q), _f32(k), _f32(v)
    alpha = _f32(np.atleast_1d(alpha))
    o = np.empty(cfg.d_v, np.float64)
    x = np.empty((cfg.d_v, cfg.d_k), np.float32) if want_x else None
    flag = lib().lo_tile_step_plain(C.byref(cfg.c), _p(state), _p(scales), _p(q), _p(k), _p(v),
                                    _p(alpha), float(np.float32(beta)), tkey, _p(o),
                                    _p(x) if want_x else None)
    return o, int(flag), x


def tile_quantize(cfg: TileCfg, S, tkey):
    S = _f32(S)
    codes = np.zeros(cfg.code_bytes(), np.uint8)
    scales = np.zeros(cfg.scale_shape(), np.float32)
    flag = lib().lo_tile_quantize(C.byref(cfg.c), _p(S), _p(codes), _p(scales), tkey)
    return codes, scales, int(flag)


def tile_dequant(cfg: TileCfg, codes, scales):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = _f32(scales)
    S = np.empty((cfg.d_v, cfg.d_k), np.float32)
    lib().lo_tile_dequant(C.byref(cfg.c), _p(codes), _p(scales), _p(S))
    return S


_lib_omp = None


def lib_omp():
    """The oracle built with its OpenMP tile loop (lores_oracle_omp.c)."""
    global _lib_omp
    if _lib_omp is None:
        L = C.CDLL(_build.build_omp())
        L.lo_batch_step.restype = C.c_int
        L.lo_batch_step.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                                    C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                    C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p,
                                    C.c_void_p, C.c_int]
        _lib_omp = L
    return _lib_omp


def batch_step(cfgs, cfg_of, states, scales, q, k, v, alpha, beta, tile_keys, threads=0):
    """One decode step of n tiles on all host cores: tile t is lo_tile_step with
    cfgs[cfg_of[t]], states[t], scales[t] (in place) and row t of q, k, v [n, d], alpha
    [n, 1 or d_k], beta [n], tile_keys [n].  Returns (o [n, d_v] float64, flags [n], the
    number of threads used)."""
    n = len(states)
    d_k, d_v = cfgs[0].d_k, cfgs[0].d_v
    q, k, v = _f32(q).reshape(n, d_k), _f32(k).reshape(n, d_k), _f32(v).reshape(n, d_v)
    alpha = _f32(alpha).reshape(n, -1)
    beta = _f32(beta).reshape(n)
    keys = np.ascontiguousarray(tile_keys, dtype=np.uint32)
    cfg_ptrs = (C.c_void_p * len(cfgs))(*[C.cast(C.pointer(c.c), C.c_void_p) for c in cfgs])
    idx = np.ascontiguousarray(cfg_of, dtype=np.int32)
    sp = (C.c_void_p * n)(*[st.ctypes.data for st in states])
    scp = (C.c_void_p * n)(*[sc.ctypes.data for sc in scales])
    o = np.empty((n, d_v), np.float64)
    flags = np.zeros(n, np.int32)
    used = lib_omp().lo_batch_step(cfg_ptrs, _p(idx), n, sp, scp, _p(q), _p(k), _p(v),
                                   _p(alpha), _p(beta), _p(keys), d_k, d_v, alpha.shape[1],
                                   _p(o), _p(flags), int(threads))
    return o, flags, int(used)


def assign_bits_by_decay(mean_decay, frac_high, bits_high=8, bits_low=4):
    d = _f32(mean_decay)
    out = np.empty(d.size, np.int32)
    lib().lo_assign_bits_by_decay(_p(d), d.size, float(frac_high), bits_high, bits_low, _p(out))
    return out
