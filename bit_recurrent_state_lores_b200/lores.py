"""Thin ctypes binding of liblores.so (include/lores.h): same names, argument
marshalling only.  Every step of the decode path runs in the library's kernels.

Pointers may be given as ints or as torch tensors (their data_ptr() is passed);
`stream` may be a torch.cuda.Stream, an int handle, or None for the current torch
stream.  A non-OK status raises LoresError, except from lores_check_errors, which
returns the status so that callers can test for NONFINITE.
"""
import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblores.so")
# the index-checked build of the same sources (a debugging aid, not the product)
CHECKED_LIB_PATH = os.path.join(_PKG, "liblores_checked.so")

LORES_OK = 0
LORES_ERR_INVALID_ARG = 1
LORES_ERR_OOM = 2
LORES_ERR_CUDA = 3
LORES_ERR_NONFINITE = 4
LORES_ERR_UNSUPPORTED = 5
LORES_ERR_TIMEOUT = 6
LORES_ERR_CORRUPT = 7
LORES_ERR_INDEX = 8


class LoresError(RuntimeError):
    def __init__(self, status, where):
        self.status = int(status)
        super().__init__(f"{where}: {lores_status_string(status)} ({status})")


class lores_config(C.Structure):
    _fields_ = [("batch", C.c_int32), ("heads", C.c_int32), ("d_k", C.c_int32),
                ("d_v", C.c_int32), ("group_size", C.c_int32), ("delta", C.c_int32),
                ("decay_diag", C.c_int32), ("head_bits", C.POINTER(C.c_int32)),
                ("stochastic", C.c_int32), ("seed", C.c_uint64), ("device", C.c_int32),
                ("scale_axis", C.c_int32), ("group_bits", C.POINTER(C.c_int32)),
                ("dense_codes", C.c_int32)]


class lores_layout(C.Structure):
    _fields_ = [("code_bytes", C.c_int64), ("seq_code_bytes", C.c_int64),
                ("scale_count", C.c_int64), ("n_groups", C.c_int32),
                ("units_per_step", C.c_int32), ("grid", C.c_int32), ("smem_bytes", C.c_int32),
                ("codes_dev", C.c_void_p), ("scales_dev", C.c_void_p),
                ("step_kernel", C.c_int32)]


def load_library(path=LIB_PATH):
    """Load a build of the library (the product, or CHECKED_LIB_PATH) and declare its
    signatures.  The functions below call the module's `_lib`; a caller that wants the
    index-checked build swaps it in before creating handles."""
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run `python -m "
                          "bit_recurrent_state_lores_b200.build` (needs nvcc)")
    L = C.CDLL(path)
    P, U64, I32, F32 = C.c_void_p, C.c_uint64, C.c_int32, C.c_float
    sig = {
        "lores_create": (I32, [C.POINTER(lores_config), C.POINTER(P)]),
        "lores_destroy": (I32, [P]),
        "lores_decode_step": (I32, [P, P, P, P, P, P, P, U64, P]),
        "lores_decode_step_host": (I32, [P, P, P, P, P, P, P, U64, P]),
        "lores_decode_step_host_async": (I32, [P, P, P, P, P, P, P, U64, P]),
        "lores_decode_steps": (I32, [P, I32, P, P, P, P, P, P, U64, P]),
        "lores_decode_step_dev": (I32, [P, P, P, P, P, P, P, P, P]),
        "lores_advance_step": (I32, [P, U64, P]),
        "lores_decode_step_noalloc": (I32, [C.POINTER(lores_config), P, P, P, P, P, P, P, P, U64,
                                            P, P]),
        "lores_dequant_state": (I32, [P, P, P]),
        "lores_load_state": (I32, [P, P, U64, P]),
        "lores_export_codes": (I32, [P, P, P, P]),
        "lores_load_codes": (I32, [P, P, P, P]),
        "lores_get_layout": (I32, [P, C.POINTER(lores_layout), P]),
        "lores_check_errors": (I32, [P, P]),
        "lores_set_fault_injection": (I32, [P, I32, I32, C.c_uint32]),
        "lores_assign_bits_by_decay": (I32, [P, I32, F32, I32, I32, P]),
        "lores_status_string": (C.c_char_p, [I32]),
        "lores_index_checked": (I32, []),
        "lores_debug_trim_range": (I32, [P, I32, U64]),
        "lores_debug_last_flags": (I32, [P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    return L


_lib = load_library()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):            # numpy array (host memory)
        return x.ctypes.data
    raise TypeError(f"cannot pass {type(x)} as a pointer")


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st, where):
    if st != LORES_OK:
        raise LoresError(st, where)


def lores_status_string(status):
    return _lib.lores_status_string(int(status)).decode()


def lores_create(batch, heads, d_k, d_v, group_size=0, delta=1, decay_diag=0, head_bits=None,
                 stochastic=1, seed=0, device=0, scale_axis=0, group_bits=None, dense_codes=0):
    """Returns an opaque handle (int).  group_bits: None or [H][d_k/G] bits per key group;
    dense_codes: 5- to 7-bit codes in bit planes instead of one byte each."""
    cfg = make_config(batch, heads, d_k, d_v, group_size, delta, decay_diag, head_bits,
                      stochastic, seed, device, scale_axis, group_bits, dense_codes)
    out = C.c_void_p()
    _check(_lib.lores_create(C.byref(cfg), C.byref(out)), "lores_create")
    return out.value


def lores_destroy(h):
    _check(_lib.lores_destroy(h), "lores_destroy")


def lores_decode_step(h, q, k, v, alpha, beta, o, step, stream=None):
    _check(_lib.lores_decode_step(h, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                  _ptr(o), step & (2**64 - 1), _stream(stream)),
           "lores_decode_step")


def lores_decode_step_dev(h, q, k, v, alpha, beta, o, step, stream=None):
    """The step with its counter in device memory (`step`: int64 tensor of one element)."""
    _check(_lib.lores_decode_step_dev(h, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                      _ptr(o), _ptr(step), _stream(stream)),
           "lores_decode_step_dev")


def lores_advance_step(step, n=1, stream=None):
    _check(_lib.lores_advance_step(_ptr(step), n & (2**64 - 1), _stream(stream)),
           "lores_advance_step")


def lores_decode_steps(h, T, q, k, v, alpha, beta, o, step0, stream=None):
    """T consecutive tokens in one call; inputs token-major [T, B, H, ...]."""
    _check(_lib.lores_decode_steps(h, int(T), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                   _ptr(o), step0 & (2**64 - 1), _stream(stream)),
           "lores_decode_steps")


def lores_decode_step_host_async(h, q, k, v, alpha, beta, o, step, stream=None):
    """Host-buffer step, enqueued only (pinned buffers; o valid when the stream gets there)."""
    _check(_lib.lores_decode_step_host_async(h, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                             _ptr(beta), _ptr(o), step & (2**64 - 1),
                                             _stream(stream)),
           "lores_decode_step_host_async")


def lores_decode_step_host(h, q, k, v, alpha, beta, o, step, stream=None):
    _check(_lib.lores_decode_step_host(h, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                       _ptr(o), step & (2**64 - 1), _stream(stream)),
           "lores_decode_step_host")


def lores_decode_step_noalloc(cfg, codes, scales, q, k, v, alpha, beta, o, step,
                              flags_out=None, stream=None):
    """The decode step on caller-owned state buffers, allocating nothing (see
    include/lores.h).  `cfg` is a lores_config (make_config builds one)."""
    _check(_lib.lores_decode_step_noalloc(C.byref(cfg), _ptr(codes), _ptr(scales), _ptr(q),
                                          _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o),
                                          step & (2**64 - 1), _ptr(flags_out), _stream(stream)),
           "lores_decode_step_noalloc")


def make_config(batch, heads, d_k, d_v, group_size=0, delta=1, decay_diag=0, head_bits=None,
                stochastic=1, seed=0, device=0, scale_axis=0, group_bits=None, dense_codes=0):
    """A lores_config; the bit arrays are kept alive on the returned object."""
    hb = gb = None
    arr = garr = None
    if head_bits is not None:
        arr = (C.c_int32 * heads)(*[int(b) for b in head_bits])
        hb = C.cast(arr, C.POINTER(C.c_int32))
    if group_bits is not None:
        flat = [int(b) for row in group_bits for b in row]
        garr = (C.c_int32 * len(flat))(*flat)
        gb = C.cast(garr, C.POINTER(C.c_int32))
    cfg = lores_config(batch, heads, d_k, d_v, group_size, delta, decay_diag, hb, stochastic,
                       seed & (2**64 - 1), device, scale_axis, gb, dense_codes)
    cfg._keepalive = (arr, garr)
    return cfg


def lores_dequant_state(h, out, stream=None):
    _check(_lib.lores_dequant_state(h, _ptr(out), _stream(stream)), "lores_dequant_state")


def lores_load_state(h, S, step, stream=None):
    _check(_lib.lores_load_state(h, _ptr(S), step & (2**64 - 1), _stream(stream)),
           "lores_load_state")


def lores_export_codes(h, codes, scales, stream=None):
    _check(_lib.lores_export_codes(h, _ptr(codes), _ptr(scales), _stream(stream)),
           "lores_export_codes")


def lores_load_codes(h, codes, scales, stream=None):
    _check(_lib.lores_load_codes(h, _ptr(codes), _ptr(scales), _stream(stream)),
           "lores_load_codes")


def lores_get_layout(h, heads=None):
    """Returns (lores_layout, head_offsets list or None)."""
    lay = lores_layout()
    offs = (C.c_int64 * heads)() if heads else None
    _check(_lib.lores_get_layout(h, C.byref(lay), C.cast(offs, C.c_void_p) if offs else None),
           "lores_get_layout")
    return lay, (list(offs) if offs else None)


def lores_check_errors(h, stream=None):
    """Returns the status (LORES_OK, LORES_ERR_NONFINITE, LORES_ERR_TIMEOUT,
    LORES_ERR_CORRUPT or LORES_ERR_INDEX); raises on other failures."""
    st = _lib.lores_check_errors(h, _stream(stream))
    if st not in (LORES_OK, LORES_ERR_NONFINITE, LORES_ERR_TIMEOUT, LORES_ERR_CORRUPT,
                  LORES_ERR_INDEX):
        raise LoresError(st, "lores_check_errors")
    return st


def lores_set_fault_injection(h, seq, unit=0, wait_us=0):
    """Testing hook of the failure path: withhold the copies of unit `unit` of sequence
    `seq` (-1: none) and bound every wait by `wait_us` microseconds (0: the default)."""
    _check(_lib.lores_set_fault_injection(h, int(seq), int(unit), int(wait_us)),
           "lores_set_fault_injection")


def lores_index_checked():
    """True in the index-checked build."""
    return bool(_lib.lores_index_checked())


def lores_debug_trim_range(h, which, nbytes):
    """Index-checked build: declare buffer `which` (0 codes, 1 scales, 2 q, 3 k, 4 v,
    5 alpha, 6 beta, 7 o, 8 the fp32 state) `nbytes` shorter on later launches of h."""
    _check(_lib.lores_debug_trim_range(h, int(which), int(nbytes)), "lores_debug_trim_range")


def lores_debug_last_flags(h):
    """The raw error word the last lores_check_errors on h read."""
    f = C.c_uint32()
    _check(_lib.lores_debug_last_flags(h, C.byref(f)), "lores_debug_last_flags")
    return f.value


def lores_assign_bits_by_decay(mean_decay, frac_high, bits_high=8, bits_low=4):
    H = len(mean_decay)
    d = (C.c_float * H)(*[float(x) for x in mean_decay])
    out = (C.c_int32 * H)()
    _check(_lib.lores_assign_bits_by_decay(C.cast(d, C.c_void_p), H, float(frac_high), bits_high,
                                           bits_low, C.cast(out, C.c_void_p)),
           "lores_assign_bits_by_decay")
    return list(out)


def raw_library():
    """The loaded CDLL (for callers that marshal arguments themselves)."""
    return _lib
