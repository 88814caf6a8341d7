"""The C-ABI library loads and exports every symbol include/lores.h declares, and its
host-only logic (validation, status strings, the decay-based precision policy)
behaves as specified.  No compute call runs here (no GPU is needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "lores.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lores_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    from bit_recurrent_state_lores_b200 import lores as L
    names = declared_functions()
    assert len(names) >= 12, names
    lib = ctypes.CDLL(L.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"liblores.so does not export {n}"
    assert "lores_decode_step" in names and "lores_create" in names
    assert lib.lores_index_checked() == 0


def test_checked_library_exports_the_same_symbols():
    """The index-checked debugging build (when built) exports the same ABI and says so."""
    from bit_recurrent_state_lores_b200 import lores as L
    if not os.path.exists(L.CHECKED_LIB_PATH):
        pytest.skip("liblores_checked.so is not built")
    lib = L.load_library(L.CHECKED_LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), f"liblores_checked.so does not export {n}"
    assert lib.lores_index_checked() == 1
    assert lib.lores_debug_trim_range(None, 0, 0) == L.LORES_ERR_INVALID_ARG
    assert lib.lores_debug_last_flags(None, None) == L.LORES_ERR_INVALID_ARG


def test_status_strings():
    from bit_recurrent_state_lores_b200 import lores as L
    for s in range(9):
        assert L.lores_status_string(s) and "unknown" not in L.lores_status_string(s)
    assert "unknown" in L.lores_status_string(99)


@pytest.mark.parametrize("kw", [
    dict(batch=0), dict(heads=0), dict(d_k=48), dict(d_k=512), dict(d_v=6), dict(d_v=0),
    dict(d_v=8192), dict(group_size=8), dict(group_size=48), dict(delta=2), dict(decay_diag=3),
    dict(stochastic=5), dict(head_bits=[8, 3]), dict(head_bits=[9, 8]), dict(head_bits=[16, 8]),
    dict(device=-1), dict(scale_axis=2), dict(scale_axis=-1), dict(scale_axis=1, group_size=16),
    dict(group_size=32, group_bits=[[8, 4], [4, 4]], head_bits=[8, 8]),
    dict(group_size=32, group_bits=[[8, 3], [4, 4]]), dict(group_size=32, group_bits=[[8, 9], [4, 4]]),
    dict(scale_axis=1, group_size=64, group_bits=[[8], [8]]), dict(dense_codes=2),
    dict(dense_codes=1, group_size=32, group_bits=[[6, 6], [6, 6]]),
    dict(dense_codes=1, scale_axis=1, head_bits=[6, 6])])
def test_create_rejects_bad_config_before_touching_cuda(kw):
    from bit_recurrent_state_lores_b200 import lores as L
    args = dict(batch=2, heads=2, d_k=64, d_v=16)
    args.update(kw)
    with pytest.raises(L.LoresError) as e:
        L.lores_create(**args)
    assert e.value.status == L.LORES_ERR_INVALID_ARG


def test_noalloc_rejects_group_bits_before_touching_cuda():
    import ctypes as C
    from bit_recurrent_state_lores_b200 import lores as L
    cfg = L.make_config(1, 1, 64, 64, group_size=32, group_bits=[[8, 4]])
    a = 0x10000
    assert L.raw_library().lores_decode_step_noalloc(C.byref(cfg), a, a, a, a, a, a, a, a, 0,
                                                     None, None) == L.LORES_ERR_UNSUPPORTED


def test_noalloc_rejects_dense_codes_before_touching_cuda():
    import ctypes as C
    from bit_recurrent_state_lores_b200 import lores as L
    cfg = L.make_config(1, 1, 64, 64, head_bits=[6], dense_codes=1)
    a = 0x10000
    assert L.raw_library().lores_decode_step_noalloc(C.byref(cfg), a, a, a, a, a, a, a, a, 0,
                                                     None, None) == L.LORES_ERR_UNSUPPORTED


def test_noalloc_rejects_key_axis_before_touching_cuda():
    # validation returns before any pointer is used, so plain aligned addresses do
    import ctypes as C
    from bit_recurrent_state_lores_b200 import lores as L
    cfg = L.make_config(1, 1, 64, 64, group_size=64, scale_axis=1)
    raw = L.raw_library()
    a = 0x10000
    rc = raw.lores_decode_step_noalloc(C.byref(cfg), a, a, a, a, a, a, a, a, 0, None, None)
    assert rc == L.LORES_ERR_UNSUPPORTED


def test_null_handle_calls_are_rejected():
    from bit_recurrent_state_lores_b200 import lores as L
    lib = L.raw_library()
    assert lib.lores_destroy(None) == L.LORES_OK
    assert lib.lores_decode_step(None, 16, 16, 16, 16, 16, 16, 0, None) == L.LORES_ERR_INVALID_ARG
    assert lib.lores_dequant_state(None, 16, None) == L.LORES_ERR_INVALID_ARG
    assert lib.lores_check_errors(None, None) == L.LORES_ERR_INVALID_ARG
    assert lib.lores_get_layout(None, None, None) == L.LORES_ERR_INVALID_ARG


def test_policy_matches_oracle_policy():
    # two independent implementations of the decay-based precision map agree
    from bit_recurrent_state_lores_b200 import lores as L
    g = np.random.default_rng(0)
    for H in (1, 2, 7, 32, 64):
        for frac in (0.0, 0.25, 0.5, 0.37, 1.0):
            d = g.uniform(0.3, 1.0, H).astype(np.float32)
            d[g.integers(H)] = d[0]                 # a tie
            assert L.lores_assign_bits_by_decay(d, frac) == O.assign_bits_by_decay(d, frac).tolist()


def test_policy_rejects_bad_arguments():
    from bit_recurrent_state_lores_b200 import lores as L
    for args in [([0.5], 1.5), ([0.5], -0.1)]:
        with pytest.raises(L.LoresError):
            L.lores_assign_bits_by_decay(*args)
    with pytest.raises(L.LoresError):
        L.lores_assign_bits_by_decay([0.5, 0.6], 0.5, bits_high=3)
    assert L.lores_assign_bits_by_decay([0.5, 0.6], 0.5, bits_high=6, bits_low=4) == [4, 6]


def test_fast_unpack_matches_oracle_unpack():
    from tests.harness import unpack_fast
    g = np.random.default_rng(1)
    for bits, r in ((8, 127), (4, 7)):
        cfg = O.TileCfg(32, 8, bits=bits)
        ints = g.integers(-r, r + 1, (8, 32))
        b = O.pack_codes(cfg, ints)
        assert (unpack_fast(cfg, b) == ints).all()
