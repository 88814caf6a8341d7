"""The index-checked build (liblores_checked.so: the library compiled with
LORES_INDEX_CHECKS), a stand-in for a memory sanitizer.

In that build every global access of the decode, loader and dequantizer kernels is checked
against the extent of the buffer it belongs to before it runs; an access outside is
skipped and raises the INDEX flag with the buffer's bit.  Two kinds of test:
- every kernel family (tensor-core, two-rows-per-lane, general, key-axis, dense bit planes,
  per-channel widths; single and multi-token steps; the loader and the dequantizer) runs
  in both builds from the same seeds: codes, scales and outputs agree bit for bit, and the
  checked build raises no flag;
- a buffer declared a little shorter than it is (lores_debug_trim_range: the memory is
  untouched, so nothing can fault) makes the checks see the accesses at its end as out of
  range: the call reports LORES_ERR_INDEX with that buffer's bit, and exactly the accesses
  past the declared end are skipped.
"""
import numpy as np
import pytest
import torch

from bit_recurrent_state_lores_b200 import synth

from .harness import GpuRun

pytestmark = pytest.mark.gpu

# buffer numbers of lores_debug_trim_range / the flag bits 8 + n
CODES, SCALES, Q, K, V, ALPHA, BETA, O, STATE = range(9)
INDEX_BIT = 4


def lib():
    from bit_recurrent_state_lores_b200 import lores
    return lores


@pytest.fixture(scope="module")
def checked_lib():
    from bit_recurrent_state_lores_b200 import build
    L = lib()
    lb = L.load_library(build.build(checked=True))
    assert lb.lores_index_checked() == 1
    return lb


@pytest.fixture
def use_checked(checked_lib, monkeypatch):
    """Swap the binding over to the checked build for one test."""
    def swap(on):
        monkeypatch.setattr(lib(), "_lib", checked_lib if on else lib().load_library())
    return swap


def group_bits_of(H, ng, seed):
    rng = np.random.default_rng(seed)
    return [[int(rng.choice([4, 8])) for _ in range(ng)] for _ in range(H)]


# (name, workload, head bits, GpuRun keyword arguments, expected step_kernel)
CASES = [
    ("tensor-core", synth.Workload("ic-mma", B=96, H=6, d_k=128, d_v=128, steps=3, decay="tau",
                                   group=128, outliers=2, seed=31), [8, 4, 8, 4, 8, 8], {}, 3),
    ("two-rows-per-lane", synth.Workload("ic-pair", B=96, H=6, d_k=128, d_v=128, steps=3,
                                         decay="tau", group=32, outliers=2, seed=32),
     [8, 4, 8, 4, 8, 8], {}, 1),
    ("general", synth.Workload("ic-gen", B=3, H=3, d_k=64, d_v=40, steps=3, decay="tau",
                               group=16, outliers=2, seed=33), [8, 32, 4], {}, 0),
    ("key-axis", synth.Workload("ic-key", B=3, H=3, d_k=32, d_v=24, steps=3, decay="tau",
                                outliers=2, seed=34), [8, 4, 32], {"axis": 1}, 2),
    ("dense", synth.Workload("ic-dense", B=2, H=3, d_k=64, d_v=24, steps=3, decay="tau",
                             group=32, outliers=2, seed=35), [5, 6, 7], {"dense": 1}, 0),
    ("per-channel", synth.Workload("ic-chan", B=2, H=3, d_k=64, d_v=24, steps=3, decay="kda",
                                   delta=1, diag=1, group=16, outliers=2, seed=36), [8, 8, 8],
     {"group_bits": group_bits_of(3, 4, 7)}, 0),
]


def run_case(wl, bits, kw, kernel):
    """Loader, three single steps, one three-token call, the dequantizer; returns every
    output and the error status of each phase."""
    L = lib()
    g = GpuRun(wl, bits, seed=9, **kw)
    try:
        assert g.layout.step_kernel == kernel
        hp = synth.head_params(wl)
        torch.manual_seed(5)
        S = (torch.randn(wl.B, wl.H, wl.d_v, wl.d_k, device="cuda") *
             torch.exp(torch.randn(wl.B, wl.H, wl.d_v, 1, device="cuda")))
        L.lores_load_state(g.h, S, 3)
        status = [g.check()]
        outs = [g.export()]
        for t in range(4, 7):
            outs.append(g.step(synth.step_inputs(wl, t, hp, device="cuda"), t).clone())
        status.append(g.check())
        T = 3
        toks = [synth.step_inputs(wl, 7 + t, hp, device="cuda") for t in range(T)]
        st = [torch.stack([tok[i] for tok in toks]).contiguous() for i in range(5)]
        o = torch.empty(T, wl.B, wl.H, wl.d_v, device="cuda")
        L.lores_decode_steps(g.h, T, *st, o, 7)
        outs.append(o)
        status.append(g.check())
        outs.append(g.export())
        outs.append(g.dequant())
        status.append(g.check())
        torch.cuda.synchronize()
        return status, outs
    finally:
        g.close()


def same(a, b):
    if isinstance(a, tuple):
        return all(same(x, y) for x, y in zip(a, b))
    if isinstance(a, torch.Tensor):
        return torch.equal(a.cpu(), b.cpu()) or (
            a.shape == b.shape and np.array_equal(a.cpu().numpy().view(np.uint32),
                                                  b.cpu().numpy().view(np.uint32)))
    return np.array_equal(np.asarray(a).view(np.uint8), np.asarray(b).view(np.uint8))


@pytest.mark.parametrize("name,wl,bits,kw,kernel", CASES, ids=[c[0] for c in CASES])
def test_checked_build_is_bit_identical_and_raises_nothing(name, wl, bits, kw, kernel,
                                                           use_checked):
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    L = lib()
    st_p, out_p = run_case(wl, bits, kw, kernel)
    use_checked(True)
    assert L.lores_index_checked()
    st_c, out_c = run_case(wl, bits, kw, kernel)
    assert st_p == [L.LORES_OK] * 4 and st_c == [L.LORES_OK] * 4, (st_p, st_c)
    assert len(out_p) == len(out_c)
    for i, (a, b) in enumerate(zip(out_p, out_c)):
        assert same(a, b), (name, i)


def one_step(g, wl, t, o_fill=None):
    hp = synth.head_params(wl)
    inp = synth.step_inputs(wl, t, hp, device="cuda")
    if o_fill is not None:
        g.o.fill_(o_fill)
    return g.step(inp, t).clone()


def test_trimmed_output_is_flagged_and_only_its_end_is_skipped(use_checked):
    L = lib()
    wl = synth.Workload("ic-trim-o", B=3, H=3, d_k=64, d_v=40, steps=2, decay="tau", group=16,
                        outliers=2, seed=41)
    bits = [8, 4, 8]
    ref = GpuRun(wl, bits, seed=3)
    o_ref = one_step(ref, wl, 0)
    ref_state = ref.export()
    ref.close()
    use_checked(True)
    g = GpuRun(wl, bits, seed=3)
    try:
        L.lores_debug_trim_range(g.h, O, 8)              # the last two floats of o
        o = one_step(g, wl, 0, o_fill=float("nan"))
        assert g.check() == L.LORES_ERR_INDEX
        flags = L.lores_debug_last_flags(g.h)
        assert flags & INDEX_BIT and flags & (256 << O)
        assert not flags & ~(INDEX_BIT | (256 << O))     # o only, nothing else
        flat, flat_ref = o.reshape(-1), o_ref.reshape(-1)
        assert torch.isnan(flat[-2:]).all()              # the two trimmed floats: skipped
        assert torch.equal(flat[:-2], flat_ref[:-2])     # every other output: written
        assert same(g.export(), ref_state)               # the state is not affected
        L.lores_debug_trim_range(g.h, O, 0)
        one_step(g, wl, 1)
        assert g.check() == L.LORES_OK
    finally:
        g.close()


def test_trimmed_code_pool_is_flagged_and_the_state_outside_is_exact(use_checked):
    """The last 16 bytes of the code pool declared away: the last unit's copy (which
    reads them) is not issued, so its warp waits out a short limit, and stores there are
    skipped; the call reports INDEX with the code-pool bit.  Every sequence but the last
    keeps the ordinary build's state bit for bit."""
    L = lib()
    wl = synth.Workload("ic-trim-c", B=3, H=2, d_k=64, d_v=32, steps=2, decay="tau", group=16,
                        outliers=2, seed=42)
    bits = [8, 8]
    ref = GpuRun(wl, bits, seed=4)
    one_step(ref, wl, 0)
    rc, rs = ref.export()
    ref.close()
    use_checked(True)
    g = GpuRun(wl, bits, seed=4)
    try:
        L.lores_set_fault_injection(g.h, -1, 0, 2000)   # waits give up after 2 ms
        L.lores_debug_trim_range(g.h, CODES, 16)
        one_step(g, wl, 0)
        torch.cuda.synchronize()
        assert g.check() == L.LORES_ERR_INDEX
        flags = L.lores_debug_last_flags(g.h)
        assert flags & INDEX_BIT and flags & (256 << CODES)
        L.lores_debug_trim_range(g.h, CODES, 0)
        L.lores_set_fault_injection(g.h, -1, 0, 0)
        c, s = g.export()
        assert np.array_equal(c[:-1], rc[:-1]) and np.array_equal(s[:-1], rs[:-1])
    finally:
        g.close()


def test_trimmed_state_input_of_the_loader_is_flagged(use_checked):
    L = lib()
    wl = synth.Workload("ic-trim-s", B=2, H=2, d_k=32, d_v=16, steps=1, decay="tau", group=32,
                        outliers=0, seed=43)
    use_checked(True)
    g = GpuRun(wl, [8, 4], seed=5)
    try:
        S = torch.randn(wl.B, wl.H, wl.d_v, wl.d_k, device="cuda")
        L.lores_debug_trim_range(g.h, STATE, 64)          # the last lane's 16 floats
        L.lores_load_state(g.h, S, 0)
        assert g.check() == L.LORES_ERR_INDEX
        assert L.lores_debug_last_flags(g.h) == INDEX_BIT | (256 << STATE)
        L.lores_debug_trim_range(g.h, STATE, 0)
        L.lores_load_state(g.h, S, 0)
        assert g.check() == L.LORES_OK
    finally:
        g.close()


def test_ordinary_build_has_no_checks():
    L = lib()
    assert not L.lores_index_checked()
    h = L.lores_create(1, 1, 16, 16)
    try:
        with pytest.raises(L.LoresError) as e:
            L.lores_debug_trim_range(h, O, 4)
        assert e.value.status == L.LORES_ERR_UNSUPPORTED
        with pytest.raises(L.LoresError) as e:
            L.lores_debug_trim_range(h, 9, 4)
        assert e.value.status == L.LORES_ERR_INVALID_ARG
    finally:
        L.lores_destroy(h)
