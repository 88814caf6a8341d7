"""Multi-token decode steps (lores_decode_steps): T tokens per call must give, bit for bit,
the state, scales, outputs and flags of T single-token calls, and match the oracle's T
consecutive steps (the recurrence of the General Recurrence Form applied token by token,
requantizing after every token as Key properties item 3 states)."""
import numpy as np
import pytest
import torch

from bit_recurrent_state_lores_b200 import synth

from .harness import GpuRun, OracleTiles, assert_parity, host_tile_inputs, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def lib():
    from bit_recurrent_state_lores_b200 import lores
    return lores


def same(a, b):
    """Bit-equal, with NaN equal to NaN (a non-finite row's output is NaN on both paths)."""
    na, nb = torch.isnan(a), torch.isnan(b)
    return torch.equal(na, nb) and torch.equal(a[~na], b[~nb])


def token_inputs(wl, hp, t0, T):
    """Per-token inputs of steps t0 .. t0+T-1 and their token-major stacks."""
    toks = [synth.step_inputs(wl, t0 + t, hp, device="cuda") for t in range(T)]
    stacked = [torch.stack([tok[i] for tok in toks]).contiguous() for i in range(5)]
    return toks, stacked


def run_pair(wl, bits, T, seed=3, stochastic=1, chunks=3, axis=0, inject=None):
    """Handle A takes `chunks` calls of T tokens; handle B the same tokens one by one."""
    L = lib()
    hp = synth.head_params(wl)
    a = GpuRun(wl, bits, seed, stochastic=stochastic, axis=axis)
    b = GpuRun(wl, bits, seed, stochastic=stochastic, axis=axis)
    for ch in range(chunks):
        t0 = ch * T
        toks, st = token_inputs(wl, hp, t0, T)
        if inject is not None:
            inject(t0, toks, st)
        o_a = torch.empty(T, wl.B, wl.H, wl.d_v, device="cuda")
        L.lores_decode_steps(a.h, T, *st, o_a, t0)
        for t in range(T):
            b.step(toks[t], t0 + t)
            assert same(o_a[t], b.o), f"chunk {ch} token {t}: o differs"
        fa, fb = a.check(), b.check()
        assert fa == fb, (fa, fb)
        ea, eb = a.export(), b.export()
        assert np.array_equal(ea[0], eb[0]) and np.array_equal(ea[1], eb[1]), f"chunk {ch}"
    return a, b


MT_CASES = [
    # name, d_k, d_v, G, bits, delta, diag, sr, B, H, T
    ("int8", 128, 128, 128, [8, 8], 1, 0, 1, 3, 2, 4),
    ("mixed-diag", 128, 64, 32, [8, 4, 6, 32], 0, 1, 1, 2, 4, 3),
    ("ragged", 64, 100, 32, [4, 8], 1, 1, 1, 2, 2, 5),
    ("rtn", 32, 36, 16, [8, 5], 1, 0, 0, 3, 2, 2),
    ("dk16", 16, 20, 16, [8, 4, 8], 1, 0, 1, 2, 3, 6),
    ("dk256", 256, 64, 256, [4, 8], 1, 0, 1, 2, 2, 3),
]


@pytest.mark.parametrize("name,d_k,d_v,G,bits,delta,diag,sr,B,H,T", MT_CASES)
def test_tokens_per_call_equal_single_steps(name, d_k, d_v, G, bits, delta, diag, sr, B, H, T):
    wl = synth.Workload(name, B=B, H=H, d_k=d_k, d_v=d_v, steps=3 * T, delta=delta, diag=diag,
                        group=G, decay="kda" if diag else "tau", outliers=2, seed=5)
    a, b = run_pair(wl, bits, T, stochastic=sr)
    assert a.check() == lib().LORES_OK
    a.close()
    b.close()


def test_tokens_per_call_match_oracle_every_tile():
    wl = synth.Workload("mt-oracle", B=2, H=3, d_k=64, d_v=48, steps=8, delta=1, diag=1,
                        group=32, decay="kda", outliers=2, seed=9)
    bits = [8, 4, 32]
    L = lib()
    hp = synth.head_params(wl)
    tiles = [(bb, hh) for bb in range(wl.B) for hh in range(wl.H)]
    g = GpuRun(wl, bits, seed=4)
    ref = OracleTiles(wl, bits, 4, tiles)
    T = 4
    for t0 in (0, T):
        toks, st = token_inputs(wl, hp, t0, T)
        o = torch.empty(T, wl.B, wl.H, wl.d_v, device="cuda")
        L.lores_decode_steps(g.h, T, *st, o, t0)
        oh = o.cpu().numpy()
        for t in range(T):
            oref, flags = ref.step(host_tile_inputs(toks[t], tiles), t0 + t)
            for tl in tiles:
                assert flags[tl] == 0
                r = rel_l2(oh[t][tl], oref[tl])
                assert r <= 1e-5, (t0 + t, tl, r)
        codes, scales = g.export()
        for tl in tiles:
            gs, gsc = g.tile(codes, scales, *tl)
            rs, rsc = ref.state[tl]
            if bits[tl[1]] == 32:
                assert np.array_equal(gs, rs)
                continue
            assert assert_parity(ref.cfg[tl], gs, gsc, rs, rsc, f"{t0} {tl}") == 0
            assert np.array_equal(gsc, rsc)
    assert g.check() == L.LORES_OK
    g.close()


def test_nonfinite_token_inside_a_call():
    # a NaN value at the second token of a call: the row is zeroed in the on-chip state,
    # the later tokens continue from zero, and the flag is raised, as with single steps
    wl = synth.Workload("mt-nan", B=2, H=2, d_k=128, d_v=64, steps=8, delta=1, diag=0,
                        group=128, decay="tau", outliers=0, seed=2)

    def inject(t0, toks, st):
        if t0 == 4:
            toks[1] = list(toks[1])
            toks[1][2] = toks[1][2].clone()
            toks[1][2][1, 0, 7] = float("nan")
            st[2][1] = toks[1][2]

    a, b = run_pair(wl, [8, 4], 4, chunks=3, inject=inject)
    a.close()
    b.close()


def test_key_axis_and_single_token_calls():
    L = lib()
    wl = synth.Workload("mt-key", B=2, H=2, d_k=64, d_v=32, steps=6, delta=1, diag=0,
                        group=64, decay="tau", outliers=2, seed=8)
    a, b = run_pair(wl, [8, 4], 3, chunks=2, axis=1)
    a.close()
    b.close()
    wl = synth.Workload("mt-one", B=2, H=2, d_k=64, d_v=32, steps=3, delta=1, diag=0,
                        group=64, decay="tau", outliers=2, seed=8)
    a, b = run_pair(wl, [8, 32], 1, chunks=3)
    h = a.h
    q = torch.zeros(1, 2, 2, 64, device="cuda")
    raw = L.raw_library()
    s = torch.cuda.current_stream().cuda_stream
    assert raw.lores_decode_steps(h, 0, q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(),
                                  q.data_ptr(), q.data_ptr(), 0, s) == L.LORES_ERR_INVALID_ARG
    a.close()
    b.close()


def test_gdn_shape_eight_tokens_per_call():
    wl = synth.Workload("mt-gdn", B=64, H=32, d_k=128, d_v=128, steps=16, delta=1, diag=0,
                        group=32, decay="tau", outliers=4, seed=1)
    a, b = run_pair(wl, [8] * 32, 8, chunks=2)
    a.close()
    b.close()


@pytest.mark.parametrize("diag,delta,sr", [(1, 1, 1), (0, 0, 0)])
def test_two_rows_per_lane_kernel_tokens_per_call(diag, delta, sr):
    """Handles that step with the two-rows-per-lane kernel (byte and nibble heads with
    several scales per row, full row blocks): T tokens per call equal T single-token calls
    bit for bit."""
    bits = [8, 4, 8, 8, 4, 8, 4, 8]
    wl = synth.Workload("mt-pair", B=72, H=len(bits), d_k=128, d_v=128, steps=8, delta=delta,
                        diag=diag, group=32, decay="kda" if diag else "tau", outliers=2, seed=9)
    a, b = run_pair(wl, bits, 4, stochastic=sr, chunks=2)
    assert a.layout.step_kernel == 1 and b.layout.step_kernel == 1
    assert a.check() == lib().LORES_OK
    a.close()
    b.close()


@pytest.mark.parametrize("diag,delta,sr", [(1, 1, 1), (0, 1, 1), (0, 0, 0)])
def test_tensor_core_kernel_against_multi_token_calls(diag, delta, sr):
    """Heads with one scale per row: single-token calls run the tensor-core kernel, T tokens
    per call the general kernel's exact-projection path.  The two agree bit for bit."""
    bits = [8, 4, 8, 8, 4, 8, 4, 8]
    wl = synth.Workload("mt-mma", B=72, H=len(bits), d_k=128, d_v=128, steps=8, delta=delta,
                        diag=diag, group=128, decay="kda" if diag else "tau", outliers=2, seed=19)
    a, b = run_pair(wl, bits, 4, stochastic=sr, chunks=2)
    assert a.layout.step_kernel == 3 and b.layout.step_kernel == 3
    assert a.check() == lib().LORES_OK
    a.close()
    b.close()
