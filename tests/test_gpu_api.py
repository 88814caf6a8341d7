"""GPU tests of the C ABI beyond numerics: error handling (faults injected on the host:
NaN inputs, bad arguments), checkpoint/resume, the host-buffer step, and several
handles in one process.  Every expected state comes from the oracle or from the
library's own earlier output on the same inputs (for determinism checks)."""
import numpy as np
import pytest
import torch

from bit_recurrent_state_lores_b200 import synth
from oracle import oracle as O

from .harness import GpuRun, OracleTiles, host_tile_inputs, rel_l2, tile_cfg

pytestmark = pytest.mark.gpu


def lib():
    from bit_recurrent_state_lores_b200 import lores
    return lores


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def small(B=3, H=3, d_k=128, d_v=64, diag=0, group=32):
    return synth.Workload("api", B=B, H=H, d_k=d_k, d_v=d_v, steps=4, diag=diag, group=group,
                          decay="kda" if diag else "tau", outliers=2, seed=7)


@pytest.mark.parametrize("bits", [[8, 8, 8], [4, 8, 32]])
def test_nonfinite_rows_zeroed_flagged_and_gpu_stays_usable(bits):
    L = lib()
    wl = small()
    hp = synth.head_params(wl)
    g = GpuRun(wl, bits, seed=3)
    tiles = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    ref = OracleTiles(wl, bits, 3, tiles)
    for step in range(3):
        inp = list(synth.step_inputs(wl, step, hp, device="cuda"))
        if step == 1:
            inp[2] = inp[2].clone()
            inp[2][1, 2, 5] = float("nan")          # row 5 of tile (1, 2)
            inp[2][2, 0, 17] = float("inf")         # row 17 of tile (2, 0)
        g.step(inp, step)
        _, flags = ref.step(host_tile_inputs(inp, tiles), step)
        st = g.check()
        if step == 1:
            assert flags[(1, 2)] == 1 and flags[(2, 0)] == 1
        # quantized rows are zeroed, so the flag does not come back on the next step; an
        # fp32 head keeps its non-finite state (and the flag) as the oracle does
        expect = L.LORES_ERR_NONFINITE if any(flags.values()) else L.LORES_OK
        assert st == expect, (step, st)
        codes, scales = g.export()
        for t in tiles:
            gs, gsc = g.tile(codes, scales, *t)
            rs, rsc = ref.state[t]
            cfg = ref.cfg[t]
            if cfg.bits == 32:
                both_nan = np.isnan(gs) & np.isnan(rs)
                assert np.array_equal(np.where(both_nan, 0, gs), np.where(both_nan, 0, rs))
            else:
                assert np.array_equal(gs, rs) and np.array_equal(gsc, rsc), (step, t)
        if step == 1 and bits[2] != 32:
            gs, gsc = g.tile(codes, scales, 1, 2)
            assert not gsc[5].any()
    g.close()


def test_bad_arguments_are_rejected_before_launch():
    L = lib()
    wl = small()
    h = L.lores_create(wl.B, wl.H, wl.d_k, wl.d_v)
    try:
        q, k, v, a, b = synth.step_inputs(wl, 0, device="cuda")
        o = torch.empty(wl.B, wl.H, wl.d_v, device="cuda")
        raw = L.raw_library()
        s = torch.cuda.current_stream().cuda_stream
        assert raw.lores_decode_step(h, q.data_ptr() + 4, k.data_ptr(), v.data_ptr(), a.data_ptr(),
                                     b.data_ptr(), o.data_ptr(), 0, s) == L.LORES_ERR_INVALID_ARG
        assert raw.lores_decode_step(h, q.data_ptr(), None, v.data_ptr(), a.data_ptr(),
                                     b.data_ptr(), o.data_ptr(), 0, s) == L.LORES_ERR_INVALID_ARG
        assert raw.lores_dequant_state(h, o.data_ptr() + 4, s) == L.LORES_ERR_INVALID_ARG
        # the handle still works afterwards
        L.lores_decode_step(h, q, k, v, a, b, o, 0)
        assert L.lores_check_errors(h) == L.LORES_OK
    finally:
        L.lores_destroy(h)


def test_export_load_round_trip_and_bit_identical_resume():
    L = lib()
    wl = small(diag=1)
    bits = [8, 4, 8]
    hp = synth.head_params(wl)
    inputs = [synth.step_inputs(wl, t, hp, device="cuda") for t in range(10)]
    a = GpuRun(wl, bits, seed=21)
    for t in range(5):
        a.step(inputs[t], t)
    ckpt = a.export()
    for t in range(5, 10):
        a.step(inputs[t], t)
    final_a = a.export()
    o_a = a.o.clone()
    # a fresh handle restored from the checkpoint replays steps 5..9 bit for bit
    b = GpuRun(wl, bits, seed=21)
    b.load(*ckpt)
    assert all(np.array_equal(x, y) for x, y in zip(b.export(), ckpt))
    for t in range(5, 10):
        b.step(inputs[t], t)
    final_b = b.export()
    assert np.array_equal(final_a[0], final_b[0]) and np.array_equal(final_a[1], final_b[1])
    assert torch.equal(o_a, b.o)
    # a different seed gives a different trajectory (the dither is keyed on the seed)
    c = GpuRun(wl, bits, seed=22)
    c.load(*ckpt)
    for t in range(5, 10):
        c.step(inputs[t], t)
    assert not np.array_equal(c.export()[0], final_a[0])
    for r in (a, b, c):
        r.close()


def test_host_buffer_step_equals_device_step():
    L = lib()
    wl = small(diag=1)
    bits = [8, 4, 32]
    hp = synth.head_params(wl)
    d = GpuRun(wl, bits, seed=5)
    hst = GpuRun(wl, bits, seed=5)
    for t in range(3):
        inp = synth.step_inputs(wl, t, hp, device="cuda")
        d.step(inp, t)
        host = [x.cpu().pin_memory() for x in inp]
        o_h = torch.empty(wl.B, wl.H, wl.d_v).pin_memory()
        L.lores_decode_step_host(hst.h, *host, o_h, t)
        torch.cuda.synchronize()
        assert torch.equal(o_h, d.o.cpu())
    assert all(np.array_equal(x, y) for x, y in zip(d.export(), hst.export()))
    # the enqueue-only variant on two streams (pinned buffers) gives the same steps
    a1 = GpuRun(wl, bits, seed=5)
    a2 = GpuRun(wl, bits, seed=5)
    lanes = [torch.cuda.Stream(), torch.cuda.Stream()]
    for t in range(3):
        inp = synth.step_inputs(wl, t, hp, device="cuda")
        host = [x.cpu().pin_memory() for x in inp]
        outs = [torch.empty(wl.B, wl.H, wl.d_v).pin_memory() for _ in range(2)]
        for r, ls, oh in zip((a1, a2), lanes, outs):
            L.lores_decode_step_host_async(r.h, *host, oh, t, ls.cuda_stream)
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1])
    assert all(np.array_equal(x, y) for x, y in zip(d.export(), a1.export()))
    assert all(np.array_equal(x, y) for x, y in zip(d.export(), a2.export()))
    for r in (d, hst, a1, a2):
        r.close()


def test_load_state_and_dequant_match_oracle_on_every_tile():
    L = lib()
    wl = small(B=2, H=3, d_k=64, d_v=36, group=16)
    bits = [8, 4, 32]
    g = GpuRun(wl, bits, seed=8)
    S = (torch.randn(wl.B, wl.H, wl.d_v, wl.d_k, device="cuda") *
         torch.exp(torch.randn(wl.B, wl.H, wl.d_v, 1, device="cuda")))
    L.lores_load_state(g.h, S, 41)
    codes, scales = g.export()
    Sh = S.cpu().numpy()
    sk = O.step_key(8, 41)
    Sd = g.dequant().cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.H):
            cfg = tile_cfg(wl, bits[h])
            gs, gsc = g.tile(codes, scales, b, h)
            if bits[h] == 32:
                assert np.array_equal(gs, Sh[b, h])
                continue
            rc, rs, _ = O.tile_quantize(cfg, Sh[b, h], O.tile_key(sk, b * wl.H + h))
            assert np.array_equal(gs, rc) and np.array_equal(gsc, rs)
            assert np.array_equal(Sd[b, h], O.tile_dequant(cfg, rc, rs))
    g.close()


def test_many_handles_with_different_shared_memory_needs():
    # the kernels' shared-memory attribute is shared by all handles; it must only grow
    wls = [small(d_k=128, d_v=128, group=128), small(d_k=128, d_v=64, group=16),
           small(d_k=16, d_v=256, group=16)]
    runs = [GpuRun(wl, bits, seed=i) for i, (wl, bits) in
            enumerate(zip(wls, [[32, 32, 32], [8, 8, 8], [4, 4, 4]]))]
    for t in range(2):
        for wl, r in zip(wls, runs):
            hp = synth.head_params(wl)
            r.step(synth.step_inputs(wl, t, hp, device="cuda"), t)
    for r in runs:
        assert r.check() == lib().LORES_OK
        r.close()


def test_guard_bands_report_writes_outside_the_state():
    # host-side fault injection: write one byte just past the code pool and one just
    # before the scales (inside the guard bands the library allocates around them)
    L = lib()
    wl = small()
    g = GpuRun(wl, [8, 4, 8], seed=1)
    hp = synth.head_params(wl)
    g.step(synth.step_inputs(wl, 0, hp, device="cuda"), 0)
    assert g.check() == L.LORES_OK
    from cuda.bindings import runtime as rt
    lay = g.layout
    torch.cuda.synchronize()
    (err,) = rt.cudaMemset(lay.codes_dev + lay.code_bytes, 0x11, 1)
    assert err == rt.cudaError_t.cudaSuccess
    assert rt.cudaDeviceSynchronize()[0] == rt.cudaError_t.cudaSuccess
    assert g.check() == L.LORES_ERR_CORRUPT
    assert "overwritten" in L.lores_status_string(L.LORES_ERR_CORRUPT)
    g.close()
    g = GpuRun(wl, [8, 4, 8], seed=1)
    (err,) = rt.cudaMemset(g.layout.scales_dev - 1, 0x11, 1)
    assert err == rt.cudaError_t.cudaSuccess
    assert g.check() == L.LORES_ERR_CORRUPT
    g.close()
