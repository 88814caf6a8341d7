"""The allocation-free decode step (lores_decode_step_noalloc) against the handle step.

Some callers cannot let a library allocate device memory (a serving engine that plans
every buffer from its own pool, or a fixed device-memory budget); they own the state
buffers and call the step that keeps its bookkeeping in a fixed array compiled into
the library.  Its results must equal those of the ordinary handle step on the same
state and inputs.  This file is collected last so that a run stopping at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from bit_recurrent_state_lores_b200 import synth

pytestmark = pytest.mark.gpu


def test_noalloc_step_equals_handle_step_on_two_calls_in_a_row():
    from bit_recurrent_state_lores_b200 import lores as L
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    # mixed int8 / int4 / fp32 heads, key-block scales, delta rule, decay per key column,
    # and a ragged last unit (d_v = 100) so both kernel paths run
    wl = synth.Workload("noalloc", B=6, H=3, d_k=128, d_v=100, steps=2, diag=1, group=32,
                        decay="kda", outliers=2, seed=11)
    bits = [8, 4, 32]
    seed = 99
    hp = synth.head_params(wl)
    h = L.lores_create(wl.B, wl.H, wl.d_k, wl.d_v, group_size=wl.G, delta=1, decay_diag=1,
                       head_bits=bits, stochastic=1, seed=seed)
    try:
        lay, _ = L.lores_get_layout(h, wl.H)
        cfg = L.make_config(wl.B, wl.H, wl.d_k, wl.d_v, group_size=wl.G, delta=1, decay_diag=1,
                            head_bits=bits, stochastic=1, seed=seed)
        # the caller owns the state: zero state = zero codes and scales
        codes = torch.zeros(lay.code_bytes, dtype=torch.uint8, device="cuda")
        scales = torch.zeros(lay.scale_count, dtype=torch.float32, device="cuda")
        flags = torch.full((1,), 7, dtype=torch.int32, device="cuda")
        o_ref = torch.empty(wl.B, wl.H, wl.d_v, device="cuda")
        o_new = torch.empty_like(o_ref)
        for step in (0, 1):
            q, k, v, a, b = synth.step_inputs(wl, step, hp, device="cuda")
            L.lores_decode_step(h, q, k, v, a, b, o_ref, step)
            L.lores_decode_step_noalloc(cfg, codes, scales, q, k, v, a, b, o_new, step,
                                        flags_out=flags)
            torch.cuda.synchronize()
            ref_codes = torch.empty(lay.code_bytes, dtype=torch.uint8)
            ref_scales = torch.empty(lay.scale_count, dtype=torch.float32)
            L.lores_export_codes(h, ref_codes, ref_scales)
            assert torch.equal(codes.cpu(), ref_codes), f"codes differ at step {step}"
            assert torch.equal(scales.cpu(), ref_scales), f"scales differ at step {step}"
            err = (o_new - o_ref).norm() / o_ref.norm()
            assert err <= 1e-5, f"o rel-L2 {err} at step {step}"
            assert int(flags.item()) == 0
        assert L.lores_check_errors(h) == L.LORES_OK
    finally:
        L.lores_destroy(h)


def test_noalloc_rejects_more_units_than_its_table():
    from bit_recurrent_state_lores_b200 import lores as L
    # 4096 heads of 128 x 128 int8 need 4096 * 4 units per sequence, over the 2048 limit
    cfg = L.make_config(1, 4096, 128, 128)
    t = torch.zeros(16, device="cuda")
    with pytest.raises(L.LoresError) as e:
        L.lores_decode_step_noalloc(cfg, t, t, t, t, t, t, t, t, 0)
    assert e.value.status == L.LORES_ERR_UNSUPPORTED


def test_noalloc_large_table_read_from_the_fixed_array_on_a_side_stream():
    """160 heads of 128 x 128 int8 give 640 work units per sequence, more than the kernel
    copies into shared memory, so it reads its table straight from the fixed array; the
    calls run on a stream other than the default one."""
    from bit_recurrent_state_lores_b200 import lores as L
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    wl = synth.Workload("noalloc-large", B=2, H=160, d_k=128, d_v=128, steps=2, decay="tau",
                        outliers=2, seed=12)
    bits = [8] * wl.H
    seed = 41
    hp = synth.head_params(wl)
    side = torch.cuda.Stream()
    h = L.lores_create(wl.B, wl.H, wl.d_k, wl.d_v, head_bits=bits, stochastic=1, seed=seed)
    try:
        lay, _ = L.lores_get_layout(h, wl.H)
        assert lay.units_per_step // wl.B > 512
        cfg = L.make_config(wl.B, wl.H, wl.d_k, wl.d_v, head_bits=bits, stochastic=1, seed=seed)
        codes = torch.zeros(lay.code_bytes, dtype=torch.uint8, device="cuda")
        scales = torch.zeros(lay.scale_count, dtype=torch.float32, device="cuda")
        flags = torch.full((1,), 7, dtype=torch.int32, device="cuda")
        o_ref = torch.empty(wl.B, wl.H, wl.d_v, device="cuda")
        o_new = torch.empty_like(o_ref)
        for step in (0, 1):
            q, k, v, a, b = synth.step_inputs(wl, step, hp, device="cuda")
            L.lores_decode_step(h, q, k, v, a, b, o_ref, step)
            side.wait_stream(torch.cuda.current_stream())
            L.lores_decode_step_noalloc(cfg, codes, scales, q, k, v, a, b, o_new, step,
                                        flags_out=flags, stream=side.cuda_stream)
            torch.cuda.current_stream().wait_stream(side)
            torch.cuda.synchronize()
            ref_codes = torch.empty(lay.code_bytes, dtype=torch.uint8)
            ref_scales = torch.empty(lay.scale_count, dtype=torch.float32)
            L.lores_export_codes(h, ref_codes, ref_scales)
            assert torch.equal(codes.cpu(), ref_codes), f"codes differ at step {step}"
            assert torch.equal(scales.cpu(), ref_scales), f"scales differ at step {step}"
            err = (o_new - o_ref).norm() / o_ref.norm()
            assert err <= 1e-5, f"o rel-L2 {err} at step {step}"
            assert int(flags.item()) == 0
        assert L.lores_check_errors(h) == L.LORES_OK
    finally:
        L.lores_destroy(h)
