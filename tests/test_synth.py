"""The seeded generators honour the recurrence's domain (General recurrence form:
unit q, k; beta in (0, 2); alpha in (0, 1]) and the workloads' stated shapes."""
import numpy as np
import pytest
import torch

from bit_recurrent_state_lores_b200 import synth


@pytest.mark.parametrize("name", ["tiny", "gdn", "mamba2", "kda", "sweep"])
def test_domain_and_shapes(name):
    wl = synth.workload(name, B=min(4, synth.WORKLOADS[name].B))
    hp = synth.head_params(wl)
    q, k, v, a, b = synth.step_inputs(wl, 3, hp)
    assert q.shape == (wl.B, wl.H, wl.d_k) and v.shape == (wl.B, wl.H, wl.d_v)
    assert a.shape == ((wl.B, wl.H, wl.d_k) if wl.diag else (wl.B, wl.H))
    for x in (q, k):
        n = torch.linalg.vector_norm(x.double(), dim=-1)
        assert torch.allclose(n, torch.ones_like(n), atol=1e-6)
    assert (b > 0).all() and (b < 2).all()
    assert (a > 0).all() and (a <= 1).all()
    assert all(x.dtype == torch.float32 and x.is_contiguous() for x in (q, k, v, a, b))


def test_seeded_and_step_dependent():
    wl = synth.workload("gdn", B=2)
    hp = synth.head_params(wl)
    a = synth.step_inputs(wl, 5, hp)
    b = synth.step_inputs(wl, 5, hp)
    c = synth.step_inputs(wl, 6, hp)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert not torch.equal(a[0], c[0])


def test_tau_decay_and_outliers():
    wl = synth.workload("gdn")
    hp = synth.head_params(wl)
    tau = -1.0 / np.log(hp["alpha_h"].double().numpy())
    assert tau.min() >= 1.0 - 1e-6 and tau.max() <= 1000.0 + 1e-3
    assert hp["outlier_idx"].shape == (wl.H, 4)
    q, k, v, _, _ = synth.step_inputs(synth.replace(wl, B=64), 0, hp)
    sd = v.std(dim=(0,))                                    # [H, d_v]
    for h in range(wl.H):
        idx = hp["outlier_idx"][h]
        mask = torch.ones(wl.d_v, dtype=torch.bool)
        mask[idx] = False
        assert sd[h, idx].mean() > 5 * sd[h, mask].mean()


def test_kda_head_mean_decay_targets():
    wl = synth.workload("kda", B=1)
    hp = synth.head_params(wl)
    target = hp["mean_decay"]
    assert abs(target[0] - 0.5) < 1e-6 and abs(target[-1] - 0.9999) < 1e-6
    g = torch.Generator().manual_seed(0)
    y = torch.randn(400000, wl.H, generator=g, dtype=torch.float64) + hp["mu"].double()[None]
    mean = torch.exp(-torch.nn.functional.softplus(y)).mean(0).numpy()
    assert np.allclose(mean, target, atol=3e-3)


def test_mamba2_beta_clipped():
    wl = synth.workload("mamba2", B=8)
    _, _, _, _, b = synth.step_inputs(wl, 0)
    assert b.min() >= 1e-6 and b.max() <= 2 - 1e-6


def test_kda_channel_mean_decay_targets():
    # per-channel decays: each head's channels span 1 - m = 0.5 .. 1e-4 in a seeded order
    wl = synth.Workload("kdac", B=64, H=3, d_k=32, d_v=16, steps=1, diag=1, decay="kda_channel",
                        seed=5)
    hp = synth.head_params(wl)
    target = hp["mean_decay_channel"]
    assert target.shape == (3, 32) and hp["mu"].shape == (3, 32)
    for h in range(3):
        assert np.allclose(np.sort(1 - target[h].astype(np.float64)),
                           np.sort(np.logspace(np.log10(0.5), -4, 32)), rtol=0, atol=1e-7)
    assert not np.array_equal(target[0], target[1])          # orders differ per head
    alphas = torch.stack([synth.step_inputs(wl, t, hp)[3] for t in range(200)])
    mean = alphas.double().mean(dim=(0, 1)).numpy()           # [H, d_k]
    assert np.allclose(mean, target, atol=6e-3)
