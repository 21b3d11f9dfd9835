"""The seeded input generator: determinism, distributions, slicing (CPU)."""
import math

import numpy as np
import torch

import synth


def test_deterministic_and_slice_independent():
    s = synth.WORKLOADS["tiny_f32_T64_d32_N4"]
    a = synth.make_layer_inputs(s)
    b = synth.make_layer_inputs(s)
    for k in a:
        if a[k] is not None:
            assert torch.equal(a[k], b[k]), k
    one = synth.expert_slice(s, [2])
    for k in ("W1", "b1", "W2", "b2"):
        assert torch.equal(one[k][0], a[k][2])


def test_distributions():
    s = synth.LayerSpec("stats", 512, 256, 512, 8, 1.0, "f32")
    inp = synth.make_layer_inputs(s)
    x = inp["x"].double()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1.0) < 0.01
    # truncated normal at 2 sigma: std = sigma*sqrt(1 - 2*2*phi(2)/(2*Phi(2)-1))
    phi2 = math.exp(-2.0) / math.sqrt(2 * math.pi)
    Phi = 0.5 * (1 + math.erf(2 / math.sqrt(2)))
    ratio = math.sqrt(1 - 4 * phi2 / (2 * Phi - 1))
    for name, fan in (("W1", s.d), ("W2", s.d_ff), ("W_r", s.d)):
        sig = math.sqrt(0.1 / fan)
        w = inp[name].double()
        assert w.abs().max().item() <= 2 * sig * (1 + 1e-6)
        tol = 4.0 / math.sqrt(2 * w.numel())          # ~4 standard errors
        assert abs(w.std().item() / (sig * ratio) - 1) < tol, name
        assert abs(w.mean().item()) < 4.0 * sig / math.sqrt(w.numel())


def test_hash_buckets_uniform_and_uncorrelated():
    idx = torch.arange(1 << 20, dtype=torch.int64)
    k1, k2 = synth._key_words(("t",))
    b = synth._bucket(idx, k1, k2)
    hist = torch.bincount(b >> 12, minlength=256).double()     # 256 coarse bins
    exp = (1 << 20) / 256
    chi2 = (((hist - exp) ** 2) / exp).sum().item()
    assert chi2 < 400          # 255 dof: mean 255, sd ~22.6
    u = (b.double() + 0.5) / (1 << synth.TABLE_BITS) - 0.5
    r = (u[1:] * u[:-1]).mean().item() / (u * u).mean().item()
    assert abs(r) < 0.01


def test_bf16_is_rounded_fp32_table():
    s = synth.LayerSpec("r", 16, 8, 8, 2, 1.0, "bf16")
    f = synth.LayerSpec("r", 16, 8, 8, 2, 1.0, "f32")
    xb = synth.make_x(s)
    xf = synth.make_x(f)
    assert torch.equal(xb, xf.to(torch.bfloat16))


def test_redraw_changes_only_listed_rows():
    s = synth.WORKLOADS["tiny_f32_T64_d32_N4"]
    a = synth.make_x(s)
    b = synth.make_x(s, redraws={3: 0, 10: 2})
    diff = (a != b).any(dim=1).nonzero().flatten().tolist()
    assert diff == [3, 10]


def test_router_bias_zipf():
    s = synth.WORKLOADS["skewed_T32768_d2048_N64"]
    b = synth.router_bias_values(s)
    assert b.dtype == torch.float32 and b.shape == (64,)
    assert b[0].item() == 0.0
    assert abs(b[1].item() - 1.5 * math.log(0.5)) < 1e-6
