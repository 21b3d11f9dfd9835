"""Backward pass (switch_layer_backward) against the fp64 oracle's gradients.

Every gradient is compared as a whole tensor: normwise relative error <= 2e-2
for bf16 layers (the expert rows of du and da are rounded to bf16, as the
forward's hidden rows are) and <= 1e-5 for fp32 layers, and element by element
within atol * max|ref| + rtol * |ref| with the forward's tolerances."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import sparse_mixture_experts_argmax_b200 as swl
from sparse_mixture_experts_argmax_b200 import build as swl_build

from helpers import TOL, gap_redraws

pytestmark = pytest.mark.gpu

NORMWISE = {"bf16": 2e-2, "f32": 1e-5}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    swl_build.build()
    swl.lib()


def _cmp(got, want, dtype, what):
    got = got.detach().double().cpu().numpy().reshape(want.shape)
    atol, rtol = TOL[dtype]
    scale = max(np.abs(want).max(), 1e-30)
    err = np.abs(got - want)
    assert np.all(err <= atol * scale + rtol * np.abs(want)), (what, float(err.max()), scale)
    nw = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert nw <= NORMWISE[dtype], (what, nw)


_CASES = [
    ("tiny_f32", synth.WORKLOADS["tiny_f32_T64_d32_N4"]),
    ("small_bf16_drops", synth.LayerSpec("bwd_small", 300, 64, 128, 6, 1.0, "bf16",
                                         bias_std=0.05)),
    ("ragged_f32_bias", synth.LayerSpec("bwd_ragged", 333, 40, 72, 5, 0.8, "f32", bias_std=0.05,
                                        router_bias="zipf0.3")),
    ("wide_bf16", synth.LayerSpec("bwd_wide", 500, 128, 64, 200, 2.0, "bf16", bias_std=0.05)),
    # d not a multiple of 4: the router logits tiles load element by element
    ("odd_d_f32", synth.LayerSpec("bwd_odd_d", 150, 19, 23, 3, 1.0, "f32", bias_std=0.05)),
    ("base", synth.WORKLOADS["base_T4096_d768_N64"]),
]


@pytest.mark.parametrize("case", _CASES, ids=lambda c: c[0])
def test_backward_matches_oracle(case):
    name, spec = case
    rd = synth.load_gap_redraws(spec.name) if spec.name in synth.WORKLOADS else gap_redraws(spec)
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=rd)
    ws = swl.alloc_workspace(spec.T, spec.d, spec.d_ff, spec.N, ig["x"].dtype, spec.cf)
    fwd = swl.forward(ig, spec.cf, workspace=ws)
    dout = synth.draw((0, spec.name, "dout"), (spec.T, spec.d), "normal", 1.0, spec.dtype,
                      "cuda")
    daux = 0.37
    got = swl.backward(ig, spec.cf, fwd, ws, dout, daux)
    torch.cuda.synchronize()
    ic = synth.make_layer_inputs(spec, device="cpu", redraws=rd)
    ref = oracle.switch_backward(ic["x"], ic["W_r"], ic["W1"], ic["b1"], ic["W2"], ic["b2"],
                                 spec.cf, dout.cpu(), daux, b_r=ic["b_r"])
    for k in ("dx", "dW1", "db1", "dW2", "db2", "dW_r", "db_r"):
        _cmp(got[k], ref[k], "f32" if k in ("dW_r", "db_r") and spec.dtype == "f32" else
             spec.dtype, k)
