"""No-Token-Left-Behind variant (switch_layer_forward_ntlb) against the oracle's
two-stage layer.

Seeded inputs are redrawn until every token's first/second and second/third
router-logit gaps are >= 1e-3 (both choices unique); then the choices, both
stages' positions and the expert that keeps each token must match bit for bit,
gates within 1e-4 + 1e-4|g|, outputs within the stated tolerances and aux
within 1e-5."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import sparse_mixture_experts_argmax_b200 as swl
from sparse_mixture_experts_argmax_b200 import build as swl_build

from helpers import AUX_RTOL, GATE_TOL, check_close
from test_gpu_top2 import top2_redraws

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    swl_build.build()
    swl.lib()


def _parity(spec):
    rd = top2_redraws(spec)
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=rd)
    got = swl.forward_ntlb(ig, spec.cf)
    torch.cuda.synchronize()
    ic = synth.make_layer_inputs(spec, device="cpu", redraws=rd)
    ref = oracle.switch_forward_ntlb(ic["x"], ic["W_r"], ic["W1"], ic["b1"], ic["W2"], ic["b2"],
                                     spec.cf, b_r=ic["b_r"])
    e = got["expert_idx"].cpu().numpy().astype(np.int64)
    pos = got["pos_in_expert"].cpu().numpy().astype(np.int64)
    assert np.array_equal(e, ref["expert_idx"]), "expert_idx differs"
    assert np.array_equal(pos, ref["pos_in_expert"]), "pos_in_expert differs"
    g = got["gate"].cpu().numpy().astype(np.float64)
    atol, rtol = GATE_TOL
    assert np.all(np.abs(g - ref["gate"]) <= atol + rtol * np.abs(ref["gate"])), "gate"
    aux = float(got["aux_loss"].cpu()[0])
    assert abs(aux - ref["aux"]) <= AUX_RTOL * abs(ref["aux"]), (aux, ref["aux"])
    out = got["out"].double().cpu().numpy()
    check_close(out, ref["out"], spec.dtype)
    dropped = ref["assigned"] < 0
    assert not out[dropped].any(), "a token neither stage keeps has a non-zero row"
    return got, ref


_SHAPES = [
    # name, T, d, d_ff, N, cf, dtype, router bias
    ("zipf_reroutes", 3000, 256, 64, 40, 1.0, "bf16", "zipf0.5"),
    ("heavy_overflow", 4096, 256, 128, 64, 1.0, "bf16", "zipf1.5"),
    ("no_overflow", 600, 128, 64, 8, 8.0, "bf16", None),
    ("stream_n200_ragged", 700, 256, 128, 200, 1.0, "bf16", "zipf0.2"),
    ("rows_n202", 500, 128, 64, 202, 0.75, "bf16", None),
    ("f32_small", 257, 32, 48, 5, 0.75, "f32", "zipf0.5"),
]


@pytest.mark.parametrize("shape", _SHAPES, ids=lambda s: s[0])
def test_ntlb_matches_oracle(shape):
    name, T, d, d_ff, N, cf, dtype, rb = shape
    spec = synth.LayerSpec("ntlb_" + name, T, d, d_ff, N, cf, dtype, bias_std=0.05,
                           router_bias=rb)
    got, ref = _parity(spec)
    C = ref["capacity"]
    pos = ref["pos_in_expert"]
    rerouted = (pos[:, 0] >= C) & (pos[:, 1] >= 0) & (pos[:, 1] < C)
    if name == "no_overflow":
        assert (pos[:, 0] < C).all() and (pos[:, 1] == -1).all()
    elif name in ("zipf_reroutes", "heavy_overflow", "stream_n200_ragged", "f32_small"):
        assert rerouted.any(), "the case reroutes no token"
    if name == "heavy_overflow":
        assert (ref["assigned"] < 0).any(), "the case drops no token in stage 2"


def test_ntlb_keeps_the_top1_tokens():
    """Every token the top-1 layer keeps is kept by the same expert at the same
    position, with the same output row (the stage-1 part of the layer)."""
    spec = synth.LayerSpec("ntlb_vs_top1", 2048, 128, 64, 16, 1.0, "bf16", bias_std=0.05,
                           router_bias="zipf0.5")
    rd = top2_redraws(spec)
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=rd)
    a = swl.forward_ntlb(ig, spec.cf)
    b = swl.forward(ig, spec.cf)
    torch.cuda.synchronize()
    C = swl.switch_layer_capacity(spec.T, spec.N, spec.cf)
    kept1 = (b["pos_in_expert"] < C).cpu()
    assert torch.equal(a["expert_idx"][:, 0].cpu(), b["expert_idx"].cpu())
    assert torch.equal(a["pos_in_expert"][:, 0].cpu(), b["pos_in_expert"].cpu())
    # the same rows through the same FFN; the two routers' softmax kernels may
    # round the gate differently in its last bits
    check_close(a["out"].double().cpu()[kept1].numpy(), b["out"].double().cpu()[kept1].numpy(),
                spec.dtype)


def test_ntlb_rejects_small_workspace():
    spec = synth.LayerSpec("ntlb_ws", 64, 32, 32, 4, 1.0, "bf16")
    ig = synth.make_layer_inputs(spec, device="cuda")
    ws1 = swl.alloc_workspace(64, 32, 32, 4, torch.bfloat16, 1.0)          # top-1 size
    with pytest.raises(swl.SwitchLayerError) as ei:
        swl.forward_ntlb(ig, 1.0, workspace=ws1)
    assert ei.value.status == 3
