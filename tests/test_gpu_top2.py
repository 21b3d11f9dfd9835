"""Top-2 variant (switch_layer_forward_top2) against the oracle's top-2 layer.

Seeded inputs are redrawn until every token's first/second and second/third
router-logit gaps are >= 1e-3, so that both choices are unique; then expert
choices, positions and the drop mask must match bit for bit, gates within
1e-4 + 1e-4|g|, outputs within the stated tolerances and aux within 1e-5."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import sparse_mixture_experts_argmax_b200 as swl
from sparse_mixture_experts_argmax_b200 import build as swl_build

from helpers import AUX_RTOL, GAP, GATE_TOL, check_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    swl_build.build()
    swl.lib()


def _gaps12_23(z):
    s = np.sort(z, axis=1)
    return s[:, -1] - s[:, -2], s[:, -2] - s[:, -3] if z.shape[1] > 2 else np.full(len(z), np.inf)


def top2_redraws(spec, seed=0):
    r = synth.make_router(spec, seed)
    x = synth.make_x(spec, seed)
    g1, g2 = _gaps12_23(oracle.router_logits(x, r["W_r"], r["b_r"]))
    rows = {}
    todo = [int(t) for t in np.nonzero((g1 < GAP) | (g2 < GAP))[0]]
    while todo:
        nxt = []
        for t in todo:
            rows[t] = rows.get(t, -1) + 1
            xt = synth.draw((seed, spec.name, "x_redraw", t, rows[t]), (1, spec.d), "normal", 1.0,
                            spec.dtype)
            a, b = _gaps12_23(oracle.router_logits(xt, r["W_r"], r["b_r"]))
            if a[0] < GAP or b[0] < GAP:
                nxt.append(t)
        todo = nxt
    return rows


def _parity(spec, normalize=True):
    rd = top2_redraws(spec)
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=rd)
    got = swl.forward_top2(ig, spec.cf, normalize)
    torch.cuda.synchronize()
    ic = synth.make_layer_inputs(spec, device="cpu", redraws=rd)
    ref = oracle.switch_forward_top2(ic["x"], ic["W_r"], ic["W1"], ic["b1"], ic["W2"], ic["b2"],
                                     spec.cf, b_r=ic["b_r"], normalize=normalize)
    C = ref["capacity"]
    e = got["expert_idx"].cpu().numpy().astype(np.int64)
    pos = got["pos_in_expert"].cpu().numpy().astype(np.int64)
    assert np.array_equal(e, ref["expert_idx"]), "expert_idx differs"
    assert np.array_equal(pos, ref["pos_in_expert"]), "pos_in_expert differs"
    assert np.array_equal(pos < C, ref["kept"]), "drop mask differs"
    g = got["gate"].cpu().numpy().astype(np.float64)
    atol, rtol = GATE_TOL
    assert np.all(np.abs(g - ref["gate"]) <= atol + rtol * np.abs(ref["gate"])), "gate"
    aux = float(got["aux_loss"].cpu()[0])
    assert abs(aux - ref["aux"]) <= AUX_RTOL * abs(ref["aux"]), (aux, ref["aux"])
    check_close(got["out"].double().cpu().numpy(), ref["out"], spec.dtype)
    return got, ref


_SHAPES = [
    # name, T, d, d_ff, N, cf, dtype, router bias
    ("base_like", 4096, 768, 3072, 64, 1.25, "bf16", None),
    ("n2_no_drops", 300, 64, 128, 2, 2.0, "bf16", None),
    ("stream_n200", 700, 256, 128, 200, 1.0, "bf16", None),
    ("rows_n202_bias", 500, 128, 64, 202, 1.0, "bf16", "zipf0.1"),
    ("ragged_tiny_capacity", 333, 200, 136, 6, 0.05, "bf16", None),
    ("f32_small", 257, 32, 48, 5, 1.0, "f32", None),
    ("f32_wide", 300, 48, 40, 150, 1.5, "f32", None),
    ("zipf_drops", 3000, 256, 64, 40, 1.0, "bf16", "zipf1.5"),
]


@pytest.mark.parametrize("shape", _SHAPES, ids=lambda s: s[0])
def test_top2_matches_oracle(shape):
    name, T, d, d_ff, N, cf, dtype, rb = shape
    spec = synth.LayerSpec("top2_" + name, T, d, d_ff, N, cf, dtype, bias_std=0.05,
                           router_bias=rb)
    got, ref = _parity(spec)
    if name in ("ragged_tiny_capacity", "zipf_drops"):
        assert (~ref["kept"]).any()
    if name == "n2_no_drops":
        assert ref["kept"].all()


def test_top2_unnormalised_gates():
    spec = synth.LayerSpec("top2_unnorm", 900, 128, 256, 8, 1.0, "bf16", bias_std=0.05)
    got, ref = _parity(spec, normalize=False)
    g = got["gate"].cpu().numpy()
    assert np.all(g.sum(axis=1) < 1.0)


def test_top2_rejects_one_expert_and_small_workspace():
    spec = synth.LayerSpec("top2_bad", 64, 32, 32, 1, 1.0, "bf16")
    ig = synth.make_layer_inputs(spec, device="cuda")
    with pytest.raises(swl.SwitchLayerError) as ei:
        swl.forward_top2(ig, 1.0, workspace=torch.empty(1 << 20, dtype=torch.uint8,
                                                        device="cuda"))
    assert ei.value.status == 1
    spec = synth.LayerSpec("top2_ws", 64, 32, 32, 4, 1.0, "bf16")
    ig = synth.make_layer_inputs(spec, device="cuda")
    ws1 = swl.alloc_workspace(64, 32, 32, 4, torch.bfloat16, 1.0)          # top-1 size
    with pytest.raises(swl.SwitchLayerError) as ei:
        swl.forward_top2(ig, 1.0, workspace=ws1)
    assert ei.value.status == 3
