"""GEGLU experts and router input jitter (switch_layer_forward_variant)
against the oracle, also combined with top-2 routing.  With jitter the router
sees x * noise, so the gap filter redraws rows on those logits; the experts
see x itself."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import sparse_mixture_experts_argmax_b200 as swl
from sparse_mixture_experts_argmax_b200 import build as swl_build

from helpers import AUX_RTOL, GAP, GATE_TOL, check_close, check_routing

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    swl_build.build()
    swl.lib()


def _gaps(z, top_k):
    s = np.sort(z, axis=1)
    g = s[:, -1] - s[:, -2]
    if top_k == 2 and z.shape[1] > 2:
        g = np.minimum(g, s[:, -2] - s[:, -3])
    return g


def redraws(spec, noise, top_k):
    r = synth.make_router(spec)
    x = synth.make_x(spec)
    n = noise.double().numpy() if noise is not None else None

    def gaps(xs, rows):
        xr = xs if n is None else xs.double().numpy() * n[rows]
        return _gaps(oracle.router_logits(xr, r["W_r"], r["b_r"]), top_k)

    out = {}
    todo = [int(t) for t in np.nonzero(gaps(x, slice(None)) < GAP)[0]]
    while todo:
        nxt = []
        for t in todo:
            out[t] = out.get(t, -1) + 1
            xt = synth.draw((0, spec.name, "x_redraw", t, out[t]), (1, spec.d), "normal", 1.0,
                            spec.dtype)
            if gaps(xt, slice(t, t + 1))[0] < GAP:
                nxt.append(t)
        todo = nxt
    return out


_CASES = [
    # name, T, d, d_ff, N, cf, dtype, activation, jitter, top_k
    ("geglu_bf16", 1500, 256, 320, 8, 1.25, "bf16", "geglu", False, 1),        # d_ff % 128 != 0
    ("geglu_bf16_wide_tiles", 900, 128, 256, 3, 1.0, "bf16", "geglu", False, 1),  # 2 bn = 512
    ("geglu_bf16_small_tiles", 1200, 128, 128, 40, 1.0, "bf16", "geglu", False, 1),
    ("geglu_f32", 300, 40, 56, 5, 1.0, "f32", "geglu", False, 1),
    ("jitter_bf16", 2000, 256, 128, 16, 1.0, "bf16", "relu", True, 1),
    ("jitter_bf16_wide", 700, 128, 64, 200, 2.0, "bf16", "relu", True, 1),
    ("jitter_f32", 257, 32, 48, 6, 1.0, "f32", "relu", True, 1),
    ("top2_geglu_jitter", 1000, 128, 192, 12, 1.0, "bf16", "geglu", True, 2),
]


@pytest.mark.parametrize("case", _CASES, ids=lambda c: c[0])
def test_variant_matches_oracle(case):
    name, T, d, d_ff, N, cf, dtype, act, jitter, top_k = case
    spec = synth.LayerSpec("var_" + name, T, d, d_ff, N, cf, dtype, bias_std=0.05,
                           activation=act)
    noise = synth.router_noise(spec) if jitter else None
    rd = redraws(spec, noise, top_k)
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=rd)
    got = swl.forward_variant(ig, cf, top_k=top_k, activation=act,
                              router_noise=None if noise is None else noise.cuda())
    torch.cuda.synchronize()
    ic = synth.make_layer_inputs(spec, device="cpu", redraws=rd)
    if top_k == 1:
        ref = oracle.switch_forward(ic["x"], ic["W_r"], ic["W1"], ic["b1"], ic["W2"], ic["b2"], cf,
                                    b_r=ic["b_r"], activation=act, router_noise=noise)
        check_routing(got, ref, ref["capacity"], T)
    else:
        xr = ic["x"].double() * noise.double() if jitter else ic["x"]
        # the oracle's top-2 routing of the jittered router input; the experts
        # (GEGLU) see x itself
        p = oracle.router_probs(oracle.router_logits(xr, ic["W_r"], ic["b_r"]))
        e2, g2 = oracle.top2(p)
        pos2 = oracle.positions_top2(e2, N)
        C2 = oracle.capacity_k(T, N, cf, 2)
        f, P = oracle.load_balance_stats(e2[:, 0], p)
        routed = {"expert_idx": e2, "gate": g2, "pos_in_expert": pos2, "kept": pos2 < C2,
                  "aux": oracle.aux_loss(f, P)}
        assert np.array_equal(got["expert_idx"].cpu().numpy(), routed["expert_idx"])
        assert np.array_equal(got["pos_in_expert"].cpu().numpy(), routed["pos_in_expert"])
        g = got["gate"].cpu().numpy().astype(np.float64)
        atol, rtol = GATE_TOL
        assert np.all(np.abs(g - routed["gate"]) <= atol + rtol * np.abs(routed["gate"]))
        a = float(got["aux_loss"].item())
        assert abs(a - routed["aux"]) <= AUX_RTOL * routed["aux"]
        # outputs: the routed assignments applied to x with GEGLU experts
        xs = ic["x"].double().numpy()
        want = np.zeros((T, d))
        for t in range(T):
            for k in range(2):
                if routed["kept"][t, k]:
                    e = routed["expert_idx"][t, k]
                    want[t] += routed["gate"][t, k] * oracle.expert_ffn_geglu(
                        xs[t:t + 1], ic["W1"][e], ic["b1"][e], ic["W2"][e], ic["b2"][e])[0]
        ref = {"out": want}
    check_close(got["out"].double().cpu().numpy(), ref["out"], dtype)


def test_unit_noise_is_the_inference_layer():
    spec = synth.WORKLOADS["base_T4096_d768_N64"]
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=synth.load_gap_redraws(spec.name))
    ones = torch.ones((spec.T, spec.d), dtype=torch.float32, device="cuda")
    a = swl.forward_variant(ig, spec.cf, router_noise=ones)
    b = swl.forward(ig, spec.cf)
    for k in ("expert_idx", "pos_in_expert"):
        assert torch.equal(a[k], b[k]), k
    # FFMA versus tensor-core fp32 router: the gates differ by accumulation order only
    assert (a["gate"] - b["gate"]).abs().max().item() <= 1e-5
    check_close(a["out"].double().cpu().numpy(), b["out"].double().cpu().numpy(), "bf16")
