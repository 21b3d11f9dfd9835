"""Expert parallelism through the C ABI, ranks emulated one after another on
one GPU: every rank holds a contiguous token range of one global batch and the
weights of N / world experts; the record all-gather and the two row
all-to-alls are done on the host side between the steps (no kernel of one rank
waits for another's).  Together the ranks must give the unsharded layer's
routing bit for bit, its aux loss, and its outputs within the stated
tolerances of the fp64 oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import sparse_mixture_experts_argmax_b200 as swl
from sparse_mixture_experts_argmax_b200 import build as swl_build

from helpers import AUX_RTOL, check_close, check_routing, gap_redraws

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    swl_build.build()
    swl.lib()


def _ep_run(ig, cf, bounds, world):
    x = ig["x"]
    T, d = x.shape
    N, d_ff, _ = ig["W1"].shape
    L = N // world
    dt = swl.dtype_code(x.dtype)
    out = swl.alloc_outputs(T, d, x.dtype)
    R = swl.switch_layer_shard_record_bytes(N)
    recs = torch.empty(world * R, dtype=torch.uint8, device="cuda")
    ws, auxes = [], []
    for g in range(world):
        a, b = bounds[g], bounds[g + 1]
        ws.append(torch.empty(swl.switch_layer_ep_workspace_size(b - a, d, d_ff, N, dt, world, T,
                                                                 cf),
                              dtype=torch.uint8, device="cuda"))
        swl.switch_layer_forward_shard_begin(
            x[a:b], ig["W_r"], cf, T, out["expert_idx"][a:b], out["gate"][a:b],
            out["pos_in_expert"][a:b], recs[g * R:(g + 1) * R], d_ff, b_r=ig.get("b_r"),
            workspace=ws[g])
    gathered = recs.clone()                       # the all-gather
    gh = gathered.cpu()
    counts = [swl.switch_layer_ep_counts(N, world, g, T, cf, gh) for g in range(world)]
    sends = []
    for g in range(world):
        a, b = bounds[g], bounds[g + 1]
        send = torch.empty((sum(counts[g][0]), d), dtype=x.dtype, device="cuda")
        aux = torch.empty(1, dtype=torch.float32, device="cuda")
        swl.switch_layer_ep_dispatch(x[a:b], d_ff, N, world, g, T, cf, gathered,
                                     out["expert_idx"][a:b], out["pos_in_expert"][a:b], aux,
                                     send, ws[g])
        sends.append(send)
        auxes.append(aux)

    def alltoall(blocks, cnts_send):
        # rank r receives, in source order, block r of every source's rows
        parts = [list(torch.split(blocks[g], cnts_send[g])) for g in range(world)]
        return [torch.cat([parts[g][r] for g in range(world)]) for r in range(world)]

    recvs = alltoall(sends, [counts[g][0] for g in range(world)])
    rets = []
    for r in range(world):
        assert recvs[r].shape[0] == sum(counts[r][1])
        ret = torch.empty_like(recvs[r])
        sl = slice(r * L, (r + 1) * L)
        swl.switch_layer_ep_experts(bounds[r + 1] - bounds[r], d, d_ff, N, x.dtype, world, r, T,
                                    cf, gathered, recvs[r], ig["W1"][sl].contiguous(),
                                    ig["b1"][sl].contiguous(), ig["W2"][sl].contiguous(),
                                    ig["b2"][sl].contiguous(), ret, ws[r])
        rets.append(ret)
    backs = alltoall(rets, [counts[r][1] for r in range(world)])
    for g in range(world):
        a, b = bounds[g], bounds[g + 1]
        swl.switch_layer_ep_combine(b - a, d, d_ff, N, x.dtype, world, g, T, cf, backs[g],
                                    out["expert_idx"][a:b], out["gate"][a:b],
                                    out["pos_in_expert"][a:b], out["out"][a:b], ws[g])
    torch.cuda.synchronize()
    for w in ws:
        assert swl.switch_layer_device_status(w) == 0
    out["aux_loss"] = auxes[0]
    return out, [float(a.item()) for a in auxes]


_CASES = [
    ("base_two", synth.WORKLOADS["base_T4096_d768_N64"], 2, [0, 2048, 4096]),
    ("base_four_uneven", synth.WORKLOADS["base_T4096_d768_N64"], 4, [0, 100, 1500, 1500, 4096]),
    ("tiny_f32_two", synth.WORKLOADS["tiny_f32_T64_d32_N4"], 2, [0, 30, 64]),
    ("zipf_drops_four", synth.LayerSpec("ep_zipf", 3000, 256, 64, 40, 1.0, "bf16",
                                        bias_std=0.05, router_bias="zipf1.5"),
     4, [0, 750, 1500, 2250, 3000]),
    ("wide_two", synth.LayerSpec("ep_wide", 2000, 128, 64, 256, 1.25, "bf16", bias_std=0.05),
     2, [0, 1000, 2000]),
]


@pytest.mark.parametrize("case", _CASES, ids=lambda c: c[0])
def test_expert_parallel_matches_oracle(case):
    name, spec, world, bounds = case
    rd = synth.load_gap_redraws(spec.name) if spec.name in synth.WORKLOADS else gap_redraws(spec)
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=rd)
    got, auxes = _ep_run(ig, spec.cf, bounds, world)
    assert len(set(auxes)) == 1, auxes
    ic = synth.make_layer_inputs(spec, device="cpu", redraws=rd)
    ref = oracle.switch_forward(ic["x"], ic["W_r"], ic["W1"], ic["b1"], ic["W2"], ic["b2"],
                                spec.cf, b_r=ic["b_r"])
    check_routing(got, ref, ref["capacity"], spec.T)
    check_close(got["out"].double().cpu().numpy(), ref["out"], spec.dtype)
    if name == "zipf_drops_four":
        assert (~ref["kept"]).any()
    one = swl.forward(ig, spec.cf)
    for k in ("expert_idx", "pos_in_expert"):
        assert torch.equal(got[k], one[k]), k
    a1 = float(one["aux_loss"].item())
    assert abs(auxes[0] - a1) <= AUX_RTOL * abs(a1)


def test_forward_ep_single_rank_helper():
    """forward_ep with world = 1 (the exchanges are copies) equals forward."""
    spec = synth.WORKLOADS["base_T4096_d768_N64"]
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=synth.load_gap_redraws(spec.name))
    got = swl.forward_ep(ig, spec.cf, spec.N, spec.T, 0, 1, lambda r: r.clone(),
                         lambda rows, s, r: rows.clone())
    one = swl.forward(ig, spec.cf)
    for k in ("expert_idx", "pos_in_expert", "gate"):
        assert torch.equal(got[k], one[k]), k
    check_close(got["out"].double().cpu().numpy(), one["out"].double().cpu().numpy(), "bf16")
