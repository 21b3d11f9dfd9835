"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch every one of them.  A pin set that lets a planted mistake through would
not be evidence that the oracle is right."""
import numpy as np
import pytest

import oracle.switch_layer as S
import oracle_pins as P


def _top1_highest_tie(p):
    e = p.shape[1] - 1 - np.argmax(p[:, ::-1], axis=1)
    return e.astype(np.int64), p[np.arange(p.shape[0]), e]


def _positions_one_based(expert_idx, N):
    return _orig_positions(expert_idx, N) + 1


def _ffn_no_relu(x_rows, W1e, b1e, W2e, b2e):
    h = S._f64(x_rows) @ S._f64(W1e).T + S._f64(b1e)[None, :]
    return h @ S._f64(W2e).T + S._f64(b2e)[None, :]


def _ffn_transposed_w2(x_rows, W1e, b1e, W2e, b2e):
    h = np.maximum(S._f64(x_rows) @ S._f64(W1e).T + S._f64(b1e)[None, :], 0.0)
    W2 = S._f64(W2e)
    W2 = W2.T if W2.shape[0] == W2.shape[1] else W2
    return h @ W2.T + S._f64(b2e)[None, :]


def _ffn_no_b2(x_rows, W1e, b1e, W2e, b2e):
    h = np.maximum(S._f64(x_rows) @ S._f64(W1e).T + S._f64(b1e)[None, :], 0.0)
    return h @ S._f64(W2e).T


def _aux_no_N(f, P_):
    return float(np.sum(np.asarray(f) * np.asarray(P_)))


def _probs_no_shift(z):
    with np.errstate(over="ignore", invalid="ignore"):
        e = np.exp(z)
        return e / e.sum(axis=1, keepdims=True)


def _capacity_floor(T, N, cf):
    import math
    from fractions import Fraction
    if N <= 0 or T < 0 or not math.isfinite(cf) or cf <= 0:
        raise ValueError
    return math.floor(Fraction(cf) * T / N)


def _stats_after_cut(expert_idx, p):
    T, N = p.shape
    # mistake: counts only the first T//2 tokens (as if capacity applied to f)
    counts = np.bincount(expert_idx[: max(1, T // 2)], minlength=N).astype(np.float64)
    return counts / T, p.sum(axis=0) / T


def _logits_sign(x, W_r, b_r=None):
    z = -(S._f64(x) @ S._f64(W_r).T)
    if b_r is not None:
        z = z + S._f64(b_r)[None, :]
    return z


def _gate_is_one(p):
    e = np.argmax(p, axis=1)
    return e.astype(np.int64), np.ones(p.shape[0])


def _gap_top1_minus_min(z):
    if z.shape[1] < 2:
        return np.full(z.shape[0], np.inf)
    return z.max(axis=1) - z.min(axis=1)


def _gap_on_probs(z):
    if z.shape[1] < 2:
        return np.full(z.shape[0], np.inf)
    s = np.sort(S.router_probs(z), axis=1)
    return s[:, -1] - s[:, -2]


def _gap_distinct_values(z):
    # mistake: the runner-up is the largest value *different* from the top, so
    # an exact tie at the top does not read as a zero gap
    out = []
    for r in z:
        u = np.unique(r)
        out.append(np.inf if len(u) < 2 else u[-1] - u[-2])
    return np.asarray(out)


def _top2_second_is_last(p, normalize=True):
    # mistake: the second choice is the smallest probability
    T, N = p.shape
    e1 = np.argmax(p, axis=1)
    e2 = np.argmin(p, axis=1)
    rows = np.arange(T)
    g = np.stack([p[rows, e1], p[rows, e2]], axis=1)
    if normalize:
        g = g / g.sum(axis=1, keepdims=True)
    return np.stack([e1, e2], axis=1).astype(np.int64), g


def _top2_never_normalised(p, normalize=True):
    return _orig_top2(p, False)


def _capacity_k_ignores_k(T, N, cf, k):
    return S.capacity(T, N, cf)


def _positions_top2_firsts_first(e, N):
    # mistake: all first choices claim slots before any second choice
    seen = [0] * N
    pos = np.zeros(e.shape, dtype=np.int64)
    for k in range(e.shape[1]):
        for t in range(e.shape[0]):
            pos[t, k] = seen[int(e[t, k])]
            seen[int(e[t, k])] += 1
    return pos


def _gelu_tanh(u):
    u = np.asarray(u, dtype=np.float64)
    return 0.5 * u * (1 + np.tanh(np.sqrt(2 / np.pi) * (u + 0.044715 * u ** 3)))


def _geglu_gate_on_value(x_rows, W1e, b1e, W2e, b2e):
    a = S._f64(x_rows) @ S._f64(W1e).T + S._f64(b1e)[None, :]
    d_ff = a.shape[1] // 2
    h = a[:, :d_ff] * S.gelu(a[:, d_ff:])
    return h @ S._f64(W2e).T + S._f64(b2e)[None, :]


def _forward_noise_everywhere(x, W_r, W1, b1, W2, b2, capacity_factor, b_r=None,
                              activation="relu", router_noise=None):
    # mistake: the experts also see the jittered input
    xs = x if router_noise is None else S._f64(x) * S._f64(router_noise)
    return _orig_forward(xs, W_r, W1, b1, W2, b2, capacity_factor, b_r=b_r,
                         activation=activation)


def _ntlb_no_capacity_clip(e, N, C):
    # mistake: stage 2 counts every stage-1 token as a taken slot (no min with C)
    T = e.shape[0]
    pos = np.full((T, 2), -1, dtype=np.int64)
    count = [0] * N
    for t in range(T):
        pos[t, 0] = count[int(e[t, 0])]
        count[int(e[t, 0])] += 1
    for t in range(T):
        if pos[t, 0] >= C:
            pos[t, 1] = count[int(e[t, 1])]
            count[int(e[t, 1])] += 1
    return pos


def _ntlb_reverse_order(e, N, C):
    # mistake: stage 2 serves the overflow tokens last-first
    T = e.shape[0]
    pos = _orig_positions_ntlb(e, N, C)
    filled = [min(int((e[:, 0] == i).sum()), C) for i in range(N)]
    pos[:, 1] = -1
    for t in reversed(range(T)):
        if pos[t, 0] >= C:
            pos[t, 1] = filled[int(e[t, 1])]
            filled[int(e[t, 1])] += 1
    return pos


def _ntlb_single_stage(e, N, C):
    # mistake: no rerouting at all (the top-1 layer)
    pos = _orig_positions_ntlb(e, N, C)
    pos[:, 1] = -1
    return pos


def _patched_ntlb(old_line: str, new_line: str):
    import inspect
    src = inspect.getsource(_orig_forward_ntlb)
    assert old_line in src, old_line
    ns = dict(vars(S))
    exec(src.replace(old_line, new_line), ns)
    return ns["switch_forward_ntlb"]


def _patched_backward(old_line: str, new_line: str):
    """The oracle's switch_backward with one line replaced (a planted mistake)."""
    import inspect
    src = inspect.getsource(_orig_backward)
    assert old_line in src, old_line
    ns = dict(vars(S))
    exec(src.replace(old_line, new_line), ns)
    return ns["switch_backward"]


MUTATIONS = {
    "ties_to_highest": ("top1", _top1_highest_tie),
    "positions_one_based": ("positions", _positions_one_based),
    "no_relu": ("expert_ffn", _ffn_no_relu),
    "w2_transposed": ("expert_ffn", _ffn_transposed_w2),
    "no_b2": ("expert_ffn", _ffn_no_b2),
    "aux_without_N": ("aux_loss", _aux_no_N),
    "softmax_unshifted": ("router_probs", _probs_no_shift),
    "capacity_floor": ("capacity", _capacity_floor),
    "f_after_cut": ("load_balance_stats", _stats_after_cut),
    "logit_sign": ("router_logits", _logits_sign),
    "gate_one": ("top1", _gate_is_one),
    "gap_top1_minus_min": ("logit_gap", _gap_top1_minus_min),
    "gap_on_probs": ("logit_gap", _gap_on_probs),
    "gap_ties_ignored": ("logit_gap", _gap_distinct_values),
    "top2_second_is_last": ("top2", _top2_second_is_last),
    "top2_never_normalised": ("top2", _top2_never_normalised),
    "top2_capacity_ignores_k": ("capacity_k", _capacity_k_ignores_k),
    "top2_firsts_first": ("positions_top2", _positions_top2_firsts_first),
    "gelu_tanh_approximation": ("gelu", _gelu_tanh),
    "geglu_gate_on_value": ("expert_ffn_geglu", _geglu_gate_on_value),
    "jitter_reaches_experts": ("switch_forward", _forward_noise_everywhere),
}

_orig_positions_ntlb = S.positions_ntlb
_orig_forward_ntlb = S.switch_forward_ntlb
MUTATIONS["ntlb_no_capacity_clip"] = ("positions_ntlb", _ntlb_no_capacity_clip)
MUTATIONS["ntlb_reverse_order"] = ("positions_ntlb", _ntlb_reverse_order)
MUTATIONS["ntlb_single_stage"] = ("positions_ntlb", _ntlb_single_stage)
MUTATIONS["ntlb_first_gate_for_rerouted"] = (
    "switch_forward_ntlb",
    _patched_ntlb("gsel = np.where(stage1, g[:, 0], g[:, 1])", "gsel = g[:, 0]"))
MUTATIONS["ntlb_normalised_gates"] = (
    "switch_forward_ntlb",
    _patched_ntlb("e, g = top2(p, normalize=False)", "e, g = top2(p, normalize=True)"))

_orig_backward = S.switch_backward
_BACKWARD_MUTATIONS = {
    "backward_no_gate_path": ("dz += (dg * g)[:, None] * (onehot - p)",
                              "dz += 0.0 * (onehot - p)"),
    "backward_no_aux_path": ("dz += daux * (N / T) * p * (f[None, :] - (p @ f)[:, None])",
                             "dz += 0.0"),
    "backward_aux_without_mean": ("dz += daux * (N / T) * p * (f[None, :] - (p @ f)[:, None])",
                                  "dz += daux * (N / T) * p * f[None, :]"),
    "backward_gate_not_scaling_du": ("du = g[rows, None] * dy[rows]", "du = dy[rows]"),
    "backward_relu_mask_dropped": ("da = (du @ W2s[i]) * (a > 0)", "da = du @ W2s[i]"),
    "backward_router_grad_to_x_dropped": ("dx += dz @ Wr", "dx += 0.0"),
}
for _name, (_old, _new) in _BACKWARD_MUTATIONS.items():
    MUTATIONS[_name] = ("switch_backward", _patched_backward(_old, _new))

_orig_forward = S.switch_forward

_orig_top2 = S.top2


def _orig_positions(expert_idx, N):
    seen = [0] * N
    out = []
    for e in expert_idx:
        out.append(seen[int(e)])
        seen[int(e)] += 1
    return np.asarray(out, dtype=np.int64)



@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(S, attr, fn)
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            failed.append(pin.__name__)
    assert failed, "planted mistake %r passed every pin" % name
