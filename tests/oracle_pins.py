"""Checks that pin the fp64 oracle to facts fixed by the pages and by mathematics.

Each ``pin_*`` function raises AssertionError when the oracle disagrees.  They
are run as tests in ``test_oracle_pins.py`` and, with mistakes planted in the
oracle, in ``test_oracle_mutations.py`` (each planted mistake must trip a pin).

None of the checks retypes the oracle's own formula: they use the pages'
printed worked example, closed forms, invariants, brute force, or special cases
that reduce to a library routine (torch float64 linear / relu / softmax / sigmoid).
"""
from __future__ import annotations

import itertools
import json
import os
from fractions import Fraction

import numpy as np
import torch
import torch.nn.functional as F

import oracle.switch_layer as S

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _gold(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_ffn(rng, N, d, d_ff, scale=0.5):
    W1 = rng.normal(size=(N, d_ff, d)) * scale
    b1 = rng.normal(size=(N, d_ff)) * 0.1
    W2 = rng.normal(size=(N, d, d_ff)) * scale
    b2 = rng.normal(size=(N, d)) * 0.1
    return W1, b1, W2, b2


# ---------------------------------------------------------------------------
# load-balancing loss: the worked example printed on the "Penalize uneven
# expert traffic" card (N=4, T=8) and its "check your understanding" case.
# ---------------------------------------------------------------------------
def pin_lb_worked_example():
    g = _gold("lb_card_worked_example.json")
    bb = g["book_batch"]
    assert abs(S.aux_loss(bb["f"], bb["P"]) - bb["loss"]) < 1e-12
    assert abs(S.aux_loss(bb["f"], bb["P"]) / bb["N"] - bb["inner_sum"]) < 1e-12
    ev = g["even_router_weights"]
    assert abs(S.aux_loss(ev["f"], ev["P"]) - ev["loss"]) < 1e-12

    # The same batch end to end through router -> softmax -> argmax -> stats.
    # Eight tokens whose router probabilities have argmax counts (3,2,1,2) and
    # column means P; with W_r = I and x_t = log p_t, softmax(W_r x_t) = p_t.
    rows = ([[.60, .20, .05, .15]] * 3 + [[.30, .50, .05, .15]] * 2 +
            [[.30, .10, .45, .15]] + [[.25, .15, .05, .55]] * 2)
    order = [5, 0, 7, 2, 6, 1, 4, 3]          # token order must not matter
    p_rows = np.array(rows)[order]
    x = np.log(p_rows)
    rng = np.random.default_rng(1)
    W1, b1, W2, b2 = _rand_ffn(rng, 4, 4, 3)
    r = S.switch_forward(x, np.eye(4), W1, b1, W2, b2, capacity_factor=1.0)
    assert np.allclose(r["probs"], p_rows, rtol=0, atol=1e-15)
    assert np.array_equal(np.sort(np.bincount(r["expert_idx"], minlength=4)), [1, 2, 2, 3])
    assert np.allclose(r["f"], bb["f"], rtol=0, atol=0)
    assert np.allclose(r["P"], bb["P"], rtol=0, atol=1e-15)
    assert abs(r["aux"] - bb["loss"]) < 1e-12


def pin_even_routing_is_one():
    """Uniform router (W_r = 0): every p_i = 1/N and the loss is exactly 1,
    whatever the traffic split (card 08: 1 whenever p is uniform)."""
    g = _gold("lb_card_worked_example.json")
    rng = np.random.default_rng(2)
    for N in (1, 2, 3, 7):
        T, d = 11, 5
        x = rng.normal(size=(T, d))
        W1, b1, W2, b2 = _rand_ffn(rng, N, d, 4)
        r = S.switch_forward(x, np.zeros((N, d)), W1, b1, W2, b2, capacity_factor=1.0)
        assert abs(r["aux"] - g["even_routing_loss"]) < 1e-12
        assert np.allclose(r["gate"], 1.0 / N, rtol=0, atol=1e-15)
        # all logits tie, so the lowest index wins every token
        assert np.all(r["expert_idx"] == 0)


def pin_collapse_tends_to_N():
    """One expert takes every token with probability -> 1: loss -> N
    (Switch Transformer, explained: 'climbs toward N').  Logits of 1e3 also
    need the max-shifted softmax to stay finite."""
    rng = np.random.default_rng(3)
    for N in (2, 4, 9):
        T, d = 13, 6
        x = rng.normal(size=(T, d))
        b_r = np.zeros(N)
        b_r[N - 1] = 1000.0
        W1, b1, W2, b2 = _rand_ffn(rng, N, d, 3)
        r = S.switch_forward(x, rng.normal(size=(N, d)), W1, b1, W2, b2,
                             capacity_factor=float(N), b_r=b_r)
        assert np.all(r["expert_idx"] == N - 1)
        assert abs(r["aux"] - N) < 1e-9


def pin_not_a_lower_bound():
    """Card 08: for unrelated f and p the value 1 is not a lower bound.
    N=3, p rows (.34,.33,.33) and (.01,.50,.49): f=(1/2,1/2,0),
    P=(.175,.415,.41), loss = 3*(.0875+.2075) = 0.885."""
    p_rows = np.array([[.34, .33, .33], [.01, .50, .49]])
    rng = np.random.default_rng(4)
    W1, b1, W2, b2 = _rand_ffn(rng, 3, 3, 2)
    r = S.switch_forward(np.log(p_rows), np.eye(3), W1, b1, W2, b2, capacity_factor=1.0)
    assert list(r["expert_idx"]) == [0, 1]
    assert abs(r["aux"] - 0.885) < 1e-12


# ---------------------------------------------------------------------------
# softmax and argmax
# ---------------------------------------------------------------------------
def pin_softmax_rows_and_closed_form():
    rng = np.random.default_rng(5)
    z = rng.normal(size=(50, 17)) * 30
    p = S.router_probs(z)
    assert np.all(np.abs(p.sum(axis=1) - 1) < 1e-12)
    assert np.all(p >= 0)
    # N = 2: p_0 = 1 / (1 + exp(z_1 - z_0)) = sigmoid(z_0 - z_1)
    x = rng.normal(size=(40, 6))
    Wr = rng.normal(size=(2, 6)) * 3
    b_r = np.array([0.3, -0.2])
    z2 = S.router_logits(x, Wr, b_r)
    p2 = S.router_probs(z2)
    lib = torch.sigmoid(torch.from_numpy(x @ Wr[0] - x @ Wr[1] + (b_r[0] - b_r[1]))).numpy()
    assert np.allclose(p2[:, 0], lib, rtol=0, atol=1e-12)
    assert np.allclose(p2[:, 1], 1.0 - lib, rtol=0, atol=1e-12)


def pin_ties_lowest_index():
    rng = np.random.default_rng(6)
    d, N = 5, 4
    Wr = np.zeros((N, d))
    Wr[0, 0], Wr[1, 1], Wr[2, 1], Wr[3, 3] = 1.0, 1.0, 1.0, 1.0   # experts 1, 2 equal
    x = rng.normal(size=(9, d))
    x[:, 1] = np.abs(x).max() + 1.0        # experts 1 and 2 tie and beat 0 and 3
    z = S.router_logits(x, Wr)
    e, g = S.top1(S.router_probs(z))
    assert np.all(z[:, 1] == z[:, 2]) and np.all(z[:, 1] > z[:, 0]) and np.all(z[:, 1] > z[:, 3])
    assert np.all(e == 1)
    # the top-1 choice is the largest logit otherwise
    x = rng.normal(size=(200, d))
    z = S.router_logits(x, rng.normal(size=(N, d)))
    e, g = S.top1(S.router_probs(z))
    assert np.array_equal(e, torch.from_numpy(z).argmax(dim=1).numpy())
    assert np.allclose(g, torch.softmax(torch.from_numpy(z), dim=1).max(dim=1).values.numpy(),
                       rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------
# capacity, positions, drops
# ---------------------------------------------------------------------------
def _smallest_integer_at_least(q: Fraction) -> int:
    c = 0
    while c < q:
        c += 1
    return c


def pin_capacity():
    # exact search for the smallest integer >= cf*T/N (positive cf)
    for T in (0, 1, 5, 10, 64, 97):
        for N in (1, 3, 4, 8):
            for cf in (0.25, 0.5, 1.0, 1.1, 1.25, 2.0, 3.75):
                want = _smallest_integer_at_least(Fraction(cf) * T / N)
                assert S.capacity(T, N, cf) == want, (T, N, cf)
    assert S.capacity(10, 4, 1.0) == 3       # ceil(2.5): the ceil reading
    # The five workloads: ceil, floor(T/N)*cf and (T/N)*cf readings coincide,
    # and the tiny / many-expert descriptions print C=16 and C=32.
    table = {(64, 4, 1.0): 16, (4096, 64, 1.25): 80, (16384, 128, 1.0): 128,
             (32768, 64, 2.0): 1024, (65536, 2048, 1.0): 32}
    for (T, N, cf), C in table.items():
        assert S.capacity(T, N, cf) == C
        assert (T // N) * cf == C and T / N * cf == C
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        try:
            S.capacity(10, 2, bad)
        except ValueError:
            continue
        raise AssertionError("capacity accepted cf=%r" % bad)


def pin_positions_bruteforce():
    """All N**T assignments for T <= 6, N <= 3: the kept tokens of each expert
    are exactly its first min(count, C) tokens in index order, and positions
    count up 0,1,2,... along each expert's tokens."""
    for T in range(0, 7):
        for N in range(1, 4):
            for assign in itertools.product(range(N), repeat=T):
                pos = S.positions(list(assign), N)
                for i in range(N):
                    toks = [t for t in range(T) if assign[t] == i]
                    assert sorted(pos[toks].tolist()) == list(range(len(toks)))
                    assert all(pos[a] < pos[b] for a, b in zip(toks, toks[1:]))
                    for C in range(0, T + 2):
                        kept = [t for t in toks if pos[t] < C]
                        assert kept == toks[:min(len(toks), C)]


def pin_drops():
    """A capacity cut only removes tokens: dropped rows are exactly zero and
    kept rows equal the uncut layer's rows.  Large cf (C >= T) drops nothing."""
    rng = np.random.default_rng(7)
    T, d, d_ff, N = 40, 6, 5, 3
    x = rng.normal(size=(T, d))
    Wr = rng.normal(size=(N, d))
    Wr[0] *= 3
    W1, b1, W2, b2 = _rand_ffn(rng, N, d, d_ff)
    full = S.switch_forward(x, Wr, W1, b1, W2, b2, capacity_factor=float(N))
    assert full["kept"].all() and full["capacity"] >= T
    cut = S.switch_forward(x, Wr, W1, b1, W2, b2, capacity_factor=0.5)
    assert (~cut["kept"]).any()
    assert np.all(cut["out"][~cut["kept"]] == 0.0)
    assert np.array_equal(cut["out"][cut["kept"]], full["out"][cut["kept"]])
    assert np.array_equal(cut["expert_idx"], full["expert_idx"])
    # f counts argmax choices before the cut: it still sums to one
    assert abs(cut["f"].sum() - 1.0) < 1e-15
    assert np.array_equal(cut["f"], full["f"]) and np.array_equal(cut["P"], full["P"])


# ---------------------------------------------------------------------------
# expert FFN and gate, via special cases that reduce to library routines
# ---------------------------------------------------------------------------
def _torch_ffn(x, W1, b1, W2, b2):
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    return F.linear(F.relu(F.linear(t(x), t(W1), t(b1))), t(W2), t(b2)).numpy()


def pin_single_expert_is_dense_ffn():
    """N = 1: p = 1, C = ceil(cf*T) >= T for cf >= 1: the layer is the dense FFN
    W_2 relu(W_1 x + b_1) + b_2 of the "Dense FFN Baseline" section."""
    rng = np.random.default_rng(8)
    for T, d, d_ff in ((23, 7, 9), (17, 8, 8)):      # square case: W_2 vs W_2^T
        x = rng.normal(size=(T, d))
        W1, b1, W2, b2 = _rand_ffn(rng, 1, d, d_ff)
        r = S.switch_forward(x, rng.normal(size=(1, d)), W1, b1, W2, b2, capacity_factor=1.0)
        ref = _torch_ffn(x, W1[0], b1[0], W2[0], b2[0])
        assert np.all(r["gate"] == 1.0) and r["kept"].all()
        assert np.allclose(r["out"], ref, rtol=1e-13, atol=1e-13)


def pin_identical_experts_scale_by_gate():
    """All experts equal to one FFN and no drops: y_t = max_i softmax(z_t)_i * FFN(x_t)
    (y_t = g_t E_{e_t}(x_t) with b_2 inside E)."""
    rng = np.random.default_rng(9)
    T, d, d_ff, N = 31, 6, 8, 5
    x = rng.normal(size=(T, d))
    W1, b1, W2, b2 = _rand_ffn(rng, 1, d, d_ff)
    rep = lambda a: np.repeat(a, N, axis=0)
    Wr = rng.normal(size=(N, d))
    b_r = rng.normal(size=N)
    r = S.switch_forward(x, Wr, rep(W1), rep(b1), rep(W2), rep(b2),
                         capacity_factor=float(N), b_r=b_r)
    z = torch.from_numpy(x) @ torch.from_numpy(Wr).T + torch.from_numpy(b_r)
    g = torch.softmax(z, dim=1).max(dim=1).values.numpy()
    ref = g[:, None] * _torch_ffn(x, W1[0], b1[0], W2[0], b2[0])
    assert np.allclose(r["out"], ref, rtol=1e-13, atol=1e-13)


def pin_sampled_matches_full():
    rng = np.random.default_rng(10)
    T, d, d_ff, N = 300, 8, 6, 7
    x = rng.normal(size=(T, d))
    Wr = rng.normal(size=(N, d))
    W1, b1, W2, b2 = _rand_ffn(rng, N, d, d_ff)
    full = S.switch_forward(x, Wr, W1, b1, W2, b2, capacity_factor=1.0)
    samp = rng.choice(T, size=60, replace=False)
    part = S.switch_forward_sampled(
        x, Wr, 1.0, samp, lambda e: {"W1": W1[e], "b1": b1[e], "W2": W2[e], "b2": b2[e]},
        chunk=64)
    for k in ("expert_idx", "pos_in_expert", "kept"):
        assert np.array_equal(full[k], part[k])
    assert np.allclose(full["gate"], part["gate"], rtol=0, atol=1e-15)
    assert abs(full["aux"] - part["aux"]) < 1e-12
    for t in samp:
        assert np.allclose(part["out_rows"][int(t)], full["out"][t], rtol=1e-13, atol=1e-13)


def _gap_bruteforce(z_row):
    """max over experts i of min over j != i of (z_i - z_j), by explicit pairs:
    for the winning expert this is its margin over the runner-up; every other
    expert scores <= 0, and an exact tie at the top gives 0."""
    N = len(z_row)
    best = -np.inf
    for i in range(N):
        worst = np.inf
        for j in range(N):
            if j != i:
                worst = min(worst, float(z_row[i]) - float(z_row[j]))
        best = max(best, worst)
    return best


def pin_logit_gap():
    """The router-logit gap that decides which seeded token rows are redrawn
    (top-1 minus top-2 logit, on logits, not probabilities)."""
    rng = np.random.default_rng(11)
    # brute force over ordered pairs on small random rows, N = 2..6
    for N in range(2, 7):
        z = rng.normal(size=(40, N)) * 2.0
        g = S.logit_gap(z)
        want = np.array([_gap_bruteforce(r) for r in z])
        assert np.array_equal(g, want), N
    # N = 2: |z_0 - z_1| exactly
    z = rng.normal(size=(100, 2))
    assert np.array_equal(S.logit_gap(z), np.abs(z[:, 0] - z[:, 1]))
    # a constructed exact tie at the top gives 0; a tie below the top does not matter
    z = rng.normal(size=(30, 5))
    top = z.max(axis=1) + 1.0
    z[:, 1] = top
    z[:, 3] = top
    assert np.all(S.logit_gap(z) == 0.0)
    z = np.array([[3.0, 1.0, 1.0, 0.5], [0.0, -2.0, 5.0, -2.0]])
    assert np.array_equal(S.logit_gap(z), [2.0, 5.0])
    # a gap of logits: unchanged by a per-row shift, scaled by a positive scale
    # (a gap of probabilities is neither)
    z = rng.normal(size=(50, 7))
    shift = rng.normal(size=(50, 1)) * 10
    assert np.allclose(S.logit_gap(z + shift), S.logit_gap(z), rtol=0, atol=1e-12)
    assert np.allclose(S.logit_gap(4.0 * z), 4.0 * S.logit_gap(z), rtol=0, atol=1e-12)
    # one expert: no runner-up, never redrawn
    assert np.all(np.isinf(S.logit_gap(rng.normal(size=(4, 1)))))


# ---------------------------------------------------------------------------
# top-2 routing (the earlier-MoE variant)
# ---------------------------------------------------------------------------
def _const_experts(outputs, d, extra):
    """Experts whose output is a constant row: W1 = 0, b1 = 1 (h = 1), W2 = 0,
    b2 = the row.  outputs: list of d-vectors; extra: further constant rows."""
    rows = np.array(list(outputs) + list(extra), dtype=np.float64)
    N = rows.shape[0]
    return (np.zeros((N, 1, d)), np.ones((N, 1)), np.zeros((N, d, 1)), rows)


def pin_top2_worked_example():
    """The attention-and-MoE note's example: router weights [0.6, 0.3, 0.1],
    top-2 normalised to [2/3, 1/3]; expert outputs [3,0] and [0,6] merge to
    [2,2].  Unnormalised (the reading note's formula): [1.8, 1.8]."""
    g = _gold("top2_worked_example.json")
    p = np.array([g["router_weights"]])
    x = np.log(p)                          # W_r = I: softmax(W_r x) = p
    W1, b1, W2, b2 = _const_experts([o + [0.0] for o in g["expert_outputs"]], 3,
                                    [[1.0, 1.0, 1.0]])
    r = S.switch_forward_top2(x, np.eye(3), W1, b1, W2, b2, capacity_factor=1.0)
    assert r["expert_idx"].tolist() == [[0, 1]]
    assert np.allclose(r["gate"][0], g["normalised_gates"], rtol=0, atol=1e-15)
    assert np.allclose(r["out"][0, :2], g["merged_output"], rtol=0, atol=1e-14)
    assert r["out"][0, 2] == 0.0
    r = S.switch_forward_top2(x, np.eye(3), W1, b1, W2, b2, capacity_factor=1.0,
                              normalize=False)
    assert np.allclose(r["out"][0, :2], g["merged_output_unnormalised"], rtol=0, atol=1e-14)


def pin_top2_choices_and_capacity():
    """Second choice = the runner-up logit (torch.topk), ties to the lowest
    index; capacity ceil(2 cf T / N) by exact search."""
    rng = np.random.default_rng(12)
    z = rng.normal(size=(300, 6))
    e, g = S.top2(S.router_probs(z), normalize=False)
    tk = torch.topk(torch.from_numpy(z), 2, dim=1)
    assert np.array_equal(e, tk.indices.numpy())
    assert np.allclose(g, torch.softmax(torch.from_numpy(z), 1).gather(1, tk.indices).numpy(),
                       rtol=0, atol=1e-15)
    # exact ties: three equal largest logits -> experts 1 and 2; two equal
    # runners-up below a clear winner -> the lower of them
    z = np.array([[0.0, 5.0, 5.0, 5.0], [9.0, 1.0, 3.0, 3.0]])
    e, _ = S.top2(S.router_probs(z))
    assert e.tolist() == [[1, 2], [0, 2]]
    for T in (0, 1, 7, 64, 97):
        for N in (2, 3, 8):
            for cf in (0.25, 1.0, 1.25, 2.0):
                want = _smallest_integer_at_least(Fraction(cf) * 2 * T / N)
                assert S.capacity_k(T, N, cf, 2) == want
    assert S.capacity_k(4096, 64, 1.25, 1) == S.capacity(4096, 64, 1.25)


def pin_top2_positions_bruteforce():
    """All top-2 assignments of T <= 5 tokens to N = 3 experts: each expert's
    kept assignments are its first min(count, C) in token order."""
    pairs = [(a, b) for a in range(3) for b in range(3) if a != b]
    for T in range(0, 5):
        for assign in itertools.product(pairs, repeat=T):
            e = np.array(assign, dtype=np.int64).reshape(T, 2)
            pos = S.positions_top2(e, 3)
            for i in range(3):
                toks = [t for t in range(T) if i in assign[t]]
                got = [int(pos[t, assign[t].index(i)]) for t in toks]
                assert got == list(range(len(toks)))


def pin_top2_closed_forms():
    """Identical experts, normalised gates, no drops: y = E(x) exactly (the two
    gates sum to one).  Two experts, no drops: y = p_0 E_0(x) + p_1 E_1(x)."""
    rng = np.random.default_rng(13)
    T, d, d_ff, N = 40, 6, 7, 4
    x = rng.normal(size=(T, d))
    W1, b1, W2, b2 = _rand_ffn(rng, 1, d, d_ff)
    rep = lambda a: np.repeat(a, N, axis=0)
    r = S.switch_forward_top2(x, rng.normal(size=(N, d)), rep(W1), rep(b1), rep(W2), rep(b2),
                              capacity_factor=float(N))
    assert r["kept"].all()
    assert np.allclose(r["out"], _torch_ffn(x, W1[0], b1[0], W2[0], b2[0]), rtol=1e-13,
                       atol=1e-13)
    W1, b1, W2, b2 = _rand_ffn(rng, 2, d, d_ff)
    Wr = rng.normal(size=(2, d))
    for norm in (True, False):
        r = S.switch_forward_top2(x, Wr, W1, b1, W2, b2, capacity_factor=2.0, normalize=norm)
        p = torch.softmax(torch.from_numpy(x @ Wr.T), dim=1).numpy()
        ref = (p[:, :1] * _torch_ffn(x, W1[0], b1[0], W2[0], b2[0]) +
               p[:, 1:] * _torch_ffn(x, W1[1], b1[1], W2[1], b2[1]))
        assert np.allclose(r["out"], ref, rtol=1e-13, atol=1e-13)
    # the aux loss counts first choices: it equals the top-1 layer's
    top1 = S.switch_forward(x, Wr, W1, b1, W2, b2, capacity_factor=2.0)
    assert abs(r["aux"] - top1["aux"]) < 1e-15


def pin_top2_drops():
    """A capacity cut removes assignments only: kept assignments contribute
    exactly what they contribute without the cut."""
    rng = np.random.default_rng(14)
    T, d, d_ff, N = 60, 5, 6, 4
    x = rng.normal(size=(T, d))
    Wr = rng.normal(size=(N, d))
    Wr[0] *= 3
    W1, b1, W2, b2 = _rand_ffn(rng, N, d, d_ff)
    full = S.switch_forward_top2(x, Wr, W1, b1, W2, b2, capacity_factor=float(N))
    cut = S.switch_forward_top2(x, Wr, W1, b1, W2, b2, capacity_factor=0.5)
    assert full["kept"].all() and (~cut["kept"]).any() and cut["capacity"] == 15
    for t in range(T):
        want = np.zeros(d)
        for k in range(2):
            if cut["kept"][t, k]:
                e = cut["expert_idx"][t, k]
                want += cut["gate"][t, k] * _torch_ffn(x[t:t + 1], W1[e], b1[e], W2[e], b2[e])[0]
        assert np.allclose(cut["out"][t], want, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------
# GEGLU experts and router input jitter
# ---------------------------------------------------------------------------
def pin_gelu():
    """Exact GELU: torch's erf form (a library routine), GELU(u) - GELU(-u) = u,
    GELU(0) = 0, and the limits u and 0 far from zero."""
    u = np.linspace(-8, 8, 1001)
    lib = F.gelu(torch.from_numpy(u), approximate="none").numpy()
    assert np.allclose(S.gelu(u), lib, rtol=0, atol=1e-15)
    assert np.allclose(S.gelu(u) - S.gelu(-u), u, rtol=0, atol=1e-14)
    assert S.gelu(np.array([0.0]))[0] == 0.0
    assert abs(S.gelu(np.array([40.0]))[0] - 40.0) < 1e-12 and S.gelu(np.array([-40.0]))[0] == 0


def pin_geglu_special_cases():
    """W_v = 0, b_v = 1: the GEGLU expert is the GELU FFN W2 GELU(W_g x + b_g) + b2
    (torch linear / gelu); scaling the value branch by c scales E(x) - b2 by c."""
    rng = np.random.default_rng(15)
    T, d, d_ff = 17, 6, 5
    x = rng.normal(size=(T, d))
    Wg = rng.normal(size=(d_ff, d))
    bg = rng.normal(size=d_ff) * 0.3
    W2 = rng.normal(size=(d, d_ff))
    b2 = rng.normal(size=d) * 0.1
    W1 = np.concatenate([Wg, np.zeros((d_ff, d))])
    b1 = np.concatenate([bg, np.ones(d_ff)])
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    ref = F.linear(F.gelu(F.linear(t(x), t(Wg), t(bg))), t(W2), t(b2)).numpy()
    assert np.allclose(S.expert_ffn_geglu(x, W1, b1, W2, b2), ref, rtol=1e-13, atol=1e-13)
    Wv = rng.normal(size=(d_ff, d))
    bv = rng.normal(size=d_ff)
    base = S.expert_ffn_geglu(x, np.concatenate([Wg, Wv]), np.concatenate([bg, bv]), W2, b2)
    scaled = S.expert_ffn_geglu(x, np.concatenate([Wg, 3 * Wv]), np.concatenate([bg, 3 * bv]),
                                W2, b2)
    assert np.allclose(scaled - b2, 3 * (base - b2), rtol=1e-12, atol=1e-12)
    # the layer with one expert and GEGLU is that expert's FFN
    r = S.switch_forward(x, rng.normal(size=(1, d)), W1[None], b1[None], W2[None], b2[None], 1.0,
                         activation="geglu")
    assert np.allclose(r["out"], ref, rtol=1e-13, atol=1e-13)


def pin_router_jitter():
    """Jitter multiplies the router input only.  Unit noise is the inference
    layer; a constant noise c scales every logit by c (gate = max softmax(c z),
    torch), while the experts still see x itself."""
    rng = np.random.default_rng(16)
    T, d, d_ff, N = 30, 6, 7, 4
    x = rng.normal(size=(T, d))
    Wr = rng.normal(size=(N, d))
    W1, b1, W2, b2 = _rand_ffn(rng, N, d, d_ff)
    plain = S.switch_forward(x, Wr, W1, b1, W2, b2, float(N))
    ones = S.switch_forward(x, Wr, W1, b1, W2, b2, float(N), router_noise=np.ones((T, d)))
    for k in ("out", "gate", "expert_idx", "aux"):
        assert np.array_equal(np.asarray(plain[k]), np.asarray(ones[k])), k
    c = 3.5
    r = S.switch_forward(x, Wr, W1, b1, W2, b2, float(N), router_noise=np.full((T, d), c))
    z = c * (torch.from_numpy(x) @ torch.from_numpy(Wr).T)
    g = torch.softmax(z, dim=1).max(dim=1).values.numpy()
    e = z.argmax(dim=1).numpy()
    assert np.array_equal(r["expert_idx"], e)
    assert np.allclose(r["gate"], g, rtol=0, atol=1e-15)
    for t0 in range(T):
        want = g[t0] * _torch_ffn(x[t0:t0 + 1], W1[e[t0]], b1[e[t0]], W2[e[t0]], b2[e[t0]])[0]
        assert np.allclose(r["out"][t0], want, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------
# backward: central finite differences of L = sum(dout * out) + daux * aux
# (routing is piecewise constant; inputs keep every decision far from a switch)
# ---------------------------------------------------------------------------
def _loss(x, Wr, W1, b1, W2, b2, cf, dout, daux, b_r):
    r = S.switch_forward(x, Wr, W1, b1, W2, b2, cf, b_r=b_r)
    return float(np.sum(dout * r["out"]) + daux * r["aux"]), r


def pin_backward_finite_differences():
    rng = np.random.default_rng(17)
    T, d, d_ff, N, cf = 12, 4, 5, 3, 1.0        # C = 4: some tokens are dropped
    x = rng.normal(size=(T, d))
    Wr = rng.normal(size=(N, d))
    b_r = rng.normal(size=N) * 0.2
    W1, b1, W2, b2 = _rand_ffn(rng, N, d, d_ff)
    b1 = b1 + 0.05                              # keep pre-activations away from 0 ...
    dout = rng.normal(size=(T, d))
    daux = 0.7
    base, r = _loss(x, Wr, W1, b1, W2, b2, cf, dout, daux, b_r)
    assert (~r["kept"]).any() and r["kept"].any()
    gr = S.switch_backward(x, Wr, W1, b1, W2, b2, cf, dout, daux, b_r=b_r)
    eps = 1e-6
    params = {"dx": x, "dW_r": Wr, "db_r": b_r, "dW1": W1, "db1": b1, "dW2": W2, "db2": b2}
    for name, arr in params.items():
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + eps
            lp, rp = _loss(x, Wr, W1, b1, W2, b2, cf, dout, daux, b_r)
            arr[idx] = old - eps
            lm, rm = _loss(x, Wr, W1, b1, W2, b2, cf, dout, daux, b_r)
            arr[idx] = old
            # the perturbation must not move a routing decision or a ReLU kink
            assert np.array_equal(rp["expert_idx"], r["expert_idx"])
            assert np.array_equal(rm["kept"], r["kept"])
            num[idx] = (lp - lm) / (2 * eps)
        assert np.allclose(gr[name], num, rtol=1e-6, atol=1e-7), name


def pin_backward_dense_ffn():
    """N = 1: no router gradient (p = 1), and dx, dW1, db1, dW2, db2 are torch
    autograd's of the dense FFN."""
    rng = np.random.default_rng(18)
    T, d, d_ff = 9, 5, 6
    x = rng.normal(size=(T, d))
    W1, b1, W2, b2 = _rand_ffn(rng, 1, d, d_ff)
    dout = rng.normal(size=(T, d))
    gr = S.switch_backward(x, rng.normal(size=(1, d)), W1, b1, W2, b2, 1.0, dout, daux=0.5)
    t = [torch.tensor(a, dtype=torch.float64, requires_grad=True)
         for a in (x, W1[0], b1[0], W2[0], b2[0])]
    y = F.linear(F.relu(F.linear(t[0], t[1], t[2])), t[3], t[4])
    (y * torch.from_numpy(dout)).sum().backward()
    for k, ten in zip(("dx", "dW1", "db1", "dW2", "db2"), t):
        got = gr[k] if k == "dx" else gr[k][0]
        assert np.allclose(got, ten.grad.numpy(), rtol=1e-12, atol=1e-12), k
    assert np.all(gr["dW_r"] == 0) and np.all(gr["db_r"] == 0)


# ---------------------------------------------------------------------------
# No-Token-Left-Behind (two stages; readings in the oracle's module doc)
# ---------------------------------------------------------------------------
def pin_ntlb_worked_example():
    """The hand-derived two-stage examples of the golden fixture: positions and
    the expert that keeps each token."""
    for g in _gold("ntlb_worked_example.json")["examples"]:
        e = np.array(g["choices"], dtype=np.int64)
        C = g["C"]
        pos = S.positions_ntlb(e, g["N"], C)
        assert pos.tolist() == g["positions"]
        got = [int(e[t, 0]) if pos[t, 0] < C else (int(e[t, 1]) if 0 <= pos[t, 1] < C else -1)
               for t in range(len(e))]
        assert got == g["assigned"]


def _ntlb_by_sets(e, N, C):
    """Assignment of a two-stage reroute written with sets: expert i keeps the
    first C tokens choosing it first; of the tokens it dropped, token order
    decides which take the slots left at their second choice."""
    T = e.shape[0]
    first = {i: [t for t in range(T) if e[t, 0] == i] for i in range(N)}
    kept1 = {t for i in range(N) for t in first[i][:C]}
    out = {t: int(e[t, 0]) for t in kept1}
    for i in range(N):
        free = C - min(len(first[i]), C)
        cands = [t for t in range(T) if t not in kept1 and e[t, 1] == i]
        for t in cands[:free]:
            out[t] = i
    return [out.get(t, -1) for t in range(T)]


def pin_ntlb_bruteforce():
    """Every first/second-choice assignment of T <= 5 tokens to N = 3 experts,
    C in 0..3: the positions give the set-based assignment, stage 1 equals the
    top-1 positions, and no expert keeps more than C tokens."""
    pairs = [(a, b) for a in range(3) for b in range(3) if a != b]
    for T in range(0, 6):
        for assign in itertools.product(pairs, repeat=T):
            e = np.array(assign, dtype=np.int64).reshape(T, 2)
            top1_pos = S.positions(e[:, 0], 3)
            for C in range(4):
                pos = S.positions_ntlb(e, 3, C)
                assert np.array_equal(pos[:, 0], top1_pos)
                got = [int(e[t, 0]) if pos[t, 0] < C else
                       (int(e[t, 1]) if 0 <= pos[t, 1] < C else -1) for t in range(T)]
                assert got == _ntlb_by_sets(e, 3, C)
                for i in range(3):
                    assert got.count(i) <= C


def pin_ntlb_reduces_and_reroutes():
    """Without drops in stage 1 the layer is the top-1 layer; otherwise stage-1
    tokens keep their top-1 rows, rerouted tokens get p_e2 E_e2(x) (torch
    reference), and the aux loss is the top-1 loss."""
    rng = np.random.default_rng(21)
    T, d, d_ff, N = 60, 6, 5, 4
    x = rng.normal(size=(T, d))
    Wr = rng.normal(size=(N, d)) * 2.0
    W1, b1, W2, b2 = _rand_ffn(rng, N, d, d_ff)
    for cf in (float(N), 1.0, 0.75):
        r = S.switch_forward_ntlb(x, Wr, W1, b1, W2, b2, capacity_factor=cf)
        t1 = S.switch_forward(x, Wr, W1, b1, W2, b2, capacity_factor=cf)
        k1 = t1["kept"]
        assert np.array_equal(r["assigned"][k1], t1["expert_idx"][k1])
        assert np.allclose(r["out"][k1], t1["out"][k1], rtol=1e-13, atol=1e-13)
        assert abs(r["aux"] - t1["aux"]) < 1e-13
        p = torch.softmax(torch.from_numpy(x @ Wr.T), dim=1).numpy()
        re = np.nonzero((~k1) & (r["assigned"] >= 0))[0]
        if cf == float(N):
            assert k1.all() and re.size == 0
            assert np.allclose(r["out"], t1["out"], rtol=1e-13, atol=1e-13)
        else:
            assert re.size > 0
        for t in re:
            i = int(r["assigned"][t])
            assert i == int(np.argsort(-p[t], kind="stable")[1])
            ref = p[t, i] * _torch_ffn(x[t:t + 1], W1[i], b1[i], W2[i], b2[i])[0]
            assert np.allclose(r["out"][t], ref, rtol=1e-13, atol=1e-13)
        dropped = np.nonzero(r["assigned"] < 0)[0]
        assert not r["out"][dropped].any()
        assert (r["assigned"] >= 0).sum() >= k1.sum()


ALL_PINS = [
    pin_lb_worked_example, pin_even_routing_is_one, pin_collapse_tends_to_N,
    pin_not_a_lower_bound, pin_softmax_rows_and_closed_form, pin_ties_lowest_index,
    pin_capacity, pin_positions_bruteforce, pin_drops, pin_single_expert_is_dense_ffn,
    pin_identical_experts_scale_by_gate, pin_sampled_matches_full, pin_logit_gap,
    pin_top2_worked_example, pin_top2_choices_and_capacity, pin_top2_positions_bruteforce,
    pin_top2_closed_forms, pin_top2_drops, pin_gelu, pin_geglu_special_cases, pin_router_jitter,
    pin_backward_finite_differences, pin_backward_dense_ffn,
    pin_ntlb_worked_example, pin_ntlb_bruteforce, pin_ntlb_reduces_and_reroutes,
]
