"""Plain fp64 oracle of one Switch Transformer layer, forward pass.

TEST INFRASTRUCTURE.  Imported only by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product path.

Sources (web pages on the Switch Transformer; cited by page title and section):

* [ST-note]  "Switch Transformer" reading note (eightmm.github.io), sections
  "Router", "Expert FFN Layer", "Dense FFN Baseline", "Capacity Factor",
  "Load-Balancing Loss", "Batch and Sequence Shape".
* [ST-paper] "Switch Transformers: Scaling to Trillion Parameter Models with
  Simple and Efficient Sparsity" (paper-graph summary of arXiv 2101.03961),
  section 3.4: "The mathematics of routing", "The loss formulation", the
  expert-capacity formula, "The routing mechanics in detail", "The selective
  precision solution".
* [ST-explained] "Switch Transformer, explained." (vibeengines), recipe steps 2-5.
* [LB-card] "Chapter 8 - Attention and Transformers" companion, card 08
  "Penalize uneven expert traffic".

Every floating-point step runs in float64 on inputs upcast exactly from their
stored fp32 / bf16 values.  Matrices act on column vectors as [ST-note] writes
them: z_t = W_r x_t, W_1 in R^{d_ff x d}, W_2 in R^{d x d_ff}; stored row-major
as W_r [N, d], W1 [N, d_ff, d], W2 [N, d, d_ff].

Readings where the pages are silent or disagree:

* capacity: C = ceil(capacity_factor * T / N) with the exact rational value of
  the given double ([ST-note] "Capacity Factor"; [ST-paper] prints a floor
  variant, [ST-explained] no rounding -- all agree when cf*T/N is an integer).
* argmax ties go to the lowest expert index (pages silent).
* positions are 0-based ranks in token order; a token is dropped iff its
  position >= C ([ST-paper] routing mechanics: cumsum over each expert's column
  in token order, overflow masked).
* f_i counts the argmax choices before the capacity cut ([ST-paper] loss
  formulation, indicator on argmax); aux is returned without the alpha factor.
* dropped tokens get a zero layer output; no residual is added here.
* b_2 sits inside the gate: y = g * (W_2 relu(W_1 x + b_1) + b_2)
  ([ST-note] "Expert FFN Layer" and "Router": y_t = g_t E_{e_t}(x_t)).
* an empty batch (T = 0) gives no outputs and aux = 0.

Top-2 variant (the earlier-MoE routing the pages compare Switch with):

* [ST-note] "Comparison to Earlier MoE": y_t = sum over the two largest p_t,i
  of p_t,i E_i(x_t) (gates unnormalised); [MoE-note] the attention-and-MoE note
  (doc.liz6.com), "From Dense FFN to Sparse Experts": the two selected weights
  are normalised within the selected set ([0.6, 0.3, 0.1] -> [2/3, 1/3]).  Both
  are provided (``normalize``).
* capacity: proportional to k * tokens / N * capacity factor for top-k
  ([ST-paper] "Expert capacity can be at least halved"): C = ceil(2 cf T / N).
* positions: the cumulative sum over each expert's column of the top-2
  dispatch mask in token order (a token's two experts differ, so its two
  assignments never compete for one column); an assignment is dropped iff its
  position >= C; a token's output sums its kept assignments.
* f_i still counts the argmax (first choice), as the loss formula's indicator
  does; P_i is the mean router probability.

Backward pass ([ST-explained] "Why one expert is enough": the chosen expert's
output is scaled by its own probability, so the gradient reaches the router
through the gate; [ST-paper] "The loss formulation": f_i is a count with no
gradient, the balancing gradient flows through P_i only; argmax, positions and
the capacity cut are piecewise constant and pass no gradient):

* upstream gradients dout [T, d] of the layer output and daux of the aux loss;
* kept token t (expert e, gate g, a = W1[e] x + b1[e], h = relu(a),
  u = W2[e] h + b2[e], y = g u): du = g dout_t, dW2[e] += du h^T, db2[e] += du,
  da = (W2[e]^T du) * [a > 0] (ReLU'(0) = 0), dW1[e] += da x^T, db1[e] += da,
  dx_t += W1[e]^T da, and the gate's gradient dg_t = dout_t . u;
* router logits: dz_t,j = dg_t g (delta_{j e} - p_t,j) for kept t, plus
  daux (N / T) p_t,j (f_j - sum_i f_i p_t,i) for every t (aux = N sum f_i P_i,
  P_i = mean_t p_t,i);
* dW_r = sum_t dz_t x_t^T (the router's input: x, or x * noise), db_r = sum_t dz_t,
  dx_t += W_r^T dz_t.

No-Token-Left-Behind ([ST-paper] Appendix B, in the capacity-factor discussion
and the router-design list: tokens that overflow their first expert are sent to
their second-choice expert, "iteratively", a two-stage process in its Figure 11;
the paper reports no benefit).  The figure itself is not in the pages; readings:

* two stages: stage 1 is the top-1 layer (first choice, capacity
  C = ceil(cf T / N), positions in token order); stage 2 takes the tokens that
  stage 1 dropped, in token order, and offers each to its second choice (the
  top-2 runner-up), whose free slots are those stage 1 left: the position of an
  overflow token there is min(count_1(e), C) + (earlier overflow tokens with the
  same second choice); it is kept iff that position < C, else dropped for good.
* a kept token's output is p_t,e E_e(x_t) with e the expert that kept it (the
  gate is that expert's router probability, unnormalised); dropped tokens give 0.
* f_i counts first choices, as in the top-1 loss formula (the rerouting is not
  part of the router's decision).

GEGLU experts and router input jitter ([ST-paper] architecture paragraph: "ReLU
or GEGLU"; Table 11: input jitter, multiplicative noise on the router input,
a training-time exploration, off at inference).  The pages name both without
defining them; the readings taken:

* GEGLU expert: E(x) = W_2 (GELU(W_g x + b_g) * (W_v x + b_v)) + b_2, stored as
  W1 = [W_g; W_v] [2 d_ff, d] and b1 = [b_g; b_v] [2 d_ff], with the exact
  GELU(u) = u Phi(u) = u (1 + erf(u / sqrt 2)) / 2.
* jitter: the router sees x * n for a caller-supplied multiplicative noise n
  [T, d] (the noise law is not stated; the tests draw n ~ U(1 - eps, 1 + eps));
  the experts see x itself.  No noise (None) is the inference layer.
"""
from __future__ import annotations

import math
from fractions import Fraction
from typing import Callable, Dict, Iterable, Optional

import numpy as np


def _f64(a) -> np.ndarray:
    """Exact upcast of an fp32/bf16 array (numpy or torch, any device) to float64."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# capacity  ([ST-note] "Capacity Factor": C = ceil(T/N * alpha))
# ---------------------------------------------------------------------------
def capacity(T: int, N: int, capacity_factor: float) -> int:
    """Expert capacity ceil(cf * T / N), evaluated exactly on the double cf."""
    if N <= 0 or T < 0 or not math.isfinite(capacity_factor) or capacity_factor <= 0:
        raise ValueError("invalid capacity arguments")
    return math.ceil(Fraction(capacity_factor) * T / N)


# ---------------------------------------------------------------------------
# router  ([ST-paper] 3.4 "The mathematics of routing"; [ST-note] "Router")
# ---------------------------------------------------------------------------
def router_logits(x, W_r, b_r=None) -> np.ndarray:
    """h(x_t) = W_r x_t (+ b_r): logits [T, N] in float64."""
    z = _f64(x) @ _f64(W_r).T
    if b_r is not None:
        z = z + _f64(b_r)[None, :]
    return z


def router_probs(z: np.ndarray) -> np.ndarray:
    """p_i = exp(h_i) / sum_j exp(h_j) over the N experts (max-shifted)."""
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=1, keepdims=True)


def top1(p: np.ndarray):
    """e_t = argmax_i p_{t,i} (lowest index on ties) and gate g_t = p_{t,e_t}."""
    e = np.argmax(p, axis=1)          # numpy returns the first maximal index
    g = p[np.arange(p.shape[0]), e]
    return e.astype(np.int64), g


def logit_gap(z: np.ndarray) -> np.ndarray:
    """Top-1 minus top-2 logit per token (inf when N == 1)."""
    if z.shape[1] < 2:
        return np.full(z.shape[0], np.inf)
    s = np.sort(z, axis=1)
    return s[:, -1] - s[:, -2]


# ---------------------------------------------------------------------------
# positions and drops ([ST-paper] "The routing mechanics in detail")
# ---------------------------------------------------------------------------
def positions(expert_idx: Iterable[int], N: int) -> np.ndarray:
    """pos_t = number of earlier tokens (in token order) routed to e_t."""
    seen = [0] * N
    out = []
    for e in expert_idx:
        out.append(seen[int(e)])
        seen[int(e)] += 1
    return np.asarray(out, dtype=np.int64)


# ---------------------------------------------------------------------------
# expert FFN ([ST-note] "Expert FFN Layer": E_i(x) = W_2i relu(W_1i x + b_1i) + b_2i)
# ---------------------------------------------------------------------------
def expert_ffn(x_rows, W1e, b1e, W2e, b2e) -> np.ndarray:
    """E(x) for rows of x: relu(x W1^T + b1) W2^T + b2, float64."""
    h = _f64(x_rows) @ _f64(W1e).T + _f64(b1e)[None, :]
    h = np.maximum(h, 0.0)
    return h @ _f64(W2e).T + _f64(b2e)[None, :]


def gelu(u: np.ndarray) -> np.ndarray:
    """GELU(u) = u Phi(u) = u (1 + erf(u / sqrt 2)) / 2 (the exact form)."""
    from scipy.special import erf
    u = np.asarray(u, dtype=np.float64)
    return 0.5 * u * (1.0 + erf(u / math.sqrt(2.0)))


def expert_ffn_geglu(x_rows, W1e, b1e, W2e, b2e) -> np.ndarray:
    """GEGLU expert for rows of x: W1e = [W_g; W_v] [2 d_ff, d], b1e = [b_g; b_v];
    (GELU(x W_g^T + b_g) * (x W_v^T + b_v)) W2^T + b2, float64."""
    a = _f64(x_rows) @ _f64(W1e).T + _f64(b1e)[None, :]
    d_ff = a.shape[1] // 2
    h = gelu(a[:, :d_ff]) * a[:, d_ff:]
    return h @ _f64(W2e).T + _f64(b2e)[None, :]


def _ffn_of(activation: str):
    if activation == "relu":
        return expert_ffn
    if activation == "geglu":
        return expert_ffn_geglu
    raise ValueError(activation)


# ---------------------------------------------------------------------------
# load-balancing loss ([ST-paper] "The loss formulation"; [LB-card])
# ---------------------------------------------------------------------------
def load_balance_stats(expert_idx: np.ndarray, p: np.ndarray):
    """f_i = fraction of tokens whose argmax is i; P_i = mean router prob of i."""
    T, N = p.shape
    if T == 0:
        return np.zeros(N), np.zeros(N)
    counts = np.bincount(expert_idx, minlength=N).astype(np.float64)
    return counts / T, p.sum(axis=0) / T


def aux_loss(f: np.ndarray, P: np.ndarray) -> float:
    """N * sum_i f_i P_i (the alpha factor is left to the caller)."""
    f = np.asarray(f, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    return float(len(f) * np.sum(f * P))


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------
def switch_forward(x, W_r, W1, b1, W2, b2, capacity_factor: float, b_r=None,
                   activation: str = "relu", router_noise=None) -> Dict:
    """Full forward pass in float64 (``activation``: "relu" or "geglu";
    ``router_noise``: multiplicative noise [T, d] on the router input, or None).

    Returns out [T, d] (float64; zero rows for dropped tokens), expert_idx,
    gate, pos_in_expert, kept, capacity, f, P, aux, probs, logits."""
    xs = _f64(x)
    T = xs.shape[0]
    N = _f64(W_r).shape[0]
    ffn = _ffn_of(activation)
    xr = xs if router_noise is None else xs * _f64(router_noise)
    z = router_logits(xr, W_r, b_r)
    p = router_probs(z) if T else np.zeros((0, N))
    e, g = top1(p) if T else (np.zeros(0, np.int64), np.zeros(0))
    C = capacity(T, N, capacity_factor)
    pos = positions(e, N)
    kept = pos < C
    out = np.zeros((T, xs.shape[1]))
    for i in range(N):
        rows = np.nonzero((e == i) & kept)[0]
        if rows.size == 0:
            continue
        u = ffn(xs[rows], W1[i], b1[i], W2[i], b2[i])
        out[rows] = g[rows, None] * u
    f, P = load_balance_stats(e, p)
    aux = aux_loss(f, P) if T else 0.0
    return {"out": out, "expert_idx": e, "gate": g, "pos_in_expert": pos, "kept": kept,
            "capacity": C, "f": f, "P": P, "aux": aux, "probs": p, "logits": z}


def switch_forward_sampled(x, W_r, capacity_factor: float, sample_tokens,
                           expert_weights: Callable[[int], Dict], b_r=None,
                           chunk: int = 4096, activation: str = "relu") -> Dict:
    """Routing for every token, expert outputs only for ``sample_tokens``.

    ``expert_weights(e)`` returns {"W1","b1","W2","b2"} of expert e, so large
    layers never hold all expert weights at once.  The router runs over token
    chunks (rows are independent); positions need every token's choice."""
    xs = x
    T = xs.shape[0]
    N = W_r.shape[0]
    e_all = np.empty(T, dtype=np.int64)
    g_all = np.empty(T)
    psum = np.zeros(N)
    for s in range(0, T, chunk):
        z = router_logits(xs[s:s + chunk], W_r, b_r)
        p = router_probs(z)
        e, g = top1(p)
        e_all[s:s + chunk] = e
        g_all[s:s + chunk] = g
        psum += p.sum(axis=0)
    C = capacity(T, N, capacity_factor)
    pos = positions(e_all, N)
    kept = pos < C
    counts = np.bincount(e_all, minlength=N).astype(np.float64)
    f, P = counts / T, psum / T
    sample_tokens = np.asarray(sorted(set(int(t) for t in sample_tokens)), dtype=np.int64)
    out = {}
    by_expert: Dict[int, list] = {}
    for t in sample_tokens:
        if kept[t]:
            by_expert.setdefault(int(e_all[t]), []).append(int(t))
        else:
            out[int(t)] = np.zeros(xs.shape[1])
    for i, toks in sorted(by_expert.items()):
        w = expert_weights(i)
        u = _ffn_of(activation)(_f64(xs[toks]), w["W1"], w["b1"], w["W2"], w["b2"])
        for j, t in enumerate(toks):
            out[t] = g_all[t] * u[j]
    return {"out_rows": out, "expert_idx": e_all, "gate": g_all, "pos_in_expert": pos,
            "kept": kept, "capacity": C, "f": f, "P": P, "aux": aux_loss(f, P)}


# ---------------------------------------------------------------------------
# top-2 routing ([ST-note] "Comparison to Earlier MoE"; [MoE-note] top-2 example)
# ---------------------------------------------------------------------------
def capacity_k(T: int, N: int, capacity_factor: float, k: int) -> int:
    """Capacity of top-k routing, ceil(k * cf * T / N), exact on the double cf."""
    if N <= 0 or T < 0 or k < 1 or not math.isfinite(capacity_factor) or capacity_factor <= 0:
        raise ValueError("invalid capacity arguments")
    return math.ceil(Fraction(capacity_factor) * k * T / N)


def top2(p: np.ndarray, normalize: bool = True):
    """First choice e1 = argmax_i p_i and second choice e2 = argmax over i != e1
    (lowest index on ties for both); gates p_e1, p_e2, divided by their sum when
    ``normalize``.  Returns e [T, 2] and g [T, 2]."""
    T, N = p.shape
    if N < 2:
        raise ValueError("top-2 routing needs at least two experts")
    rows = np.arange(T)
    e1 = np.argmax(p, axis=1)
    rest = p.copy()
    rest[rows, e1] = -np.inf
    e2 = np.argmax(rest, axis=1)
    g = np.stack([p[rows, e1], p[rows, e2]], axis=1)
    if normalize:
        g = g / g.sum(axis=1, keepdims=True)
    return np.stack([e1, e2], axis=1).astype(np.int64), g


def positions_top2(e: np.ndarray, N: int) -> np.ndarray:
    """pos[t, k] = number of assignments to expert e[t, k] by tokens before t
    (token order; a token's two experts differ)."""
    seen = [0] * N
    pos = np.zeros(e.shape, dtype=np.int64)
    for t in range(e.shape[0]):
        for k in range(e.shape[1]):
            pos[t, k] = seen[int(e[t, k])]
        for k in range(e.shape[1]):
            seen[int(e[t, k])] += 1
    return pos


def switch_forward_top2(x, W_r, W1, b1, W2, b2, capacity_factor: float, b_r=None,
                        normalize: bool = True) -> Dict:
    """Top-2 layer in float64: out [T, d], expert_idx [T, 2], gate [T, 2],
    pos_in_expert [T, 2], kept [T, 2], capacity, f, P, aux."""
    xs = _f64(x)
    T = xs.shape[0]
    N = _f64(W_r).shape[0]
    z = router_logits(xs, W_r, b_r)
    p = router_probs(z) if T else np.zeros((0, N))
    e, g = top2(p, normalize) if T else (np.zeros((0, 2), np.int64), np.zeros((0, 2)))
    C = capacity_k(T, N, capacity_factor, 2)
    pos = positions_top2(e, N)
    kept = pos < C
    out = np.zeros((T, xs.shape[1]))
    for i in range(N):
        for k in range(2):
            rows = np.nonzero((e[:, k] == i) & kept[:, k])[0]
            if rows.size == 0:
                continue
            u = expert_ffn(xs[rows], W1[i], b1[i], W2[i], b2[i])
            out[rows] += g[rows, k, None] * u
    f, P = load_balance_stats(e[:, 0], p)
    aux = aux_loss(f, P) if T else 0.0
    return {"out": out, "expert_idx": e, "gate": g, "pos_in_expert": pos, "kept": kept,
            "capacity": C, "f": f, "P": P, "aux": aux, "probs": p, "logits": z}


def positions_ntlb(e: np.ndarray, N: int, C: int) -> np.ndarray:
    """No-Token-Left-Behind positions, two stages (readings in the module doc).
    e [T, 2] holds the first and second choices; returns pos [T, 2]: pos[t, 0]
    the stage-1 position at the first choice (its top-1 position), pos[t, 1]
    the stage-2 position at the second choice for a token stage 1 dropped
    (pos[t, 0] >= C), -1 for a token stage 1 kept."""
    T = e.shape[0]
    pos = np.full((T, 2), -1, dtype=np.int64)
    count = [0] * N
    for t in range(T):                      # stage 1: first choices, token order
        i = int(e[t, 0])
        pos[t, 0] = count[i]
        count[i] += 1
    filled = [min(c, C) for c in count]     # slots stage 1 took
    for t in range(T):                      # stage 2: overflow, token order
        if pos[t, 0] >= C:
            i = int(e[t, 1])
            pos[t, 1] = filled[i]
            filled[i] += 1
    return pos


def switch_forward_ntlb(x, W_r, W1, b1, W2, b2, capacity_factor: float,
                        b_r=None) -> Dict:
    """No-Token-Left-Behind layer in float64: out [T, d], expert_idx [T, 2]
    (first, second choice), gate [T, 2] (their router probabilities),
    pos_in_expert [T, 2] (``positions_ntlb``), assigned [T] (the expert that
    processes the token, -1 if dropped), capacity, f, P, aux."""
    xs = _f64(x)
    T = xs.shape[0]
    N = _f64(W_r).shape[0]
    z = router_logits(xs, W_r, b_r)
    p = router_probs(z) if T else np.zeros((0, N))
    e, g = top2(p, normalize=False) if T else (np.zeros((0, 2), np.int64), np.zeros((0, 2)))
    C = capacity(T, N, capacity_factor)
    pos = positions_ntlb(e, N, C)
    stage1 = pos[:, 0] < C
    stage2 = (~stage1) & (pos[:, 1] >= 0) & (pos[:, 1] < C)
    assigned = np.where(stage1, e[:, 0], np.where(stage2, e[:, 1], -1))
    gsel = np.where(stage1, g[:, 0], g[:, 1])
    out = np.zeros((T, xs.shape[1]))
    for i in range(N):
        rows = np.nonzero(assigned == i)[0]
        if rows.size == 0:
            continue
        u = expert_ffn(xs[rows], W1[i], b1[i], W2[i], b2[i])
        out[rows] = gsel[rows, None] * u
    f, P = load_balance_stats(e[:, 0], p)
    aux = aux_loss(f, P) if T else 0.0
    return {"out": out, "expert_idx": e, "gate": g, "pos_in_expert": pos, "assigned": assigned,
            "capacity": C, "f": f, "P": P, "aux": aux, "probs": p, "logits": z}


# ---------------------------------------------------------------------------
# backward ([ST-explained] gate gradient; [ST-paper] "The loss formulation")
# ---------------------------------------------------------------------------
def switch_backward(x, W_r, W1, b1, W2, b2, capacity_factor: float, dout, daux: float = 0.0,
                    b_r=None) -> Dict:
    """Gradients of L = sum(dout * out) + daux * aux for the top-1 ReLU layer:
    dx [T, d], dW_r [N, d], db_r [N], dW1, db1, dW2, db2 (the shapes of the
    weights), all float64."""
    xs = _f64(x)
    T, d = xs.shape
    Wr = _f64(W_r)
    N = Wr.shape[0]
    fw = switch_forward(xs, W_r, W1, b1, W2, b2, capacity_factor, b_r=b_r)
    p, e, g, kept, f = fw["probs"], fw["expert_idx"], fw["gate"], fw["kept"], fw["f"]
    dy = _f64(dout)
    W1s, b1s, W2s, b2s = _f64(W1), _f64(b1), _f64(W2), _f64(b2)
    dx = np.zeros((T, d))
    dW1, db1 = np.zeros_like(W1s), np.zeros_like(b1s)
    dW2, db2 = np.zeros_like(W2s), np.zeros_like(b2s)
    dg = np.zeros(T)
    for i in range(N):
        rows = np.nonzero((e == i) & kept)[0]
        if rows.size == 0:
            continue
        a = xs[rows] @ W1s[i].T + b1s[i][None, :]
        h = np.maximum(a, 0.0)
        u = h @ W2s[i].T + b2s[i][None, :]
        dg[rows] = np.sum(dy[rows] * u, axis=1)
        du = g[rows, None] * dy[rows]
        dW2[i] = du.T @ h
        db2[i] = du.sum(axis=0)
        da = (du @ W2s[i]) * (a > 0)
        dW1[i] = da.T @ xs[rows]
        db1[i] = da.sum(axis=0)
        dx[rows] += da @ W1s[i]
    dz = np.zeros((T, N))
    if T:
        onehot = np.zeros((T, N))
        onehot[np.arange(T), e] = 1.0
        dz += (dg * g)[:, None] * (onehot - p)                 # zero for dropped tokens
        dz += daux * (N / T) * p * (f[None, :] - (p @ f)[:, None])
    dW_r = dz.T @ xs
    db_r = dz.sum(axis=0)
    dx += dz @ Wr
    return {"dx": dx, "dW_r": dW_r, "db_r": db_r, "dW1": dW1, "db1": db1, "dW2": dW2,
            "db2": db2, "dgate": dg, "dlogits": dz}
