"""Seeded synthetic inputs for one Switch layer (forward pass).

This module only *draws numbers*; it holds none of the layer's arithmetic.
Both the CUDA path (tests, bench, smoke) and the fp64 oracle take their inputs
from here, so the two sides always see identical tensors.

Generator
---------
Every tensor slice has a key (seed, workload name, tensor name, expert, attempt).
Element ``i`` of the slice takes the value ``table[h(key, i) >> 12]``, where ``h``
is a 32-bit counter-based integer hash (two rounds of the "hash prospector"
two-multiply mixer, constants 0x21f0aaad / 0x735a2d97, shifts 16/15/15) and
``table`` holds the 2**20 mid-point quantiles of the target distribution:

* ``normal``  : standard normal, quantiles at (k+1/2)/2**20 (|v| <= 4.9).
* ``trunc2``  : normal truncated to two standard deviations, which is what
  "resample every value more than two standard deviations from the mean"
  produces (T5 initialisation with scale s=0.1, sigma = sqrt(s / fan_in);
  Switch Transformer, explained, recipe step 6; paper-graph summary of
  arXiv 2101.03961, section 3.4, initialisation paragraph).  Drawing from
  the inverse CDF of the truncated law gives the same distribution as
  rejection, quantised to 2**-20 in probability.

The tables are computed once in fp64 (``scipy.special.ndtri``), scaled by sigma
in fp64, rounded to fp32 (and to bf16 for bf16 tensors) on the CPU, and the
device only gathers from them.  All per-element work is exact int64 arithmetic
(products stay below 2**63), so CPU and CUDA produce bit-identical tensors and
any slice (one expert's weights, one token row) can be regenerated alone.

Router-logit gap filter
-----------------------
To make the argmax decision unique, token rows whose top-1 / top-2 router-logit
gap is below 1e-3 are redrawn from the follow-on key ``("x_redraw", t, attempt)``.
Which rows to redraw is *not* decided here (that needs the router's
arithmetic); callers pass a ``{row: attempt}`` map, stored for the named
workloads in ``tests/golden/gap_redraws.json`` by a script that uses the oracle.
"""
from __future__ import annotations

import functools
import hashlib
import json
import math
import os
from dataclasses import dataclass, asdict
from typing import Dict, Optional

import numpy as np
import torch

__all__ = [
    "LayerSpec", "WORKLOADS", "make_layer_inputs", "expert_slice", "draw",
    "load_gap_redraws", "TABLE_BITS", "router_noise",
]

TABLE_BITS = 20
_M32 = 0xFFFFFFFF


@dataclass(frozen=True)
class LayerSpec:
    """Shape and input recipe of one Switch-layer forward call."""
    name: str
    T: int            # tokens (batch x sequence, flattened b*S + s)
    d: int            # model width
    d_ff: int         # expert FFN width
    N: int            # experts
    cf: float         # capacity factor
    dtype: str        # "f32" or "bf16": dtype of x, W1, b1, W2, b2, out
    bias_std: float = 0.0       # std of b1 / b2 (0 -> zero biases)
    router_bias: Optional[str] = None  # None or "zipf<a>": b_r[i] = a*ln(1/(i+1))
    activation: str = "relu"    # "relu" or "geglu" (W1 [N, 2 d_ff, d]: gate rows, value rows)

    def to_json(self) -> dict:
        return asdict(self)


# The five synthetic workloads.  Sizes and distributions as stated for each:
# x ~ N(0,1); W_r, W1, W2 ~ truncated normal, std sqrt(0.1/fan_in);
# biases N(0, 0.01) for the tiny fp32 layer and zero elsewhere.
WORKLOADS: Dict[str, LayerSpec] = {s.name: s for s in [
    LayerSpec("tiny_f32_T64_d32_N4", 64, 32, 64, 4, 1.0, "f32", bias_std=0.01),
    LayerSpec("base_T4096_d768_N64", 4096, 768, 3072, 64, 1.25, "bf16"),
    LayerSpec("large_T16384_d1024_N128", 16384, 1024, 4096, 128, 1.0, "bf16"),
    LayerSpec("skewed_T32768_d2048_N64", 32768, 2048, 5120, 64, 2.0, "bf16",
              router_bias="zipf1.5"),
    LayerSpec("many_T65536_d1024_N2048", 65536, 1024, 2048, 2048, 1.0, "bf16"),
]}


# ----------------------------------------------------------------------------
# counter-based hash
# ----------------------------------------------------------------------------
def _mix32(x: torch.Tensor) -> torch.Tensor:
    """One round of a 32-bit integer mixer on int64 tensors holding [0, 2**32)."""
    x = x ^ (x >> 16)
    x = (x * 0x21F0AAAD) & _M32
    x = x ^ (x >> 15)
    x = (x * 0x735A2D97) & _M32
    x = x ^ (x >> 15)
    return x


def _key_words(key: tuple) -> tuple:
    """Two 32-bit words derived from a key tuple (stable across machines)."""
    h = hashlib.blake2b(repr(key).encode(), digest_size=8).digest()
    return int.from_bytes(h[:4], "little"), int.from_bytes(h[4:], "little")


def _bucket(idx: torch.Tensor, k1, k2) -> torch.Tensor:
    """Table bucket in [0, 2**TABLE_BITS) for element indices ``idx``.

    ``k1``/``k2`` are ints or int64 tensors broadcastable against ``idx``."""
    h = _mix32((idx + k1) & _M32)
    h = _mix32(h ^ k2)
    return h >> (32 - TABLE_BITS)


# ----------------------------------------------------------------------------
# quantile tables
# ----------------------------------------------------------------------------
@functools.lru_cache(maxsize=None)
def _std_quantiles(kind: str) -> np.ndarray:
    from scipy.special import ndtr, ndtri
    u = (np.arange(1 << TABLE_BITS, dtype=np.float64) + 0.5) / float(1 << TABLE_BITS)
    if kind == "normal":
        return ndtri(u)
    if kind == "trunc2":
        lo, hi = ndtr(-2.0), ndtr(2.0)
        return ndtri(lo + u * (hi - lo))
    if kind == "uniform":          # U(-1, 1)
        return 2.0 * u - 1.0
    raise ValueError(kind)


@functools.lru_cache(maxsize=None)
def _table_cpu(kind: str, sigma: float, dtype: str) -> torch.Tensor:
    q = _std_quantiles(kind) * sigma                 # fp64
    t = torch.from_numpy(q.astype(np.float32))       # round to fp32
    if dtype == "bf16":
        t = t.to(torch.bfloat16)                     # round-to-nearest-even
    return t


_TABLE_DEV: dict = {}


def _table(kind: str, sigma: float, dtype: str, device) -> torch.Tensor:
    t = _table_cpu(kind, float(sigma), dtype)
    dev = torch.device(device)
    if dev.type == "cpu":
        return t
    k = (kind, float(sigma), dtype, str(dev))
    if k not in _TABLE_DEV:
        _TABLE_DEV[k] = t.to(dev)
    return _TABLE_DEV[k]


def _torch_dtype(dtype: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def draw(key: tuple, shape, kind: str, sigma: float, dtype: str,
         device="cpu") -> torch.Tensor:
    """Draw a tensor of ``shape`` for ``key`` (row-major element order)."""
    numel = int(np.prod(shape)) if len(shape) else 1
    if numel >= (1 << 32):
        raise ValueError("slice too large for a 32-bit counter")
    k1, k2 = _key_words(key)
    idx = torch.arange(numel, dtype=torch.int64, device=device)
    vals = _table(kind, sigma, dtype, device)[_bucket(idx, k1, k2)]
    return vals.reshape(shape)


def _draw_experts(base_key: tuple, experts, inner_shape, kind, sigma, dtype,
                  device, chunk_elems: int) -> torch.Tensor:
    """Stack per-expert slices ``base_key + (e,)`` for e in ``experts``."""
    experts = list(experts)
    numel = int(np.prod(inner_shape))
    out = torch.empty((len(experts),) + tuple(inner_shape), dtype=_torch_dtype(dtype),
                      device=device)
    if not experts:
        return out
    table = _table(kind, sigma, dtype, device)
    idx = torch.arange(numel, dtype=torch.int64, device=device)
    per = max(1, chunk_elems // max(numel, 1))
    flat = out.view(len(experts), numel)
    for s in range(0, len(experts), per):
        es = experts[s:s + per]
        kw = [_key_words(base_key + (e,)) for e in es]
        k1 = torch.tensor([a for a, _ in kw], dtype=torch.int64, device=device)[:, None]
        k2 = torch.tensor([b for _, b in kw], dtype=torch.int64, device=device)[:, None]
        flat[s:s + len(es)] = table[_bucket(idx[None, :], k1, k2)]
    return out


def _sigmas(spec: LayerSpec) -> dict:
    return {
        "W_r": math.sqrt(0.1 / spec.d),
        "W1": math.sqrt(0.1 / spec.d),      # fan-in d
        "W2": math.sqrt(0.1 / spec.d_ff),   # fan-in d_ff
    }


def router_bias_values(spec: LayerSpec) -> Optional[torch.Tensor]:
    """Router-logit bias b_r[i] = a * ln(1/(i+1)) for router_bias "zipf<a>" (the
    skewed workload uses a = 1.5), fp32."""
    if spec.router_bias is None:
        return None
    if spec.router_bias.startswith("zipf"):
        a = float(spec.router_bias[4:])
        v = np.array([a * math.log(1.0 / (i + 1)) for i in range(spec.N)], dtype=np.float64)
        return torch.from_numpy(v.astype(np.float32))
    raise ValueError(spec.router_bias)


def _chunk_elems(device) -> int:
    return (1 << 26) if torch.device(device).type == "cuda" else (1 << 22)


def expert_slice(spec: LayerSpec, experts, seed: int = 0, device="cpu") -> dict:
    """W1[e] [d_ff,d], b1[e] [d_ff], W2[e] [d,d_ff], b2[e] [d] for the listed experts."""
    sg = _sigmas(spec)
    ce = _chunk_elems(device)
    base = (seed, spec.name)
    h = 2 * spec.d_ff if spec.activation == "geglu" else spec.d_ff   # GEGLU: gate and value rows
    out = {
        "W1": _draw_experts(base + ("W1",), experts, (h, spec.d), "trunc2",
                            sg["W1"], spec.dtype, device, ce),
        "W2": _draw_experts(base + ("W2",), experts, (spec.d, spec.d_ff), "trunc2",
                            sg["W2"], spec.dtype, device, ce),
    }
    if spec.bias_std > 0:
        out["b1"] = _draw_experts(base + ("b1",), experts, (h,), "normal",
                                  spec.bias_std, spec.dtype, device, ce)
        out["b2"] = _draw_experts(base + ("b2",), experts, (spec.d,), "normal",
                                  spec.bias_std, spec.dtype, device, ce)
    else:
        out["b1"] = torch.zeros((len(list(experts)), h), dtype=_torch_dtype(spec.dtype),
                                device=device)
        out["b2"] = torch.zeros((len(list(experts)), spec.d), dtype=_torch_dtype(spec.dtype),
                                device=device)
    return out


def router_noise(spec: LayerSpec, eps: float = 1e-2, seed: int = 0, device="cpu") -> torch.Tensor:
    """Multiplicative router-input noise [T, d] fp32, uniform on [1 - eps, 1 + eps]
    (the input jitter of the router exploration experiments; off at inference)."""
    u = draw((seed, spec.name, "router_noise"), (spec.T, spec.d), "uniform", eps, "f32", device)
    return 1.0 + u


def make_x(spec: LayerSpec, seed: int = 0, device="cpu",
           redraws: Optional[Dict[int, int]] = None) -> torch.Tensor:
    """Token activations x [T, d] ~ N(0,1), with the given rows redrawn."""
    x = draw((seed, spec.name, "x"), (spec.T, spec.d), "normal", 1.0, spec.dtype, device)
    for t, attempt in sorted((redraws or {}).items()):
        x[int(t)] = draw((seed, spec.name, "x_redraw", int(t), int(attempt)), (spec.d,),
                         "normal", 1.0, spec.dtype, device)
    return x


def make_router(spec: LayerSpec, seed: int = 0, device="cpu") -> dict:
    """Router weight W_r [N, d] (fp32) and optional router bias b_r [N] (fp32)."""
    W_r = draw((seed, spec.name, "W_r"), (spec.N, spec.d), "trunc2", _sigmas(spec)["W_r"],
               "f32", device)
    b_r = router_bias_values(spec)
    return {"W_r": W_r, "b_r": None if b_r is None else b_r.to(device)}


def make_layer_inputs(spec: LayerSpec, seed: int = 0, device="cpu",
                      redraws: Optional[Dict[int, int]] = None,
                      with_experts: bool = True) -> dict:
    """All inputs of one forward call, resident on ``device``.

    Layouts (row-major): x [T,d]; W_r [N,d]; b_r [N] or None; W1 [N,d_ff,d];
    b1 [N,d_ff]; W2 [N,d,d_ff]; b2 [N,d]."""
    out = {"x": make_x(spec, seed, device, redraws)}
    out.update(make_router(spec, seed, device))
    if with_experts:
        out.update(expert_slice(spec, range(spec.N), seed, device))
    return out


def random_spec(rng: np.random.Generator, name: str, dtype: str = "bf16", max_T: int = 700,
                max_N: int = 9) -> LayerSpec:
    """A small random layer shape for parity sweeps (bf16 needs d, d_ff % 8 == 0)."""
    mult = 8 if dtype == "bf16" else 1
    T = int(rng.integers(1, max_T + 1))
    d = int(rng.integers(1, 40)) * mult
    d_ff = int(rng.integers(1, 48)) * mult
    N = int(rng.integers(1, max_N + 1))
    cf = float(rng.choice([0.25, 0.5, 1.0, 1.25, 2.0, 4.0]))
    return LayerSpec(name, T, d, d_ff, N, cf, dtype, bias_std=0.05)


_GAP_FILE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                         "tests", "golden", "gap_redraws.json")


def load_gap_redraws(name: str, seed: int = 0) -> Dict[int, int]:
    """Stored ``{row: attempt}`` redraw map of a named workload ({} if absent)."""
    if not os.path.exists(_GAP_FILE):
        return {}
    with open(_GAP_FILE) as f:
        data = json.load(f)
    ent = data.get("workloads", {}).get(name)
    if ent is None or int(ent.get("seed", 0)) != seed:
        return {}
    return {int(k): int(v) for k, v in ent["rows"].items()}
