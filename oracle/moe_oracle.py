"""Float64 CPU oracle of the top-k mixture-of-experts FFN forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
links this module: only the tests, the smoke check of the package entry file
and the CPU-baseline leg of the benchmark script may use it.  It shares no
code with the CUDA library (no kernels, headers, tables or helpers) and
imports nothing from the product package.

It is written to be read against the pages, not to be fast:

* every expert is evaluated on every token and the selected outputs are then
  gathered, exactly as the Flax exercise "Mixture-of-Experts FFN"
  (crackedaicode.com) does in "Compute the experts and router" and
  "Weight the selected outputs";
* the gated expert is down_proj(silu(gate) * up) with the Hugging Face
  layout of mojolearn.MoEBlock (class description and "Variables":
  router (E, D), gate_up_proj (E, 2F, D), down_proj (E, D, F));
* all arithmetic is float64 on the given (already rounded) operands, the
  check the Dew "Mixture of experts" page describes under "Expert
  computation and placement" (float64 arithmetic on the rounded operands).

Readings where the pages leave a step open (each is listed in the design doc):

* gate_up_proj rows [0, F) are the gate projection and rows [F, 2F) the up
  projection (the plain concatenation order of the name);
* the renormalisation adds 1e-9 to the denominator whenever
  norm_topk_prob is set, for both expert kinds (the exercise's formula);
  with norm_topk_prob unset the kept softmax probabilities are used as is;
* the Dense/ReLU expert is passed in the same orientation as the gated one:
  W1 (E, F, D) in the gate_up slot, W2 (E, D, F) in the down slot, b1 (E, F),
  b2 (E, D); b2 belongs to each expert's output and so is weighted with it;
* equal probabilities go to the lower expert index, and the kept experts
  are listed in descending probability (jax.lax.top_k's order, which the
  exercise states).

Parity status: every function here is pinned by the CPU tests in
``tests/test_oracle_pins.py`` (worked example, closed forms, invariants,
brute force, library special cases).  The pages' own seeded outputs (Flax
PRNG, mojolearn's generator) cannot be reproduced and are not claimed.
"""
from __future__ import annotations

import numpy as np

ACT_SILU_GATED = "silu_gated"
ACT_RELU = "relu"
RENORM_EPS = 1e-9


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def check_top_k(K: int, E: int) -> None:
    """1 <= top_k <= num_experts, else ValueError (mojolearn.MoEBlock,
    parameter top_k; the exercise's "Problem" states the same range)."""
    if not (1 <= int(K) <= int(E)):
        raise ValueError(f"top_k={K} outside [1, {E}]")


def check_act(act: str) -> None:
    """Only the SiLU-gated expert (mojolearn.MoEBlock, hidden_act: anything
    else raises NotImplementedError) and the exercise's Dense/ReLU expert."""
    if act not in (ACT_SILU_GATED, ACT_RELU):
        raise NotImplementedError(f"activation {act!r}")


# ------------------------------------------------------------------ router
def router_logits(x, router, router_bias=None):
    """logits[t, e] = sum_d x[t, d] * router[e, d] (+ router_bias[e]).

    The exercise's Dense(E) router keeps its bias ("Problem", keep all Dense
    defaults); mojolearn's router (E, D) has none."""
    lg = _f64(x) @ _f64(router).T
    if router_bias is not None:
        lg = lg + _f64(router_bias)[None, :]
    return lg


def softmax(logits):
    """Softmax over the expert axis ("Compute the experts and router"),
    shifted by the row maximum, which leaves the value unchanged."""
    lg = _f64(logits)
    z = np.exp(lg - lg.max(axis=-1, keepdims=True))
    return z / z.sum(axis=-1, keepdims=True)


def top_k(probs, K: int):
    """The K largest probabilities per token in descending order; equal
    scores favour the lower expert index ("Compute the experts and router";
    mojolearn: "Routing ties go to the lower expert index").

    A stable sort of -p keeps equal entries in ascending index order."""
    p = _f64(probs)
    check_top_k(K, p.shape[-1])
    order = np.argsort(-p, axis=-1, kind="stable")[..., :K]
    vals = np.take_along_axis(p, order, axis=-1)
    return vals, order.astype(np.int64)


def routing_weights(vals, norm_topk_prob: bool = True):
    """weights = selected / (sum(selected) + 1e-9) ("Weight the selected
    outputs"); with norm_topk_prob unset (mojolearn parameter) the kept
    probabilities are returned unchanged."""
    v = _f64(vals)
    if not norm_topk_prob:
        return v.copy()
    return v / (v.sum(axis=-1, keepdims=True) + RENORM_EPS)


def topk_gap(probs, K: int):
    """p_(K) - p_(K+1) per token: how far the K-th kept probability is above
    the best dropped one (+inf when K == E).  Selections whose gap is tiny
    are not unique up to rounding."""
    p = np.sort(_f64(probs), axis=-1)[..., ::-1]
    if K >= p.shape[-1]:
        return np.full(p.shape[:-1], np.inf)
    return p[..., K - 1] - p[..., K]


# ----------------------------------------------------------------- experts
def silu(z):
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z))."""
    z = _f64(z)
    return z / (1.0 + np.exp(-z))


def expert_silu_gated(x, gate_up_e, down_e):
    """One Mixtral-style expert: down_proj(silu(gate) * up)
    (mojolearn.MoEBlock), with gate = x @ gate_up_e[:F].T and
    up = x @ gate_up_e[F:].T, each weight row a D-vector (HF layout)."""
    gu = _f64(gate_up_e)
    F = gu.shape[0] // 2
    xx = _f64(x)
    gate = xx @ gu[:F].T
    up = xx @ gu[F:].T
    h = silu(gate) * up
    return h @ _f64(down_e).T


def expert_relu(x, w1_e, b1_e, w2_e, b2_e):
    """One exercise expert: Dense(F) -> ReLU -> Dense(D), both with biases
    ("Compute the experts and router"); weights given as W1 (F, D) and
    W2 (D, F)."""
    h = _f64(x) @ _f64(w1_e).T + _f64(b1_e)[None, :]
    h = np.maximum(h, 0.0)
    return h @ _f64(w2_e).T + _f64(b2_e)[None, :]


def expert_outputs(x, gate_up_proj, down_proj, act=ACT_SILU_GATED, b1=None, b2=None):
    """Every expert on every token, stacked on axis 1: (T, E, D) ("Compute
    the experts and router": expert_outs holds T*E*D values).  Weights are
    widened to float64 one expert at a time."""
    check_act(act)
    xx = _f64(x)
    E = gate_up_proj.shape[0]
    T, D = xx.shape
    outs = np.empty((T, E, D), dtype=np.float64)
    for e in range(E):
        if act == ACT_SILU_GATED:
            outs[:, e, :] = expert_silu_gated(xx, gate_up_proj[e], down_proj[e])
        else:
            outs[:, e, :] = expert_relu(xx, gate_up_proj[e], b1[e], down_proj[e], b2[e])
    return outs


def combine(expert_outs, idx, weights):
    """out[t] = sum_k weights[t, k] * expert_outs[t, idx[t, k]], gathering on
    the expert axis per token ("Weight the selected outputs"; each token
    selects only its own outputs)."""
    eo = _f64(expert_outs)
    chosen = np.take_along_axis(eo, np.asarray(idx, dtype=np.int64)[:, :, None], axis=1)
    return (chosen * _f64(weights)[:, :, None]).sum(axis=1)


# ------------------------------------------------------------------- layer
def moe_route(x, router, K: int, norm_topk_prob: bool = True, router_bias=None):
    """Router half of the layer: logits, softmax, top-k, weights."""
    lg = router_logits(x, router, router_bias)
    check_top_k(K, lg.shape[-1])
    p = softmax(lg)
    vals, idx = top_k(p, K)
    w = routing_weights(vals, norm_topk_prob)
    return {"router_logits": lg, "probs": p, "selected_experts": idx,
            "routing_weights": w, "gap": topk_gap(p, K)}


def moe_ffn_forward(x, router, gate_up_proj, down_proj, K: int,
                    norm_topk_prob: bool = True, act: str = ACT_SILU_GATED,
                    router_bias=None, b1=None, b2=None):
    """The whole forward, dense over experts then gathered.

    x may have any leading shape (..., D) (mojolearn forward); tokens are the
    flattened leading dims and the output has the shape of x."""
    check_act(act)
    xx = _f64(x)
    shape = xx.shape
    xx = xx.reshape(-1, shape[-1])
    r = moe_route(xx, router, K, norm_topk_prob, router_bias)
    eo = expert_outputs(xx, gate_up_proj, down_proj, act, b1, b2)
    out = combine(eo, r["selected_experts"], r["routing_weights"])
    r["out"] = out.reshape(shape)
    return r


def moe_ffn_given_routing(x, idx, weights, gate_up_proj, down_proj,
                          act: str = ACT_SILU_GATED, b1=None, b2=None):
    """The expert half for a given selection: dense expert outputs gathered
    with ``idx`` and weighted by ``weights``.  Used where several selections
    are correct (probabilities equal up to rounding)."""
    xx = _f64(x).reshape(-1, np.shape(x)[-1])
    eo = expert_outputs(xx, gate_up_proj, down_proj, act, b1, b2)
    return combine(eo, idx, weights)


def parameter_count(E: int, D: int, F: int, act: str = ACT_RELU) -> int:
    """Trainable parameters of the layer.  Dense/ReLU: each expert has
    2*D*F + F + D, the biased router D*E + E ("Selection does not imply
    sparse computation").  Gated (no biases): 3*D*F per expert + D*E."""
    if act == ACT_RELU:
        return E * (2 * D * F + F + D) + D * E + E
    return E * 3 * D * F + D * E
