"""Float64 CPU oracle of the top-k mixture-of-experts FFN forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
links this module: only the tests, the smoke check of the package entry file
and the CPU-baseline leg of the benchmark script may use it.  It shares no
code with the CUDA library (no kernels, headers, tables or helpers) and
imports nothing from the product package.

It is written to be read against the sources it cites, not to be fast:

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

Readings taken where those sources leave a step open:

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

Routing extensions ("Mixture of experts", dewml.dev, "Router behavior" and
"Expert computation and placement"; ES-MoE API page, "ESMoE" settings and
"Balancing objectives"), with these readings:

* sigmoid scores: each expert's score is sigmoid(logit) on its own;
* a selection bias is added to the scores only to choose the experts; the
  weights come from the unbiased scores;
* dynamic_threshold: a kept expert whose renormalised share is below the
  threshold is dropped, except the first (the leader), and the kept shares
  are renormalised to sum to one;
* capacity_factor: each sequence of L tokens keeps
  floor(max(ceil(L*K/E)*cf, cf)) slots per expert, the first ones in token
  order; a dropped slot contributes nothing and nothing is renormalised;
* balancing statistics of a batch from the scores and the gate, the gate
  being each token's top-k selection renormalised to sum to one.

Parity status: every function here is pinned by the CPU tests in
``tests/test_oracle_pins.py`` (worked example, closed forms, invariants,
brute force, library special cases) and ``tests/test_oracle_ext_pins.py``
(the routing extensions: hand-worked cases, independent formulations,
planted mutants).  The sources' own seeded outputs (Flax
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


# ------------------------------------------------------ routing extensions
SCORE_SOFTMAX = "softmax"
SCORE_SIGMOID = "sigmoid"


def sigmoid(z):
    """sigmoid(z) = 1 / (1 + exp(-z)), one expert at a time ("Mixture of
    experts", dewml.dev, "Router behavior": softmax or sigmoid scores)."""
    return 1.0 / (1.0 + np.exp(-_f64(z)))


def router_scores(logits, score: str = SCORE_SOFTMAX):
    if score == SCORE_SOFTMAX:
        return softmax(logits)
    if score == SCORE_SIGMOID:
        return sigmoid(logits)
    raise NotImplementedError(f"score {score!r}")


def select_experts(scores, K: int, selection_bias=None):
    """Top-K experts by score (+ selection bias), descending, equal values to
    the lower index.  Returns the chosen indices and their UNBIASED scores
    (the bias only decides which experts are picked: "Router behavior")."""
    sc = _f64(scores)
    rank_by = sc if selection_bias is None else sc + _f64(selection_bias)[None, :]
    _, idx = top_k(rank_by, K)
    return np.take_along_axis(sc, idx, axis=-1), idx


def apply_dynamic_threshold(weights, threshold: float):
    """ES-MoE's dynamic_threshold (API page, "ESMoE" settings): a routed
    expert whose share of the mixture (its weight after the top-k
    renormalisation) is below the threshold is dropped, the leader (first
    slot) always stays, and the kept shares are renormalised.  Returns
    (new weights with zeros at dropped slots, kept mask)."""
    w = _f64(weights)
    share = w / w.sum(axis=-1, keepdims=True)
    keep = share >= threshold
    keep[:, 0] = True
    kept = np.where(keep, share, 0.0)
    return kept / kept.sum(axis=-1, keepdims=True), keep


def capacity_slots(length: int, K: int, E: int, capacity_factor: float) -> int:
    """Slots per expert for one sequence: floor(max(ceil(L*K/E)*cf, cf))
    ("Expert computation and placement", capacity_factor)."""
    c = max(int(np.ceil(length * K / E)) * float(capacity_factor), float(capacity_factor))
    return int(np.floor(c))


def capacity_keep(idx, E: int, capacity_factor: float, seq_len: int = 0, active=None):
    """Which (token, slot) pairs keep their expert under the capacity: per
    sequence of seq_len tokens (0: the whole batch is one sequence) and per
    expert, the first capacity_slots(...) pairs in token order.  Slots
    already inactive (``active`` False) take no capacity."""
    idx = np.asarray(idx)
    T, K = idx.shape
    L = T if not seq_len else int(seq_len)
    keep = np.zeros((T, K), dtype=bool)
    act = np.ones((T, K), dtype=bool) if active is None else np.asarray(active, dtype=bool)
    for s0 in range(0, T, L):
        s1 = min(T, s0 + L)
        cap = capacity_slots(s1 - s0, K, E, capacity_factor)
        used = np.zeros(E, dtype=np.int64)
        for t in range(s0, s1):
            for k in range(K):
                if not act[t, k]:
                    continue
                e = idx[t, k]
                if used[e] < cap:
                    keep[t, k] = True
                    used[e] += 1
    return keep


def balance_stats(scores, idx, weights):
    """The four balancing objectives of ES-MoE's API page ("Balancing
    objectives") on one batch.  probs = the router's scores (T, E); gate =
    the top-k selection renormalised (the page's definition), i.e. each
    token's kept routing weights divided by their sum and scattered to
    (T, E).  The gate is renormalised whether or not norm_topk_prob was set
    for the output weights; slots with weight 0 (dropped by the threshold)
    stay 0.
      switch       = E * sum_i mean(probs)_i * mean(gate > 0)_i
      gshard       = E * sum_i u_i^2, u = mean(gate) normalised to sum to one
      master       = (1/E) * sum_i (u_i - 1/E)^2
      gshard_probs = E * sum_i v_i^2, v = mean(probs) normalised"""
    p = _f64(scores)
    T, E = p.shape
    w = _f64(weights)
    tot = w.sum(axis=-1, keepdims=True)
    w_renorm = np.divide(w, tot, out=np.zeros_like(w), where=tot > 0)
    gate = np.zeros((T, E))
    np.put_along_axis(gate, np.asarray(idx, dtype=np.int64), w_renorm, axis=1)
    mp = p.mean(axis=0)
    mg = gate.mean(axis=0)
    frac = (gate > 0).mean(axis=0)
    u = mg / mg.sum()
    v = mp / mp.sum()
    return {"switch": E * float((mp * frac).sum()),
            "gshard": E * float((u * u).sum()),
            "master": float(((u - 1.0 / E) ** 2).sum() / E),
            "gshard_probs": E * float((v * v).sum())}


def moe_route_ext(x, router, K: int, norm_topk_prob: bool = True, router_bias=None,
                  score: str = SCORE_SOFTMAX, selection_bias=None, dynamic_threshold: float = 0.0):
    """Router with the extensions: scores, biased choice, weights, optional
    dynamic threshold.  ``active`` marks slots still routed after the
    threshold."""
    lg = router_logits(x, router, router_bias)
    check_top_k(K, lg.shape[-1])
    sc = router_scores(lg, score)
    vals, idx = select_experts(sc, K, selection_bias)
    w = routing_weights(vals, norm_topk_prob)
    active = np.ones(idx.shape, dtype=bool)
    if dynamic_threshold and dynamic_threshold > 0:
        w, active = apply_dynamic_threshold(routing_weights(vals, True), dynamic_threshold)
    rank_by = sc if selection_bias is None else sc + _f64(selection_bias)[None, :]
    return {"router_logits": lg, "probs": sc, "selected_experts": idx, "routing_weights": w,
            "active": active, "gap": topk_gap(rank_by, K)}


def moe_ffn_forward_ext(x, router, gate_up_proj, down_proj, K: int, norm_topk_prob: bool = True,
                        act: str = ACT_SILU_GATED, router_bias=None, b1=None, b2=None,
                        score: str = SCORE_SOFTMAX, selection_bias=None,
                        dynamic_threshold: float = 0.0, capacity_factor: float = 0.0,
                        seq_len: int = 0):
    """The forward with the routing extensions: slots dropped by the
    threshold or the capacity contribute nothing."""
    check_act(act)
    xx = _f64(x)
    shape = xx.shape
    xx = xx.reshape(-1, shape[-1])
    r = moe_route_ext(xx, router, K, norm_topk_prob, router_bias, score, selection_bias,
                      dynamic_threshold)
    keep = r["active"].copy()
    if capacity_factor and capacity_factor > 0:
        keep &= capacity_keep(r["selected_experts"], router.shape[0], capacity_factor, seq_len,
                              r["active"])
    eo = expert_outputs(xx, gate_up_proj, down_proj, act, b1, b2)
    out = combine(eo, r["selected_experts"], np.where(keep, r["routing_weights"], 0.0))
    r["kept"] = keep
    r["out"] = out.reshape(shape)
    r["balance"] = balance_stats(r["probs"], r["selected_experts"], r["routing_weights"])
    return r


def parameter_count(E: int, D: int, F: int, act: str = ACT_RELU) -> int:
    """Trainable parameters of the layer.  Dense/ReLU: each expert has
    2*D*F + F + D, the biased router D*E + E ("Selection does not imply
    sparse computation").  Gated (no biases): 3*D*F per expert + D*E."""
    if act == ACT_RELU:
        return E * (2 * D * F + F + D) + D * E + E
    return E * 3 * D * F + D * E
