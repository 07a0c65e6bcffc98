"""Pins of the float64 oracle to facts outside itself (CPU only).

Each test ties one part of the oracle to something the cited sources or
the mathematics fix: the exercise's worked example, the parameter-count closed
form, invariants of the weights, lower-index tie-breaking, token
permutation equivariance, brute force on tiny inputs, and special cases that
reduce to library routines (torch float64 linear algebra, the installed
transformers Mixtral experts).  ``test_mutants_are_caught`` plants plausible
mistakes in a copy of the oracle and checks that a pin fails for each.
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle
from oracle import moe_oracle as O
from mixture_experts_ffn_09_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(seed, T, D, F, E, act=O.ACT_SILU_GATED, std=0.3):
    d = synth.random_case(seed, T, D, F, E, act=act, weight_std=std)
    return d


# ----------------------------------------------------------- worked example
def test_worked_example_two_tokens():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_two_tokens.json")))
    probs = np.array(g["probs"])
    eo = np.array(g["expert_outs"])
    vals, idx = O.top_k(probs, g["top_k"])
    assert idx.tolist() == g["expected_indices"]
    w = O.routing_weights(vals, True)
    chosen = np.take_along_axis(eo, idx[:, :, None], axis=1)
    assert list(chosen.shape) == g["expected_chosen_shape"]
    out = O.combine(eo, idx, w)
    np.testing.assert_allclose(out, np.array(g["expected_out"]), atol=g["atol"], rtol=0)
    # the unselected expert output does not enter the sum
    eo2 = eo.copy()
    eo2[0, 2] = 1e6
    eo2[1, 1] = -1e6
    np.testing.assert_array_equal(O.combine(eo2, idx, w), out)


# ------------------------------------------------------------ closed forms
@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_parameter_count_of_generated_layers(name):
    w = synth.WORKLOADS[name]
    if w.D * w.F * w.E > 10_000_000:
        # shapes only: the generator's shapes, not its draws
        gu_rows = 2 * w.F if w.act == synth.ACT_SILU_GATED else w.F
        n = w.E * w.D + w.E * gu_rows * w.D + w.E * w.D * w.F
    else:
        d = synth.make_inputs(w)
        n = sum(int(np.prod(d[k].shape)) for k in ("router", "gate_up_proj", "down_proj"))
        if w.biases:
            n += sum(int(np.prod(d[k].shape)) for k in ("router_bias", "b1", "b2"))
    assert n == O.parameter_count(w.E, w.D, w.F, w.act)


def test_parameter_count_values():
    # the exercise's formula on its layer: E*(2DF+F+D)+D*E+E
    assert O.parameter_count(4, 32, 64, O.ACT_RELU) == 16900
    assert O.parameter_count(8, 64, 128, O.ACT_SILU_GATED) == 197120
    assert O.parameter_count(8, 4096, 14336, O.ACT_SILU_GATED) == 1409318912
    assert O.parameter_count(64, 2048, 1408, O.ACT_SILU_GATED) == 553779200
    # independent of K


@pytest.mark.parametrize("act", [O.ACT_RELU, O.ACT_SILU_GATED])
def test_every_parameter_reaches_the_output(act):
    """Perturbing any single parameter changes the output (K = E, all ReLU
    units active): the count of live parameters equals the closed form, so
    no term (a bias, a gate row, the router bias) is dropped."""
    E, D, F, T = 2, 3, 4, 3
    rng = np.random.default_rng(5)
    x = rng.uniform(0.5, 1.5, (T, D))
    params = {"router": rng.normal(0, 0.5, (E, D)),
              "gate_up_proj": rng.uniform(0.2, 0.6, ((E, F, D) if act == O.ACT_RELU else (E, 2 * F, D))),
              "down_proj": rng.normal(0, 0.5, (E, D, F))}
    if act == O.ACT_RELU:
        params["router_bias"] = rng.normal(0, 0.5, E)
        params["b1"] = rng.uniform(1.0, 2.0, (E, F))   # keeps every unit active
        params["b2"] = rng.normal(0, 0.5, (E, D))

    def run(p):
        return O.moe_ffn_forward(x, p["router"], p["gate_up_proj"], p["down_proj"], K=E,
                                 act=act, router_bias=p.get("router_bias"),
                                 b1=p.get("b1"), b2=p.get("b2"))["out"]

    base = run(params)
    live = 0
    for k, v in params.items():
        for i in np.ndindex(v.shape):
            q = {kk: vv.copy() for kk, vv in params.items()}
            q[k][i] += 1e-3
            if np.abs(run(q) - base).max() > 1e-12:
                live += 1
    assert live == O.parameter_count(E, D, F, act)


def test_softmax_closed_form():
    lg = np.log(np.array([[1.0, 2.0, 3.0], [5.0, 5.0, 5.0]])) + np.array([[7.0], [-300.0]])
    np.testing.assert_allclose(O.softmax(lg), [[1 / 6, 2 / 6, 3 / 6], [1 / 3] * 3], rtol=1e-15)
    from scipy.special import softmax as sp_softmax
    z = np.random.default_rng(0).normal(0, 3, (50, 9))
    np.testing.assert_allclose(O.softmax(z), sp_softmax(z, axis=-1), rtol=1e-13)


# --------------------------------------------------------------- invariants
@pytest.mark.parametrize("seed", range(4))
def test_weight_invariants(seed):
    d = _case(seed, 16, 12, 10, 7)
    for K in range(1, 8):
        r = O.moe_route(d["x"], d["router"], K, True)
        w = r["routing_weights"]
        assert (w >= 0).all()
        assert np.abs(w.sum(-1) - 1).max() <= 1e-6
        if K == 1:
            np.testing.assert_allclose(w, 1.0, atol=1e-8)
        rn = O.moe_route(d["x"], d["router"], K, False)
        np.testing.assert_array_equal(rn["selected_experts"], r["selected_experts"])
        np.testing.assert_allclose(rn["routing_weights"],
                                   np.take_along_axis(r["probs"], r["selected_experts"], 1), rtol=0)
        # the kept weights are in descending order
        assert (np.diff(r["routing_weights"], axis=-1) <= 0).all()


@pytest.mark.parametrize("act", [O.ACT_SILU_GATED, O.ACT_RELU])
def test_k_equals_e_is_full_weighted_sum(act):
    """K = E combines every expert: out = sum_e p_e * expert_e(x) / (1+1e-9),
    with the experts evaluated by torch float64 (a library routine)."""
    import torch
    import torch.nn.functional as Fn
    E, D, F, T = 5, 8, 6, 11
    d = _case(11, T, D, F, E, act=act)
    r = O.moe_ffn_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=E, act=act,
                          router_bias=d["router_bias"], b1=d["b1"], b2=d["b2"])
    x = torch.tensor(d["x"], dtype=torch.float64)
    lg = Fn.linear(x, torch.tensor(d["router"], dtype=torch.float64),
                   None if d["router_bias"] is None else torch.tensor(d["router_bias"], dtype=torch.float64))
    p = torch.softmax(lg, -1)
    ref = torch.zeros(T, D, dtype=torch.float64)
    for e in range(E):
        gu = torch.tensor(d["gate_up_proj"][e], dtype=torch.float64)
        dn = torch.tensor(d["down_proj"][e], dtype=torch.float64)
        if act == O.ACT_SILU_GATED:
            h = Fn.silu(Fn.linear(x, gu[:F])) * Fn.linear(x, gu[F:])
            y = Fn.linear(h, dn)
        else:
            h = torch.relu(Fn.linear(x, gu, torch.tensor(d["b1"][e], dtype=torch.float64)))
            y = Fn.linear(h, dn, torch.tensor(d["b2"][e], dtype=torch.float64))
        ref += p[:, e:e + 1] * y
    ref /= (1 + 1e-9)
    np.testing.assert_allclose(r["out"], ref.numpy(), rtol=1e-12, atol=1e-14)


def test_single_expert_is_a_plain_ffn():
    """E = 1, K = 1: the layer is one SwiGLU MLP scaled by 1/(1+1e-9)."""
    import torch
    import torch.nn.functional as Fn
    d = _case(3, 9, 16, 24, 1)
    r = O.moe_ffn_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=1)
    x = torch.tensor(d["x"], dtype=torch.float64)
    gu = torch.tensor(d["gate_up_proj"][0], dtype=torch.float64)
    y = Fn.linear(Fn.silu(Fn.linear(x, gu[:24])) * Fn.linear(x, gu[24:]),
                  torch.tensor(d["down_proj"][0], dtype=torch.float64))
    np.testing.assert_allclose(r["out"], y.numpy() / (1 + 1e-9), rtol=1e-13, atol=1e-15)
    assert (r["selected_experts"] == 0).all()


# --------------------------------------------------------------- tie-break
def test_tie_break_lower_index():
    p = np.array([[0.25, 0.25, 0.25, 0.25],
                  [0.1, 0.3, 0.3, 0.3],
                  [0.4, 0.2, 0.4, 0.0],
                  [0.0, 0.5, 0.0, 0.5]])
    _, i1 = O.top_k(p, 1)
    _, i2 = O.top_k(p, 2)
    _, i3 = O.top_k(p, 3)
    assert i1[:, 0].tolist() == [0, 1, 0, 1]
    assert i2.tolist() == [[0, 1], [1, 2], [0, 2], [1, 3]]
    assert i3.tolist() == [[0, 1, 2], [1, 2, 3], [0, 2, 1], [1, 3, 0]]


def test_tie_break_duplicate_router_rows():
    """Experts 0 and 1 with identical router rows score identically; the
    lower index is always listed first."""
    d = _case(2, 32, 8, 6, 4)
    router = d["router"].copy()
    router[1] = router[0]
    r = O.moe_route(d["x"], router, 2, True)
    sel = r["selected_experts"]
    both = (sel == 0).any(1) & (sel == 1).any(1)
    assert both.any()
    for row in sel[both]:
        assert list(row).index(0) < list(row).index(1)
    r1 = O.moe_route(d["x"], router, 1, True)
    assert not (r1["selected_experts"] == 1).any()


# -------------------------------------------------------------- equivariance
def test_token_permutation_equivariance():
    d = _case(4, 40, 12, 9, 6)
    perm = np.random.default_rng(1).permutation(40)
    a = O.moe_ffn_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=3)
    b = O.moe_ffn_forward(d["x"][perm], d["router"], d["gate_up_proj"], d["down_proj"], K=3)
    np.testing.assert_array_equal(b["selected_experts"], a["selected_experts"][perm])
    np.testing.assert_allclose(b["routing_weights"], a["routing_weights"][perm], rtol=1e-14)
    np.testing.assert_allclose(b["out"], a["out"][perm], rtol=1e-13, atol=1e-15)


def test_leading_dims_flatten():
    d = synth.make_inputs(synth.SILU_SMALL)
    assert d["x"].shape == (4, 16, 64)
    r = O.moe_ffn_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=2)
    assert r["out"].shape == (4, 16, 64)
    r2 = O.moe_ffn_forward(d["x"].reshape(64, 64), d["router"], d["gate_up_proj"], d["down_proj"], K=2)
    np.testing.assert_array_equal(r["out"].reshape(64, 64), r2["out"])


# ------------------------------------------------------------- brute force
def _brute_force_forward(x, router, gate_up, down, K, act, rb, b1, b2, norm=True):
    """Token by token, scalar loops, only the selected experts evaluated."""
    T, D = x.shape
    E = router.shape[0]
    F = down.shape[2]
    out = np.zeros((T, D))
    sels = []
    for t in range(T):
        lg = [sum(float(x[t, d]) * float(router[e, d]) for d in range(D)) +
              (float(rb[e]) if rb is not None else 0.0) for e in range(E)]
        m = max(lg)
        ex = [np.exp(v - m) for v in lg]
        s = sum(ex)
        p = [v / s for v in ex]
        best = None
        for sub in itertools.combinations(range(E), K):  # ascending tuples
            tot = sum(p[e] for e in sub)
            if best is None or tot > best[0]:
                best = (tot, sub)
        chosen = sorted(best[1], key=lambda e: (-p[e], e))
        sels.append(chosen)
        den = sum(p[e] for e in chosen) + 1e-9 if norm else 1.0
        for e in chosen:
            w = p[e] / den
            h = []
            for f in range(F):
                if act == O.ACT_SILU_GATED:
                    g = sum(float(x[t, d]) * float(gate_up[e, f, d]) for d in range(D))
                    u = sum(float(x[t, d]) * float(gate_up[e, F + f, d]) for d in range(D))
                    h.append(g / (1 + np.exp(-g)) * u)
                else:
                    a = sum(float(x[t, d]) * float(gate_up[e, f, d]) for d in range(D)) + float(b1[e, f])
                    h.append(max(a, 0.0))
            for dd in range(D):
                y = sum(h[f] * float(down[e, dd, f]) for f in range(F))
                if act == O.ACT_RELU:
                    y += float(b2[e, dd])
                out[t, dd] += w * y
    return out, np.array(sels)


@pytest.mark.parametrize("act", [O.ACT_SILU_GATED, O.ACT_RELU])
@pytest.mark.parametrize("E,K", [(1, 1), (3, 2), (4, 4), (6, 3), (5, 1)])
def test_brute_force_tiny(act, E, K):
    T, D, F = 6, 5, 4
    d = _case(100 + E * 7 + K, T, D, F, E, act=act, std=0.8)
    r = O.moe_ffn_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=K, act=act,
                          router_bias=d["router_bias"], b1=d["b1"], b2=d["b2"])
    ref, sel = _brute_force_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K, act,
                                    d["router_bias"], d["b1"], d["b2"])
    np.testing.assert_array_equal(r["selected_experts"], sel)
    np.testing.assert_allclose(r["out"], ref, rtol=1e-12, atol=1e-13)


def test_brute_force_with_exact_ties():
    # four experts with duplicated router rows -> exact probability ties
    T, D, F, E = 5, 4, 3, 4
    d = _case(77, T, D, F, E, std=0.8)
    router = d["router"].copy()
    router[2] = router[0]
    router[3] = router[1]
    for K in (1, 2, 3):
        r = O.moe_ffn_forward(d["x"], router, d["gate_up_proj"], d["down_proj"], K=K)
        ref, sel = _brute_force_forward(d["x"], router, d["gate_up_proj"], d["down_proj"], K,
                                        O.ACT_SILU_GATED, None, None, None)
        np.testing.assert_array_equal(r["selected_experts"], sel)
        np.testing.assert_allclose(r["out"], ref, rtol=1e-12, atol=1e-13)


# ------------------------------------------------- library special cases
def test_relu_expert_matches_torch():
    import torch
    import torch.nn.functional as Fn
    d = _case(8, 7, 10, 12, 3, act=O.ACT_RELU)
    eo = O.expert_outputs(d["x"], d["gate_up_proj"], d["down_proj"], O.ACT_RELU, d["b1"], d["b2"])
    x = torch.tensor(d["x"], dtype=torch.float64)
    for e in range(3):
        l1 = torch.nn.Linear(10, 12, dtype=torch.float64)
        l2 = torch.nn.Linear(12, 10, dtype=torch.float64)
        with torch.no_grad():
            l1.weight.copy_(torch.tensor(d["gate_up_proj"][e]))
            l1.bias.copy_(torch.tensor(d["b1"][e]))
            l2.weight.copy_(torch.tensor(d["down_proj"][e]))
            l2.bias.copy_(torch.tensor(d["b2"][e]))
            y = l2(Fn.relu(l1(x)))
        np.testing.assert_allclose(eo[:, e], y.numpy(), rtol=1e-13, atol=1e-15)


def _mixtral_modules(E, D, F, K, router, gate_up, down):
    import torch
    from transformers.models.mixtral.configuration_mixtral import MixtralConfig
    from transformers.models.mixtral import modeling_mixtral as mm
    cfg = MixtralConfig(hidden_size=D, intermediate_size=F, num_local_experts=E,
                        num_experts_per_tok=K, hidden_act="silu")
    experts = mm.MixtralExperts(cfg).double()
    gate = mm.MixtralTopKRouter(cfg).double()
    with torch.no_grad():
        experts.gate_up_proj.copy_(torch.tensor(np.asarray(gate_up, dtype=np.float64)))
        experts.down_proj.copy_(torch.tensor(np.asarray(down, dtype=np.float64)))
        gate.weight.copy_(torch.tensor(np.asarray(router, dtype=np.float64)))
    return experts, gate


def test_mixtral_library_cross_check():
    """The installed transformers Mixtral experts (run, not copied), in
    float64, fed the oracle's selection and weights, give the oracle's out;
    its router agrees on the selection wherever the K-th/K+1-th gap is
    clear (it takes its softmax in float32)."""
    import torch
    w = synth.SILU_SMALL
    d = synth.make_inputs(w)
    x = d["x"].reshape(-1, w.D)
    r = O.moe_ffn_forward(x, d["router"], d["gate_up_proj"], d["down_proj"], K=w.K)
    experts, gate = _mixtral_modules(w.E, w.D, w.F, w.K, d["router"], d["gate_up_proj"], d["down_proj"])
    with torch.no_grad():
        y = experts(torch.tensor(x, dtype=torch.float64),
                    torch.tensor(r["selected_experts"]),
                    torch.tensor(r["routing_weights"]))
        _, scores, idx = gate(torch.tensor(x, dtype=torch.float64))
    np.testing.assert_allclose(r["out"], y.numpy(), rtol=1e-12, atol=1e-15)
    clear = r["gap"] > 1e-5
    assert clear.sum() > 50
    np.testing.assert_array_equal(idx.numpy()[clear], r["selected_experts"][clear])
    np.testing.assert_allclose(scores.numpy()[clear], r["routing_weights"][clear], rtol=2e-6)


# ----------------------------------------------------------- conventions
def test_error_conventions():
    d = _case(1, 4, 6, 5, 3)
    with pytest.raises(ValueError):
        O.moe_ffn_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=0)
    with pytest.raises(ValueError):
        O.moe_ffn_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=4)
    with pytest.raises(NotImplementedError):
        O.moe_ffn_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=1, act="gelu")


# ---------------------------------------------------------------- mutants
def _pins_pass(mod):
    """The pins above, re-run against a (possibly mutated) oracle module."""
    checks = []
    g = json.load(open(os.path.join(GOLDEN, "worked_example_two_tokens.json")))
    vals, idx = mod.top_k(np.array(g["probs"]), 2)
    w = mod.routing_weights(vals, True)
    out = mod.combine(np.array(g["expert_outs"]), idx, w)
    checks.append(idx.tolist() == g["expected_indices"] and
                  np.allclose(out, g["expected_out"], atol=1e-6, rtol=0))
    for act in (mod.ACT_SILU_GATED, mod.ACT_RELU):
        for (E, K) in ((3, 2), (4, 4)):
            d = _case(100 + E * 7 + K, 6, 5, 4, E, act=act, std=0.8)
            try:
                r = mod.moe_ffn_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=K,
                                        act=act, router_bias=d["router_bias"], b1=d["b1"], b2=d["b2"])
                ref, sel = _brute_force_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"],
                                                K, act, d["router_bias"], d["b1"], d["b2"])
                checks.append(np.array_equal(r["selected_experts"], sel) and
                              np.allclose(r["out"], ref, rtol=1e-12, atol=1e-13))
            except Exception:
                checks.append(False)
    return all(checks)


def test_mutants_are_caught(monkeypatch):
    import importlib
    import types
    assert _pins_pass(O)

    def mutant(name, fn):
        m = types.ModuleType("mutant")
        m.__dict__.update(O.__dict__)
        m.__dict__[name] = fn
        # rebind module-level callers to the mutated globals
        for f in ("moe_route", "moe_ffn_forward", "expert_outputs", "expert_silu_gated",
                  "expert_relu", "combine", "top_k", "routing_weights", "softmax", "router_logits",
                  "silu"):
            if f != name:
                g = O.__dict__[f]
                m.__dict__[f] = types.FunctionType(g.__code__, m.__dict__, f, g.__defaults__)
        return m

    def top_k_unstable(probs, K):
        p = np.asarray(probs, dtype=np.float64)
        order = np.flip(np.argsort(p, axis=-1, kind="stable"), -1)[..., :K]  # ties -> higher index
        return np.take_along_axis(p, order, -1), order

    def silu_gate_up_swapped(x, gate_up_e, down_e):
        gu = np.asarray(gate_up_e, dtype=np.float64)
        F = gu.shape[0] // 2
        return O.expert_silu_gated(x, np.concatenate([gu[F:], gu[:F]]), down_e)

    def relu_no_b2(x, w1, b1, w2, b2):
        return O.expert_relu(x, w1, b1, w2, np.zeros_like(np.asarray(b2, dtype=np.float64)))

    def router_no_bias(x, router, router_bias=None):
        return O.router_logits(x, router, None)

    def weights_unnormalised(vals, norm=True):
        return np.asarray(vals, dtype=np.float64)

    def combine_wrong_token(eo, idx, w):
        eo = np.asarray(eo, dtype=np.float64)
        return O.combine(np.roll(eo, 1, axis=0), idx, w)

    def softmax_on_logits_sum(lg):
        lg = np.asarray(lg, dtype=np.float64)
        return lg / lg.sum(-1, keepdims=True)

    def down_transposed(x, gate_up_e, down_e):
        gu = np.asarray(gate_up_e, dtype=np.float64)
        F = gu.shape[0] // 2
        h = O.silu(x @ gu[:F].T) * (x @ gu[F:].T)
        dn = np.asarray(down_e, dtype=np.float64)
        return h @ dn.reshape(dn.shape[1], dn.shape[0])

    for name, fn in [("top_k", top_k_unstable),
                     ("expert_silu_gated", silu_gate_up_swapped),
                     ("expert_relu", relu_no_b2),
                     ("router_logits", router_no_bias),
                     ("routing_weights", weights_unnormalised),
                     ("combine", combine_wrong_token),
                     ("softmax", softmax_on_logits_sum),
                     ("expert_silu_gated", down_transposed)]:
        assert not _pins_pass(mutant(name, fn)), f"mutant {name}/{fn.__name__} not caught"
