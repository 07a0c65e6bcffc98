"""Pins of the oracle's routing extensions (CPU only): sigmoid scores, the
selection-only bias, ES-MoE's dynamic threshold, the capacity factor and the
balancing statistics - each tied to hand-worked cases from the cited
definitions, closed forms, or an independent formulation."""
import itertools

import numpy as np
import pytest

from oracle import moe_oracle as O
from mixture_experts_ffn_09_b200 import synth


def _case(seed, T, D, F, E, std=0.5):
    return synth.random_case(seed, T, D, F, E, weight_std=std)


# ----------------------------------------------------------------- sigmoid
def test_sigmoid_scores_match_expit():
    from scipy.special import expit
    z = np.random.default_rng(0).normal(0, 4, (40, 7))
    np.testing.assert_allclose(O.router_scores(z, O.SCORE_SIGMOID), expit(z), rtol=1e-15)
    # one expert's score does not depend on the others (no normalisation over experts)
    z2 = z.copy()
    z2[:, 3] += 5.0
    s1, s2 = O.sigmoid(z), O.sigmoid(z2)
    np.testing.assert_array_equal(np.delete(s1, 3, 1), np.delete(s2, 3, 1))


def _brute_select(scores, bias, K):
    T, E = scores.shape
    rank_by = scores + (0 if bias is None else bias[None, :])
    out = []
    for t in range(T):
        best = None
        for sub in itertools.combinations(range(E), K):
            tot = sum(rank_by[t, e] for e in sub)
            if best is None or tot > best[0]:
                best = (tot, sub)
        out.append(sorted(best[1], key=lambda e: (-rank_by[t, e], e)))
    return np.array(out)


@pytest.mark.parametrize("score", [O.SCORE_SOFTMAX, O.SCORE_SIGMOID])
@pytest.mark.parametrize("with_bias", [False, True])
def test_selection_brute_force(score, with_bias):
    rng = np.random.default_rng(3)
    lg = rng.normal(0, 1.5, (9, 6))
    bias = rng.normal(0, 0.3, 6) if with_bias else None
    sc = O.router_scores(lg, score)
    for K in (1, 2, 4, 6):
        vals, idx = O.select_experts(sc, K, bias)
        np.testing.assert_array_equal(idx, _brute_select(sc, bias, K))
        # the weights come from the unbiased scores of the chosen experts
        np.testing.assert_array_equal(vals, np.take_along_axis(sc, idx, 1))


def test_large_selection_bias_forces_the_choice_not_the_weight():
    d = _case(4, 20, 8, 6, 5)
    bias = np.zeros(5)
    bias[3] = 100.0
    r = O.moe_route_ext(d["x"], d["router"], 2, True, None, O.SCORE_SOFTMAX, bias)
    assert (r["selected_experts"][:, 0] == 3).all()
    p = r["probs"]
    w_expected = np.take_along_axis(p, r["selected_experts"], 1)
    w_expected = w_expected / (w_expected.sum(1, keepdims=True) + 1e-9)
    np.testing.assert_allclose(r["routing_weights"], w_expected, rtol=1e-15)
    # zero bias = no bias
    r0 = O.moe_route_ext(d["x"], d["router"], 2, True, None, O.SCORE_SOFTMAX, np.zeros(5))
    rr = O.moe_route(d["x"], d["router"], 2, True)
    np.testing.assert_array_equal(r0["selected_experts"], rr["selected_experts"])
    np.testing.assert_array_equal(r0["routing_weights"], rr["routing_weights"])


def test_sigmoid_k_equals_e_full_weighted_sum():
    import torch
    import torch.nn.functional as Fn
    E, D, F, T = 4, 6, 5, 7
    d = _case(9, T, D, F, E)
    r = O.moe_ffn_forward_ext(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=E,
                              score=O.SCORE_SIGMOID)
    x = torch.tensor(d["x"], dtype=torch.float64)
    s = torch.sigmoid(x @ torch.tensor(d["router"], dtype=torch.float64).T)
    ref = torch.zeros(T, D, dtype=torch.float64)
    for e in range(E):
        gu = torch.tensor(d["gate_up_proj"][e], dtype=torch.float64)
        y = Fn.linear(Fn.silu(Fn.linear(x, gu[:F])) * Fn.linear(x, gu[F:]),
                      torch.tensor(d["down_proj"][e], dtype=torch.float64))
        ref += s[:, e:e + 1] * y
    ref /= s.sum(1, keepdim=True) + 1e-9
    np.testing.assert_allclose(r["out"], ref.numpy(), rtol=1e-12, atol=1e-14)


# ------------------------------------------------------- dynamic threshold
def test_dynamic_threshold_hand_cases():
    w = np.array([[0.6, 0.3, 0.1], [0.5, 0.3, 0.2], [0.34, 0.33, 0.33]])
    nw, keep = O.apply_dynamic_threshold(w, 0.2)
    np.testing.assert_allclose(nw, [[2 / 3, 1 / 3, 0.0], [0.5, 0.3, 0.2], [0.34, 0.33, 0.33]],
                               rtol=1e-15)
    assert keep.tolist() == [[True, True, False], [True, True, True], [True, True, True]]
    # every share below the threshold: the leader stays alone with weight one
    nw, keep = O.apply_dynamic_threshold(np.array([[0.3, 0.25, 0.25, 0.2]]), 0.5)
    np.testing.assert_array_equal(nw, [[1.0, 0.0, 0.0, 0.0]])
    assert keep.tolist() == [[True, False, False, False]]
    # the share is the renormalised weight, not the raw probability
    nw, _ = O.apply_dynamic_threshold(np.array([[0.06, 0.03, 0.01]]), 0.2)
    np.testing.assert_allclose(nw, [[2 / 3, 1 / 3, 0.0]], rtol=1e-14)


def test_dynamic_threshold_invariants():
    d = _case(5, 50, 8, 6, 8)
    for th in (0.05, 0.2, 0.4, 0.9):
        r = O.moe_route_ext(d["x"], d["router"], 4, True, dynamic_threshold=th)
        w, keep = r["routing_weights"], r["active"]
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)
        assert keep[:, 0].all() and (w[~keep] == 0).all()
        base = O.moe_route(d["x"], d["router"], 4, True)["routing_weights"]
        share = base / base.sum(1, keepdims=True)
        assert (share[:, 1:][keep[:, 1:]] >= th).all() and (share[:, 1:][~keep[:, 1:]] < th).all()


# ------------------------------------------------------------- capacity
def test_capacity_slots_formula():
    assert O.capacity_slots(6, 1, 2, 1.0) == 3
    assert O.capacity_slots(4096, 2, 8, 1.25) == 1280
    assert O.capacity_slots(10, 2, 8, 1.25) == 3          # ceil(2.5)=3, *1.25 = 3.75 -> 3
    assert O.capacity_slots(1, 1, 64, 2.0) == 2           # the floor cf itself
    assert O.capacity_slots(3, 2, 8, 0.5) == 0


def test_capacity_hand_cases():
    idx = np.zeros((6, 1), dtype=np.int64)                 # every token on expert 0
    assert O.capacity_keep(idx, 2, 1.0).ravel().tolist() == [1, 1, 1, 0, 0, 0]
    # two sequences of 3 tokens: capacity max(ceil(3/2)*1, 1) = 2 each
    assert O.capacity_keep(idx, 2, 1.0, 3).ravel().tolist() == [1, 1, 0, 1, 1, 0]
    # ragged last sequence of 2 tokens: capacity max(ceil(2/2), 1) = 1
    assert O.capacity_keep(idx, 2, 1.0, 4).ravel().tolist() == [1, 1, 0, 0, 1, 0]
    # slots already inactive take no capacity
    act = np.array([[False], [True], [True], [True], [True], [True]])
    assert O.capacity_keep(idx, 2, 1.0, 0, act).ravel().tolist() == [0, 1, 1, 1, 0, 0]


def test_capacity_against_cumulative_counts():
    """Independent formulation: a pair is kept iff the number of earlier
    active pairs of the same sequence and expert is below the capacity."""
    rng = np.random.default_rng(1)
    T, K, E = 37, 3, 5
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)])
    act = rng.random((T, K)) > 0.2
    for L in (0, 8, 10):
        for cf in (0.5, 1.0, 1.3):
            keep = O.capacity_keep(idx, E, cf, L, act)
            Lr = T if L == 0 else L
            flat_e = idx.ravel()
            flat_a = act.ravel()
            seq = np.repeat(np.arange(T) // Lr, K)
            ref = np.zeros(T * K, dtype=bool)
            for s in np.unique(seq):
                n_s = int((np.arange(T) // Lr == s).sum())
                cap = int(np.floor(max(np.ceil(n_s * K / E) * cf, cf)))
                for e in range(E):
                    m = (seq == s) & (flat_e == e) & flat_a
                    ranks = np.cumsum(m) - 1
                    ref |= m & (ranks < cap)
            np.testing.assert_array_equal(keep.ravel(), ref)


def test_capacity_dropped_slots_add_nothing():
    d = _case(6, 24, 8, 6, 4)
    full = O.moe_ffn_forward_ext(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=2)
    cap = O.moe_ffn_forward_ext(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=2,
                                capacity_factor=0.5, seq_len=8)
    assert (~cap["kept"]).any()
    eo = O.expert_outputs(d["x"], d["gate_up_proj"], d["down_proj"])
    ref = O.combine(eo, full["selected_experts"], np.where(cap["kept"], full["routing_weights"], 0))
    np.testing.assert_allclose(cap["out"], ref, rtol=1e-14)
    big = O.moe_ffn_forward_ext(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=2,
                                capacity_factor=100.0)
    assert big["kept"].all()
    np.testing.assert_array_equal(big["out"], full["out"])


# ------------------------------------------------------------- balance
# ES-MoE API page, "Balancing objectives": probs is the router's full score
# matrix, gate the top-k selection renormalised, both (batch, E); u is a
# per-expert mean normalised to sum to one.  The hand-worked cases below use
# fractional gates (so mean(gate > 0) != mean(gate)) and sigmoid scores
# (whose per-expert means do not sum to one).

# Case A: E=3, two tokens, K=2.  Token 0 scores [0.5, 0.3, 0.2] keeps experts
# 0, 1 with renormalised gate [5/8, 3/8, 0]; token 1 scores [0.1, 0.3, 0.6]
# keeps 2, 1 with gate [0, 1/3, 2/3].
#   mean(probs)    = [0.3, 0.3, 0.4]
#   mean(gate > 0) = [1/2, 1, 1/2]  -> switch = 3 * (0.15 + 0.3 + 0.2) = 1.95
#   u = mean(gate) = [5/16, 17/48, 1/3] (sums to one) -> gshard = 3 * 770/2304
#   master = (gshard - 1) / 9 = 1/3456;  gshard_probs = 3 * 0.34 = 1.02
CASE_A = dict(probs=[[0.5, 0.3, 0.2], [0.1, 0.3, 0.6]], idx=[[0, 1], [2, 1]],
              vals=[[0.5, 0.3], [0.6, 0.3]],
              expect={"switch": 1.95, "gshard": 2310 / 2304, "master": 1 / 3456,
                      "gshard_probs": 1.02})
# Case B: sigmoid scores, E=2, K=1.  Scores [0.9, 0.5] and [0.7, 0.1]: both
# tokens keep expert 0 with gate 1.
#   mean(probs) = [0.8, 0.3] (sum 1.1) -> v = [8/11, 3/11],
#   gshard_probs = 2 * 73/121;  switch = 2 * (0.8 * 1 + 0.3 * 0) = 1.6;
#   u = [1, 0] -> gshard = 2, master = ((1/2)^2 + (1/2)^2) / 2 = 1/4
CASE_B = dict(probs=[[0.9, 0.5], [0.7, 0.1]], idx=[[0], [0]], vals=[[0.9], [0.7]],
              expect={"switch": 1.6, "gshard": 2.0, "master": 0.25, "gshard_probs": 146 / 121})


def _balance_pins_pass(fn):
    """The balance pins of this file, run against a (possibly mutated)
    balance function."""
    ok = []
    for case in (CASE_A, CASE_B):
        p, idx, vals = (np.array(case[k], dtype=np.float64) for k in ("probs", "idx", "vals"))
        idx = idx.astype(np.int64)
        # the gate is the renormalised selection: raw kept scores (norm off)
        # and renormalised weights (norm on) give the same statistics
        for w in (vals, O.routing_weights(vals, True)):
            b = fn(p, idx, w)
            ok.append(all(abs(b[k] - v) <= 1e-9 * max(1.0, abs(v)) for k, v in case["expect"].items()))
    # the closed forms of a uniform router and of a collapsed one
    E, T = 4, 8
    u = np.full((T, E), 1.0 / E)
    b = fn(u, (np.arange(T) % E)[:, None], np.ones((T, 1)))
    ok.append(all(abs(b[k] - v) <= 1e-12 for k, v in
                  {"switch": 1.0, "gshard": 1.0, "master": 0.0, "gshard_probs": 1.0}.items()))
    b = fn(u, np.zeros((T, 1), dtype=np.int64), np.ones((T, 1)))
    ok.append(abs(b["gshard"] - E) <= 1e-12 and abs(b["master"] - (E - 1) / E ** 2) <= 1e-12
              and abs(b["switch"] - 1.0) <= 1e-12)
    # a slot with weight 0 (dropped by the threshold) is not a selection
    b = fn(np.array([[0.6, 0.4]]), np.array([[0, 1]]), np.array([[1.0, 0.0]]))
    ok.append(abs(b["switch"] - 2 * 0.6) <= 1e-12 and abs(b["gshard"] - 2.0) <= 1e-12)
    return all(ok)


def test_balance_hand_worked_cases():
    assert _balance_pins_pass(O.balance_stats)


def test_balance_master_is_gshard_minus_one_over_e_squared():
    d = _case(7, 64, 8, 6, 8)
    r = O.moe_route(d["x"], d["router"], 2, True)
    b = O.balance_stats(r["probs"], r["selected_experts"], r["routing_weights"])
    assert b["master"] == pytest.approx((b["gshard"] - 1) / 8 ** 2, rel=1e-12)
    assert 1.0 <= b["gshard"] <= 8.0 and 1.0 <= b["gshard_probs"] <= 8.0


@pytest.mark.parametrize("score", [O.SCORE_SOFTMAX, O.SCORE_SIGMOID])
def test_balance_does_not_depend_on_norm_topk_prob(score):
    """The gate is renormalised by definition, so the forward's statistics
    are the same with and without the output weights' renormalisation."""
    d = _case(12, 40, 8, 6, 6)
    kw = dict(score=score)
    a = O.moe_ffn_forward_ext(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=3,
                              norm_topk_prob=True, **kw)["balance"]
    b = O.moe_ffn_forward_ext(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=3,
                              norm_topk_prob=False, **kw)["balance"]
    for k in a:
        assert a[k] == pytest.approx(b[k], rel=1e-12), k


def test_balance_mutants_are_caught():
    """Plausible misreadings of the objectives, each of which the pins above
    must reject."""
    def gate_of(p, idx, w, renorm=True):
        w = np.asarray(w, dtype=np.float64)
        if renorm:
            w = w / w.sum(-1, keepdims=True)
        g = np.zeros(np.shape(p))
        np.put_along_axis(g, np.asarray(idx, dtype=np.int64), w, axis=1)
        return g

    def stats(p, g, switch_frac=None, norm_v=True, master_scale=1.0):
        p = np.asarray(p, dtype=np.float64)
        E = p.shape[1]
        mp, mg = p.mean(0), g.mean(0)
        frac = (g > 0).mean(0) if switch_frac is None else switch_frac
        u = mg / mg.sum()
        v = mp / mp.sum() if norm_v else mp
        return {"switch": E * float((mp * frac).sum()), "gshard": E * float((u * u).sum()),
                "master": master_scale * float(((u - 1 / E) ** 2).sum() / E),
                "gshard_probs": E * float((v * v).sum())}

    def switch_on_mean_gate(p, idx, w):
        g = gate_of(p, idx, w)
        return stats(p, g, switch_frac=g.mean(0))

    def gshard_probs_unnormalised(p, idx, w):
        return stats(p, gate_of(p, idx, w), norm_v=False)

    def gate_not_renormalised(p, idx, w):
        return stats(p, gate_of(p, idx, w, renorm=False))

    def master_without_one_over_e(p, idx, w):
        return stats(p, gate_of(p, idx, w), master_scale=np.shape(p)[1])

    def gshard_reads_probs(p, idx, w):
        r = stats(p, gate_of(p, idx, w))
        r["gshard"] = r["gshard_probs"]
        return r

    # the helpers reproduce the oracle when unmutated, so each mutant differs
    # from it in exactly one place
    assert _balance_pins_pass(lambda p, idx, w: stats(p, gate_of(p, idx, w)))
    for fn in (switch_on_mean_gate, gshard_probs_unnormalised, gate_not_renormalised,
               master_without_one_over_e, gshard_reads_probs):
        assert not _balance_pins_pass(fn), fn.__name__


def test_ext_forward_without_extensions_is_the_plain_forward():
    d = _case(8, 30, 8, 6, 5)
    a = O.moe_ffn_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=2)
    b = O.moe_ffn_forward_ext(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], K=2)
    np.testing.assert_array_equal(a["out"], b["out"])
    np.testing.assert_array_equal(a["selected_experts"], b["selected_experts"])
