"""GPU parity of the routing extensions (moe_ffn_forward_ex / moe_route_ex)
against the oracle: sigmoid scores, the selection-only bias, the dynamic
threshold, the capacity factor and the balancing statistics.

Downstream decisions are compared given the GPU's own selection: the
threshold decision wherever the oracle's share is not within 1e-5 of the
threshold, the capacity mask bit for bit (pure integer logic on the
selection), the weights and the output within the usual tolerances."""
import numpy as np
import pytest

from mixture_experts_ffn_09_b200 import synth
from oracle import moe_oracle as O

import parity_lib as PL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixture_experts_ffn_09_b200 import build
    build.build()


def run_gpu_ex(dev, E, K, norm, act, **opts):
    import torch
    from mixture_experts_ffn_09_b200 import moe
    x = dev["x"]
    D = x.shape[-1]
    T = x.numel() // D
    F = dev["down_proj"].shape[-1]
    dt = moe.BF16 if x.dtype == torch.bfloat16 else moe.F32
    a = moe.ACT_NAMES[act]
    ws = torch.empty(moe.workspace_size(T, D, F, E, K, dt, a), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(x)
    sel = torch.full((T, K), -1, dtype=torch.int64, device="cuda")
    w = torch.full((T, K), float("nan"), dtype=torch.float32, device="cuda")
    kept = torch.full((T, K), 7, dtype=torch.uint8, device="cuda")
    bal = torch.full((4,), float("nan"), dtype=torch.float32, device="cuda")
    if opts.get("selection_bias") is not None:
        opts["selection_bias"] = torch.from_numpy(np.asarray(opts["selection_bias"], np.float32)).cuda()
    moe.ffn_forward_ex(x, dev["router"], dev["gate_up_proj"], dev["down_proj"], E, K, norm, a, out,
                       sel, w, dev.get("router_bias"), dev.get("b1"), dev.get("b2"), None, ws,
                       slot_kept=kept, balance=bal, **opts)
    assert moe.device_status() == moe.MOE_OK
    return {"out": out.float().cpu().numpy().astype(np.float64).reshape(T, D),
            "sel": sel.cpu().numpy(), "w": w.cpu().numpy().astype(np.float64),
            "kept": kept.cpu().numpy().astype(bool), "balance": bal.cpu().numpy().astype(np.float64)}


def check_ext(d, E, K, norm, act, dtype, tokens=None, score="softmax", sel_bias=None, th=0.0,
              cf=0.0, L=0):
    h = PL.host_views(d)
    dev = PL.to_device(d)
    opts = dict(score=score, selection_bias=sel_bias, dynamic_threshold=th, capacity_factor=cf,
                seq_len=L)
    g = run_gpu_ex(dev, E, K, norm, act, **opts)
    assert set(np.unique(g["kept"]).tolist()) <= {False, True}
    x = h["x"].reshape(-1, h["x"].shape[-1])
    r = O.moe_route_ext(x, h["router"], K, norm, h["router_bias"], score, sel_bias, th)
    clear = r["gap"] > PL.GAP
    np.testing.assert_array_equal(g["sel"][clear], r["selected_experts"][clear])
    # every selection valid: K distinct experts whose biased score is within
    # the gap of the K-th
    rank_by = r["probs"] + (0 if sel_bias is None else np.asarray(sel_bias)[None, :])
    kth = np.sort(rank_by, 1)[:, ::-1][:, K - 1]
    assert (np.take_along_axis(rank_by, g["sel"], 1) >= kth[:, None] - PL.GAP).all()
    # weights on the GPU's selection
    vals = np.take_along_axis(r["probs"], g["sel"], 1)
    if th > 0:
        share = vals / vals.sum(1, keepdims=True)
        active_ref = share >= th
        active_ref[:, 0] = True
        active = g["w"] > 0
        ambiguous = np.abs(share - th) < 1e-5
        ambiguous[:, 0] = False
        np.testing.assert_array_equal(active[~ambiguous], active_ref[~ambiguous])
        kshare = np.where(active, share, 0.0)
        w_ref = kshare / kshare.sum(1, keepdims=True)
    else:
        active = np.ones_like(g["sel"], dtype=bool)
        w_ref = O.routing_weights(vals, norm)
    np.testing.assert_allclose(g["w"], w_ref, atol=1e-5, rtol=0)
    kept_ref = active.copy()
    if cf > 0:
        kept_ref &= O.capacity_keep(g["sel"], E, cf, L, active)
    np.testing.assert_array_equal(g["kept"], kept_ref)
    # output of the kept slots only
    tok = np.arange(x.shape[0]) if tokens is None else tokens
    eo = O.expert_outputs(x[tok], h["gate_up_proj"], h["down_proj"], act, h["b1"], h["b2"])
    ref = O.combine(eo, g["sel"][tok], np.where(kept_ref[tok], w_ref[tok], 0.0))
    PL.check_out(g["out"][tok], ref, dtype)
    # balancing statistics of the batch
    b = O.balance_stats(r["probs"], g["sel"], w_ref)
    got = dict(zip(("switch", "gshard", "master", "gshard_probs"), g["balance"]))
    for k in b:
        assert got[k] == pytest.approx(b[k], rel=2e-4, abs=1e-6), k
    return g


CASES = [(300, 136, 200, 8, 2, "bf16"), (100, 33, 47, 6, 3, "f32")]


@pytest.mark.parametrize("T,D,F,E,K,dtype", CASES)
@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
@pytest.mark.parametrize("biased", [False, True])
def test_scores_and_selection_bias(T, D, F, E, K, dtype, score, biased):
    d = synth.random_case(200 + T, T, D, F, E, dtype=dtype, weight_std=0.3 if dtype == "f32" else 0.05)
    bias = np.random.default_rng(1).normal(0, 0.05, E).astype(np.float32) if biased else None
    check_ext(d, E, K, True, "silu_gated", dtype, score=score, sel_bias=bias)


@pytest.mark.parametrize("T,D,F,E,K,dtype", CASES + [(256, 64, 64, 16, 10, "bf16"),
                                                      (256, 64, 64, 16, 10, "f32")])
@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
def test_balance_with_norm_topk_prob_off(T, D, F, E, K, dtype, score):
    """With norm_topk_prob off the output weights are the raw kept scores,
    but the balance statistics still read the renormalised selection (ES-MoE
    API page, "Balancing objectives").  K = 10 takes the routers'
    round-per-choice path."""
    d = synth.random_case(400 + T + K, T, D, F, E, dtype=dtype,
                          weight_std=0.3 if dtype == "f32" else 0.05)
    g = check_ext(d, E, K, False, "silu_gated", dtype, score=score)
    # the raw kept scores do not sum to one, so a gate that was not
    # renormalised would give other statistics
    assert np.abs(g["w"].sum(1) - 1.0).max() > 1e-3


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("th", [0.15, 0.3, 0.9])
def test_dynamic_threshold(dtype, th):
    d = synth.random_case(31, 256, 64, 96, 8, dtype=dtype, weight_std=0.4 if dtype == "f32" else 0.2)
    g = check_ext(d, 8, 4, True, "silu_gated", dtype, th=th)
    assert (~g["kept"]).any()
    assert g["kept"][:, 0].all()


@pytest.mark.parametrize("cf,L", [(1.0, 0), (0.5, 0), (1.0, 64), (0.75, 32), (2.0, 96)])
def test_capacity_factor(cf, L):
    d = dict(synth.random_case(41, 300, 64, 128, 8, dtype="bf16", weight_std=0.05))
    rb = np.zeros(8, np.float32)
    rb[:3] = [2.0, 1.0, 0.5]            # skew the load so the capacity binds
    d["router_bias"] = rb
    g = check_ext(d, 8, 2, True, "silu_gated", "bf16", cf=cf, L=L)
    if cf <= 1.0:
        assert (~g["kept"]).any()


def test_capacity_on_the_float32_path():
    d = synth.random_case(43, 96, 40, 24, 4, dtype="f32", weight_std=0.4)
    check_ext(d, 4, 2, True, "silu_gated", "f32", cf=0.5, L=32)


def test_all_extensions_together():
    d = synth.random_case(51, 320, 128, 128, 16, dtype="bf16", weight_std=0.05)
    bias = np.random.default_rng(2).normal(0, 0.03, 16).astype(np.float32)
    check_ext(d, 16, 4, True, "silu_gated", "bf16", score="sigmoid", sel_bias=bias, th=0.2, cf=1.0,
              L=64)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_all_extensions_with_more_than_eight_choices(dtype):
    """K > 8 takes the routers' round-per-choice path: every extension at
    once there too."""
    d = synth.random_case(52, 256, 64, 64, 16, dtype=dtype, weight_std=0.3 if dtype == "f32" else 0.05)
    bias = np.random.default_rng(5).normal(0, 0.03, 16).astype(np.float32)
    check_ext(d, 16, 10, True, "silu_gated", dtype, score="sigmoid", sel_bias=bias, th=0.05,
              cf=1.0, L=64)


def test_relu_expert_with_capacity_and_threshold():
    d = synth.random_case(61, 200, 72, 80, 5, act="relu", dtype="bf16", weight_std=0.1)
    check_ext(d, 5, 3, True, "relu", "bf16", th=0.25, cf=1.0, L=32)


def test_fine_grained_full_size_with_capacity():
    """The Zipf-skewed fine-grained layer with a capacity of 1.25 per
    sequence of 4096 tokens: the hot experts drop slots."""
    w = synth.FINE_GRAINED
    d = synth.make_inputs(w)
    h = PL.host_views(d)
    r = PL.oracle_route(h, w.K, True)
    tok = PL.sample_tokens(r["selected_experts"], w.E, 64)
    g = check_ext(d, w.E, w.K, True, w.act, w.dtype, tokens=tok, cf=1.25, L=4096)
    assert (~g["kept"]).mean() > 0.05


def test_route_ex_entry_point():
    import torch
    from mixture_experts_ffn_09_b200 import moe
    d = synth.random_case(71, 128, 64, 64, 8, dtype="bf16", weight_std=0.1)
    h = PL.host_views(d)
    dev = PL.to_device(d)
    bias = np.random.default_rng(3).normal(0, 0.05, 8).astype(np.float32)
    sel = torch.empty(128, 3, dtype=torch.int64, device="cuda")
    wt = torch.empty(128, 3, dtype=torch.float32, device="cuda")
    kept = torch.empty(128, 3, dtype=torch.uint8, device="cuda")
    moe.route_ex(dev["x"], dev["router"], 3, True, sel, wt, score="sigmoid",
                 selection_bias=torch.from_numpy(bias).cuda(), dynamic_threshold=0.2, slot_kept=kept)
    torch.cuda.synchronize()
    r = O.moe_route_ext(h["x"], h["router"], 3, True, None, "sigmoid", bias, 0.2)
    clear = r["gap"] > PL.GAP
    np.testing.assert_array_equal(sel.cpu().numpy()[clear], r["selected_experts"][clear])
    np.testing.assert_allclose(wt.cpu().numpy()[clear], r["routing_weights"][clear], atol=1e-5)
    np.testing.assert_array_equal(kept.cpu().numpy().astype(bool)[clear], r["active"][clear])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
def test_nan_tokens_are_contained(dtype, score):
    """Tokens whose x holds NaN still get K real experts (NaN scores rank
    last), nothing faults, and every other token's result is bit for bit the
    one it gets without the NaN tokens present (rows are independent)."""
    import torch
    d = synth.random_case(301, 200, 64, 96, 8, dtype=dtype, weight_std=0.1)
    bias = np.random.default_rng(4).normal(0, 0.05, 8).astype(np.float32)
    clean = PL.to_device(d)
    dirty = dict(clean)
    xd = clean["x"].clone()
    bad = [0, 5, 77, 199]
    xd[bad] = float("nan")
    dirty["x"] = xd
    opts = dict(score=score, selection_bias=bias)
    a = run_gpu_ex(clean, 8, 3, True, "silu_gated", **dict(opts))
    b = run_gpu_ex(dirty, 8, 3, True, "silu_gated", **dict(opts))
    assert ((b["sel"] >= 0) & (b["sel"] < 8)).all()
    keep = np.setdiff1d(np.arange(200), bad)
    np.testing.assert_array_equal(b["sel"][keep], a["sel"][keep])
    np.testing.assert_array_equal(b["w"][keep], a["w"][keep])
    np.testing.assert_array_equal(b["out"][keep], a["out"][keep])
