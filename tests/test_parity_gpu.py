"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded inputs.  See parity_lib for the comparison rule."""
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


def _full_check(d, E, K, norm, act, dtype, x_shape=None):
    """Whole-layer parity on every token (small cases)."""
    h = PL.host_views(d)
    dev = PL.to_device(d)
    g = PL.run_gpu(dev, E, K, norm, act)
    x = h["x"].reshape(-1, h["x"].shape[-1])
    r = O.moe_ffn_forward(x, h["router"], h["gate_up_proj"], h["down_proj"], K, norm, act,
                          h["router_bias"], h["b1"], h["b2"])
    clear = PL.check_routing(g, r, K, norm)
    ref = r["out"].copy()
    if (~clear).any():
        un = np.nonzero(~clear)[0]
        ref[un] = PL.oracle_out_for(h, un, g["sel"][un], K, norm, act)
    PL.check_out(g["out"], ref, dtype)
    lg_scale = np.abs(r["router_logits"]).max()
    assert np.abs(g["logits"] - r["router_logits"]).max() <= 1e-5 * max(lg_scale, 1.0)
    return g, r


# ------------------------------------------------------- the five workloads
def test_dense_relu_exercise_layer():
    w = synth.DENSE_RELU
    _full_check(synth.make_inputs(w), w.E, w.K, w.norm_topk_prob, w.act, w.dtype)


def test_silu_gated_mojolearn_layer():
    w = synth.SILU_SMALL
    d = synth.make_inputs(w)
    assert d["x"].shape == (4, 16, 64)
    g, _ = _full_check(d, w.E, w.K, w.norm_topk_prob, w.act, w.dtype)


@pytest.fixture(scope="module")
def decode_case():
    w = synth.DECODE[1]
    d = synth.make_inputs(w)
    h = PL.host_views(d)
    eo = O.expert_outputs(h["x"], h["gate_up_proj"], h["down_proj"], w.act)   # dense, shared by K
    return w, d, h, PL.to_device(d), eo


@pytest.mark.parametrize("K", [1, 2, 8])
def test_decode_weight_streaming(decode_case, K):
    w, d, h, dev, eo = decode_case
    g = PL.run_gpu(dev, w.E, K, True, w.act)
    r = O.moe_route(h["x"], h["router"], K, True)
    clear = PL.check_routing(g, r, K, True)
    ref = O.combine(eo, r["selected_experts"], r["routing_weights"])
    if (~clear).any():
        un = np.nonzero(~clear)[0]
        v = np.take_along_axis(r["probs"][un], g["sel"][un], 1)
        ref[un] = O.combine(eo[un], g["sel"][un], O.routing_weights(v, True))
    PL.check_out(g["out"], ref, "bf16")
    if K == w.E:
        # K = E combines every expert: the full softmax-weighted sum
        full = np.einsum("te,ted->td", r["probs"], eo) / (1 + 1e-9)
        PL.check_out(g["out"], full, "bf16", "K=E full weighted sum")


def _sampled_full_size(w, n_sample):
    d = synth.make_inputs(w)
    h = PL.host_views(d)
    dev = PL.to_device(d)
    g = PL.run_gpu(dev, w.E, w.K, w.norm_topk_prob, w.act)
    r = PL.oracle_route(h, w.K, w.norm_topk_prob)
    clear = PL.check_routing(g, r, w.K, w.norm_topk_prob)
    assert clear.mean() > 0.99
    # the sample reaches every expert's last row blocks (on the GPU's own
    # selection, which decides the sorted rows), so the tail tiles - swapped
    # on the CTA-pair GEMM - are checked at full K depth
    tails = PL.tail_tokens(g["sel"], w.E)
    tok = PL.sample_tokens(r["selected_experts"], w.E, n_sample, tails=tails)
    ref = PL.oracle_out_for(h, tok, g["sel"][tok], w.K, w.norm_topk_prob, w.act)
    PL.check_out(g["out"][tok], ref, w.dtype)
    tail_set = sorted({t for v in tails.values() for t in v})
    assert set(tail_set) <= set(tok.tolist())
    pos = {int(t): i for i, t in enumerate(tok)}
    ti = [pos[t] for t in tail_set]
    PL.check_out(g["out"][tok][ti], ref[ti], w.dtype,
                 f"tail-block tokens of every expert ({len(tail_set)} tokens)")
    # every token's output is finite and no row was left unwritten
    assert np.isfinite(g["out"]).all()
    return g, r


def test_mixtral_8x7b_full_size_sampled():
    _sampled_full_size(synth.MIXTRAL, 48)


def test_gemm_variants_agree_on_the_mixtral_layer():
    """The one-CTA and CTA-pair GEMMs on the full Mixtral-shaped layer: same
    selection, outputs within the bf16 bound of each other."""
    from mixture_experts_ffn_09_b200 import moe
    w = synth.MIXTRAL
    dev = PL.to_device(synth.make_inputs(w))
    res = []
    for mode in (1, 2):
        prev = moe.set_gemm_mode(mode)
        try:
            res.append(PL.run_gpu(dev, w.E, w.K, True, w.act, with_logits=False))
        finally:
            moe.set_gemm_mode(prev)
    np.testing.assert_array_equal(res[0]["sel"], res[1]["sel"])
    PL.check_out(res[1]["out"], res[0]["out"], "bf16", "pair vs one-CTA GEMM")


def test_fine_grained_zipf_full_size_sampled():
    g, r = _sampled_full_size(synth.FINE_GRAINED, 96)
    load = np.bincount(g["sel"].ravel(), minlength=64)
    assert load[0] == load.max()        # the rank-1 expert is the hottest


# ------------------------------------------------ shapes, tails, edge cases
CASES = [
    # T, D, F, E, K, act, dtype
    (300, 136, 200, 5, 2, "silu_gated", "bf16"),    # ragged K and N tails
    (1, 64, 64, 4, 2, "silu_gated", "bf16"),        # one token
    (257, 128, 256, 8, 8, "silu_gated", "bf16"),    # K = E
    (130, 72, 88, 3, 1, "silu_gated", "bf16"),      # K = 1
    (512, 512, 384, 8, 2, "silu_gated", "bf16"),    # several tiles per expert
    (200, 64, 64, 256, 4, "silu_gated", "bf16"),    # the maximum expert count, most empty
    (300, 136, 200, 5, 2, "relu", "bf16"),          # biased Dense/ReLU expert on tensor cores
    (100, 33, 47, 6, 3, "silu_gated", "f32"),       # odd sizes on the fp32 path
    (77, 50, 30, 4, 2, "relu", "f32"),
    (1, 8, 8, 1, 1, "silu_gated", "f32"),           # one token, one expert
    (129, 264, 520, 1, 1, "silu_gated", "bf16"),    # one expert: a plain FFN
    (160, 128, 128, 16, 12, "silu_gated", "bf16"),  # K > 8: the router's round-per-choice path
    (150, 96, 64, 100, 6, "silu_gated", "bf16"),    # E in (64, 128]: 128-column router tile
    (60, 32, 32, 20, 10, "silu_gated", "f32"),      # K > 8 on the fp32 router
]


@pytest.fixture
def gemm_mode(request):
    from mixture_experts_ffn_09_b200 import moe
    prev = moe.set_gemm_mode(request.param)
    yield request.param
    moe.set_gemm_mode(prev)


MODES = [1, 2]   # one CTA per tile / CTA pairs (the automatic choice is covered by the workloads)


@pytest.fixture
def tail_swap(request):
    from mixture_experts_ffn_09_b200 import moe
    prev = moe.set_tail_swap(request.param)
    yield request.param
    moe.set_tail_swap(prev)


TAIL_SWAPS = [0, 32, 128]   # off / tails of at most 32 rows / the default (and the maximum)


@pytest.mark.parametrize("gemm_mode", MODES, indirect=True)
@pytest.mark.parametrize("T,D,F,E,K,act,dtype", CASES)
def test_shapes_and_edges(T, D, F, E, K, act, dtype, gemm_mode):
    if dtype == "f32" and gemm_mode != MODES[0]:
        pytest.skip("the float32 path has one GEMM")
    d = synth.random_case(1000 + T + D + E, T, D, F, E, act=act, dtype=dtype,
                          weight_std=0.3 if dtype == "f32" else 0.05)
    _full_check(d, E, K, True, act, dtype)


# rows per expert around every tile boundary: 128-row tiles (one CTA) and
# 256-row pair tiles, whose last tile runs at M = 128 when it holds <= 128 rows
TAIL_COUNTS = [1, 64, 65, 127, 128, 129, 255, 256, 257, 383, 384, 385]


@pytest.mark.parametrize("tail_swap", TAIL_SWAPS, indirect=True)
@pytest.mark.parametrize("gemm_mode", MODES, indirect=True)
@pytest.mark.parametrize("act", ["silu_gated", "relu"])
def test_tile_tails_every_boundary(act, gemm_mode, tail_swap):
    """Token t is steered to a chosen expert (a dominant router column), so
    every expert gets one of TAIL_COUNTS rows; each tile shape and tail is
    then compared with the oracle on every token.  On the pair GEMM the
    counts put tails on both sides of every swap threshold tested and of
    every swapped N (tails of 1, 64, 65, 127, 128, 129 and 255 rows)."""
    if gemm_mode == 1 and tail_swap != 128:
        pytest.skip("the tail swap applies to the pair GEMM only")
    E, D, F = len(TAIL_COUNTS), 128, 192
    T = sum(TAIL_COUNTS)
    d = dict(synth.random_case(77, T, D, F, E, act=act, dtype="bf16", weight_std=0.05))
    rng = np.random.default_rng(78)
    owner = rng.permutation(np.repeat(np.arange(E), TAIL_COUNTS))
    x = rng.standard_normal((T, D), dtype=np.float32) * np.float32(0.1)
    x[np.arange(T), owner] += np.float32(2.0)
    router = rng.standard_normal((E, D), dtype=np.float32) * np.float32(0.01)
    router[np.arange(E), np.arange(E)] = np.float32(8.0)
    d["x"] = synth.f32_to_bf16_bits(x)
    d["router"] = synth.f32_to_bf16_bits(router)
    g, _ = _full_check(d, E, 1, True, act, "bf16")
    np.testing.assert_array_equal(g["sel"][:, 0], owner)


def test_gather_by_token_when_x_exceeds_l2():
    """x of 64 MB (T=8192, D=4096, bf16) is gathered token by token (each row
    of x read once); every token is checked against the oracle."""
    d = synth.random_case(91, 8192, 4096, 64, 4, dtype="bf16", weight_std=0.02)
    _full_check(d, 4, 2, True, "silu_gated", "bf16")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_norm_topk_prob_off(dtype):
    d = synth.random_case(7, 96, 64, 64, 6, dtype=dtype, weight_std=0.2)
    _full_check(d, 6, 3, False, "silu_gated", dtype)


@pytest.mark.parametrize("gemm_mode", MODES, indirect=True)
def test_all_tokens_to_one_expert(gemm_mode):
    d = dict(synth.random_case(3, 640, 128, 128, 8, dtype="bf16", weight_std=0.05))
    rb = np.zeros(8, dtype=np.float32)
    rb[3] = 30.0
    d["router_bias"] = rb
    g, _ = _full_check(d, 8, 1, True, "silu_gated", "bf16")
    assert (g["sel"] == 3).all()


def test_tie_break_on_device():
    """Identical router rows for experts 0 and 1 give identical fp32 logits;
    the lower index must come first and K=1 never picks expert 1."""
    d = dict(synth.random_case(5, 256, 64, 64, 4, dtype="bf16", weight_std=0.05))
    router = d["router"].copy()
    router[1] = router[0]
    d["router"] = router
    g, _ = _full_check(d, 4, 2, True, "silu_gated", "bf16")
    both = (g["sel"] == 0).any(1) & (g["sel"] == 1).any(1)
    assert both.any()
    for row in g["sel"][both]:
        assert list(row).index(0) < list(row).index(1)
    g1 = PL.run_gpu(PL.to_device(d), 4, 1, True, "silu_gated")
    assert not (g1["sel"] == 1).any()


def test_worked_example_through_the_device():
    """The exercise's two-token example run end to end on the device: x
    picks a column of the router (log-probabilities) and of each expert's
    linear map (the example's expert outputs)."""
    import json
    import os
    gold = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                       "worked_example_two_tokens.json")))
    probs = np.array(gold["probs"])
    eo = np.array(gold["expert_outs"])                   # (T=2, E=3, D=2)
    x = np.eye(2, dtype=np.float32)                      # token t = e_t
    router = np.log(probs).T.astype(np.float32)          # logits of token t = log p[t]
    # ReLU expert with W1 = I, b1 = 0 (h = x >= 0), W2 = [out(x0) out(x1)], b2 = 0
    W1 = np.stack([np.eye(2, dtype=np.float32)] * 3)
    W2 = np.stack([eo[:, e, :].T for e in range(3)]).astype(np.float32)
    d = {"x": x, "router": router, "router_bias": np.zeros(3, np.float32), "gate_up_proj": W1,
         "down_proj": W2, "b1": np.zeros((3, 2), np.float32), "b2": np.zeros((3, 2), np.float32)}
    g = PL.run_gpu(PL.to_device(d), 3, 2, True, "relu")
    assert g["sel"].tolist() == gold["expected_indices"]
    np.testing.assert_allclose(g["out"], gold["expected_out"], atol=gold["atol"], rtol=0)


# ------------------------------------------------------------- properties
@pytest.mark.parametrize("gemm_mode", MODES, indirect=True)
def test_deterministic_bitwise(gemm_mode):
    d = synth.random_case(11, 700, 256, 384, 8, dtype="bf16", weight_std=0.05)
    dev = PL.to_device(d)
    a = PL.run_gpu(dev, 8, 2, True, "silu_gated")
    b = PL.run_gpu(dev, 8, 2, True, "silu_gated")
    for k in ("out", "sel", "w", "logits"):
        np.testing.assert_array_equal(a[k], b[k])


@pytest.mark.parametrize("gemm_mode", MODES, indirect=True)
def test_token_permutation_equivariance_bitwise(gemm_mode):
    d = synth.random_case(12, 500, 256, 256, 8, dtype="bf16", weight_std=0.05)
    perm = np.random.default_rng(0).permutation(500)
    d2 = dict(d)
    d2["x"] = np.ascontiguousarray(d["x"][perm])
    a = PL.run_gpu(PL.to_device(d), 8, 2, True, "silu_gated")
    b = PL.run_gpu(PL.to_device(d2), 8, 2, True, "silu_gated")
    np.testing.assert_array_equal(b["sel"], a["sel"][perm])
    np.testing.assert_array_equal(b["w"], a["w"][perm])
    np.testing.assert_array_equal(b["out"], a["out"][perm])


# ------------------------------------------------------------- router only
@pytest.mark.parametrize("name", [synth.SILU_SMALL.name, synth.DENSE_RELU.name])
def test_route_entry_point(name):
    import torch
    from mixture_experts_ffn_09_b200 import moe
    w = synth.WORKLOADS[name]
    d = synth.make_inputs(w)
    h = PL.host_views(d)
    dev = PL.to_device(d)
    x = dev["x"].reshape(-1, w.D)
    sel = torch.empty(w.T, w.K, dtype=torch.int64, device="cuda")
    wt = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
    lg = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    moe.route(x, dev["router"], w.K, True, sel, wt, dev["router_bias"], lg)
    torch.cuda.synchronize()
    g = {"sel": sel.cpu().numpy(), "w": wt.cpu().numpy().astype(np.float64)}
    r = PL.oracle_route(h, w.K, True)
    PL.check_routing(g, r, w.K, True)
    np.testing.assert_allclose(lg.cpu().numpy(), r["router_logits"], atol=1e-5, rtol=0)


def test_binding_rejects_before_launch():
    import torch
    from mixture_experts_ffn_09_b200 import moe
    d = PL.to_device(synth.random_case(1, 16, 64, 64, 4, dtype="bf16"))
    out = torch.full_like(d["x"], 7.0)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        moe.ffn_forward(d["x"], d["router"], d["gate_up_proj"], d["down_proj"], 4, 5, True, 0, out,
                        workspace=ws)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoEError) as ei:
        moe.ffn_forward(d["x"].double(), d["router"].double(), d["gate_up_proj"].double(),
                        d["down_proj"].double(), 4, 2, True, 0, out.double(), workspace=ws)
    assert ei.value.status == moe.MOE_ERR_DTYPE
    torch.cuda.synchronize()
    assert (out == 7.0).all()     # nothing was launched


def test_bounded_wait_times_out_and_the_context_survives():
    """Failure detection without a fault: a bounded wait on a barrier that
    nothing completes gives up after 50 ms, the device error word reports
    the timeout (and is cleared), and a forward afterwards is correct."""
    import time
    from mixture_experts_ffn_09_b200 import moe
    import torch
    assert moe.device_status() == moe.MOE_OK
    t0 = time.perf_counter()
    moe.debug_bounded_wait(50)
    torch.cuda.synchronize()
    word = moe.device_error_peek()                 # seen without clearing it
    assert word & 1 and "bounded-wait probe" in moe.error_sites(word)
    assert moe.device_status() == moe.MOE_ERR_TIMEOUT
    assert "bounded-wait probe" in moe.last_error()
    assert time.perf_counter() - t0 < 10.0
    assert moe.device_status() == moe.MOE_OK       # the word was cleared
    assert moe.device_error_peek() == 0
    w = synth.SILU_SMALL
    _full_check(synth.make_inputs(w), w.E, w.K, w.norm_topk_prob, w.act, w.dtype)


@pytest.mark.parametrize("gemm_mode", MODES, indirect=True)
@pytest.mark.parametrize("act", ["silu_gated", "relu"])
def test_fused_gather_equals_materialised_rows(gemm_mode, act):
    """gate_up fetching token rows from x by index (TMA gather4) gives the
    bit-identical result of reading an expert-sorted copy of x."""
    from mixture_experts_ffn_09_b200 import moe
    d = synth.random_case(81, 700, 264, 200, 6, act=act, dtype="bf16", weight_std=0.05)
    dev = PL.to_device(d)
    prev = moe.set_fused_gather(False)
    try:
        a = PL.run_gpu(dev, 6, 3, True, act)
        moe.set_fused_gather(True)
        b = PL.run_gpu(dev, 6, 3, True, act)
    finally:
        moe.set_fused_gather(prev)
    for k in ("out", "sel", "w"):
        np.testing.assert_array_equal(a[k], b[k])


@pytest.mark.parametrize("T,E,K,act", [(32, 8, 1, "silu_gated"), (40, 8, 2, "relu"),
                                        (129, 1, 1, "silu_gated"), (300, 2, 1, "relu")])
def test_fused_gather_on_partial_tiles(T, E, K, act):
    """The one-CTA GEMM gathering token rows by index fetches only the rows a
    tile holds (down to one); the rest of the stage is padding.  Off, on and
    the automatic choice (on for these few-row layers, saving the gather
    kernel) agree bit for bit, and all match the oracle."""
    from mixture_experts_ffn_09_b200 import moe
    d = synth.random_case(95 + T, T, 256, 384, E, act=act, dtype="bf16", weight_std=0.05)
    dev = PL.to_device(d)
    prev_mode = moe.set_gemm_mode(moe.GEMM_1SM)
    prev = moe.set_fused_gather("off")
    try:
        g, _ = _full_check(d, E, K, True, act, "bf16")
        res = {}
        for mode in ("off", "on", "auto"):
            moe.set_fused_gather(mode)
            n0 = moe.kernel_launches()
            res[mode] = PL.run_gpu(dev, E, K, True, act)
            res[mode]["launches"] = moe.kernel_launches() - n0
    finally:
        moe.set_fused_gather(prev)
        moe.set_gemm_mode(prev_mode)
    for mode in ("on", "auto"):
        for k in ("out", "sel", "w"):
            np.testing.assert_array_equal(res[mode][k], res["off"][k])
    np.testing.assert_array_equal(res["off"]["out"], g["out"])
    assert res["on"]["launches"] == res["off"]["launches"] - 1          # no gather kernel
    auto_on = T * K <= 16 * E
    assert res["auto"]["launches"] == res["off"]["launches"] - (1 if auto_on else 0)


@pytest.mark.parametrize("gemm_mode", MODES, indirect=True)
def test_programmatic_dependent_launch_changes_nothing(gemm_mode):
    """The kernels give bit-identical results with and without programmatic
    dependent launch, over several forwards in a row on one stream."""
    from mixture_experts_ffn_09_b200 import moe
    d = synth.random_case(91, 900, 256, 384, 8, dtype="bf16", weight_std=0.05)
    dev = PL.to_device(d)
    outs = {}
    for pdl in (False, True):
        prev = moe.set_pdl(pdl)
        try:
            outs[pdl] = [PL.run_gpu(dev, 8, 2, True, "silu_gated") for _ in range(3)]
        finally:
            moe.set_pdl(prev)
    for a, b in zip(outs[False], outs[True]):
        for k in ("out", "sel", "w", "logits"):
            np.testing.assert_array_equal(a[k], b[k])


def test_debug_sync_mode_changes_nothing():
    """With a bounded wait after every kernel the forward returns the same
    bits, and the mode switches back off."""
    from mixture_experts_ffn_09_b200 import moe
    d = synth.random_case(21, 300, 128, 192, 8, dtype="bf16", weight_std=0.05)
    dev = PL.to_device(d)
    a = PL.run_gpu(dev, 8, 2, True, "silu_gated")
    prev = moe.set_debug_sync(5000)
    try:
        b = PL.run_gpu(dev, 8, 2, True, "silu_gated")
    finally:
        assert moe.set_debug_sync(prev) == 5000
    for k in ("out", "sel", "w", "logits"):
        np.testing.assert_array_equal(a[k], b[k])


@pytest.mark.parametrize("gemm_mode", MODES, indirect=True)
def test_forward_replays_from_a_cuda_graph(gemm_mode):
    """The forward makes no synchronising call, so it can be captured into a
    CUDA graph; replays give the eager result bit for bit."""
    import torch
    from mixture_experts_ffn_09_b200 import moe
    d = synth.random_case(22, 640, 256, 384, 8, dtype="bf16", weight_std=0.05)
    dev = PL.to_device(d)
    x = dev["x"]
    T, D = x.shape
    F = dev["down_proj"].shape[-1]
    ws = torch.empty(moe.workspace_size(T, D, F, 8, 2, moe.BF16, moe.ACT_SILU_GATED),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty_like(x)
    sel = torch.empty(T, 2, dtype=torch.int64, device="cuda")
    w = torch.empty(T, 2, dtype=torch.float32, device="cuda")

    def fwd():
        moe.ffn_forward(x, dev["router"], dev["gate_up_proj"], dev["down_proj"], 8, 2, True,
                        moe.ACT_SILU_GATED, out, sel, w, None, None, None, None, ws)

    fwd()                                   # first call sets kernel attributes
    torch.cuda.synchronize()
    ref = (out.clone(), sel.clone(), w.clone())
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fwd()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    for _ in range(3):
        out.zero_()
        sel.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref[0]) and torch.equal(sel, ref[1]) and torch.equal(w, ref[2])
    assert moe.device_status() == moe.MOE_OK


@pytest.mark.parametrize("name", [synth.DENSE_RELU.name, synth.SILU_SMALL.name])
def test_small_layer_replays_from_a_cuda_graph(name):
    """The one-kernel small layer, captured once after a first call (which
    sets the kernel attributes and picks the cluster size), replays from a
    CUDA graph with the eager result bit for bit."""
    import torch
    from mixture_experts_ffn_09_b200 import moe
    w = synth.WORKLOADS[name]
    dev = PL.to_device(synth.make_inputs(w))
    x = dev["x"].reshape(w.T, w.D)
    a = moe.ACT_NAMES[w.act]
    ws = torch.empty(moe.workspace_size(w.T, w.D, w.F, w.E, w.K, moe.F32, a), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty_like(x)
    sel = torch.empty(w.T, w.K, dtype=torch.int64, device="cuda")
    wt = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")

    def fwd():
        moe.ffn_forward(x, dev["router"], dev["gate_up_proj"], dev["down_proj"], w.E, w.K, True, a,
                        out, sel, wt, dev["router_bias"], dev["b1"], dev["b2"], None, ws)

    fwd()
    torch.cuda.synchronize()
    ref = (out.clone(), sel.clone(), wt.clone())
    g = torch.cuda.CUDAGraph()
    n0 = moe.kernel_launches()
    with torch.cuda.graph(g):
        fwd()
    assert moe.kernel_launches() - n0 == 1
    for _ in range(3):
        out.zero_()
        sel.zero_()
        wt.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref[0]) and torch.equal(sel, ref[1]) and torch.equal(wt, ref[2])
    assert moe.device_status() == moe.MOE_OK


def test_kernel_launch_count_per_forward():
    """A forward launches router, scatter, gather, gate_up, down and combine;
    the scan kernel only runs for block-count tables of more than 4096
    entries, and the capacity clamp and the balance finaliser add one each."""
    import torch
    from mixture_experts_ffn_09_b200 import moe

    def launches(T, E, **opts):
        d = synth.random_case(23, T, 64, 64, E, dtype="bf16", weight_std=0.05)
        dev = PL.to_device(d)
        x = dev["x"]
        ws = torch.empty(moe.workspace_size(T, 64, 64, E, 2, moe.BF16), dtype=torch.uint8,
                         device="cuda")
        out = torch.empty_like(x)
        sel = torch.empty(T, 2, dtype=torch.int64, device="cuda")
        w = torch.empty(T, 2, dtype=torch.float32, device="cuda")
        n0 = moe.kernel_launches()
        moe.ffn_forward_ex(x, dev["router"], dev["gate_up_proj"], dev["down_proj"], E, 2, True,
                           moe.ACT_SILU_GATED, out, sel, w, None, None, None, None, ws, **opts)
        n = moe.kernel_launches() - n0
        assert moe.device_status() == moe.MOE_OK
        return n

    assert launches(256, 8) == 6                     # 8 blocks x 8 experts: scanned in scatter
    assert launches(4096, 64) == 7                   # 128 x 64 entries: the scan kernel runs
    bal = torch.empty(4, dtype=torch.float32, device="cuda")
    assert launches(256, 8, capacity_factor=1.0, balance=bal) == 8


@pytest.mark.parametrize("name", [synth.DENSE_RELU.name, synth.SILU_SMALL.name, "random"])
def test_small_float32_layer_runs_as_one_kernel(name):
    """A small float32 layer (E <= 8, T*K <= 256, no routing options) runs
    as one clustered kernel; asking for slot_kept sends the same layer down
    the general six-kernel path.  Both match the oracle, and each other."""
    import torch
    from mixture_experts_ffn_09_b200 import moe
    if name == "random":
        d, E, K, act = synth.random_case(91, 37, 24, 40, 5, dtype="f32", weight_std=0.3), 5, 3, "silu_gated"
    else:
        w = synth.WORKLOADS[name]
        d, E, K, act = synth.make_inputs(w), w.E, w.K, w.act
    h = PL.host_views(d)
    dev = PL.to_device(d)
    x = dev["x"].reshape(-1, dev["x"].shape[-1])
    T, D = x.shape
    F = dev["down_proj"].shape[-1]
    a = moe.ACT_NAMES[act]
    ws = torch.empty(moe.workspace_size(T, D, F, E, K, moe.F32, a), dtype=torch.uint8, device="cuda")
    res = []
    for general in (False, True):
        out = torch.empty_like(x)
        sel = torch.empty(T, K, dtype=torch.int64, device="cuda")
        wt = torch.empty(T, K, dtype=torch.float32, device="cuda")
        kept = torch.empty(T, K, dtype=torch.uint8, device="cuda")
        n0 = moe.kernel_launches()
        moe.ffn_forward_ex(x, dev["router"], dev["gate_up_proj"], dev["down_proj"], E, K, True, a,
                           out, sel, wt, dev["router_bias"], dev["b1"], dev["b2"], None, ws,
                           **({"slot_kept": kept} if general else {}))
        n = moe.kernel_launches() - n0
        assert moe.device_status() == moe.MOE_OK
        assert n == (6 if general else 1)
        res.append({"out": out.cpu().numpy().astype(np.float64), "sel": sel.cpu().numpy(),
                    "w": wt.cpu().numpy().astype(np.float64)})
    r = O.moe_route(h["x"].reshape(T, D), h["router"], K, True, h["router_bias"])
    for g in res:
        clear = PL.check_routing(g, r, K, True)
        ref = O.moe_ffn_forward(h["x"].reshape(T, D), h["router"], h["gate_up_proj"], h["down_proj"],
                                K, True, act, h["router_bias"], h["b1"], h["b2"])["out"]
        if (~clear).any():
            un = np.nonzero(~clear)[0]
            ref[un] = PL.oracle_out_for(h, un, g["sel"][un], K, True, act)
        PL.check_out(g["out"], ref, "f32")
    same = (res[0]["sel"] == res[1]["sel"]).all(1)
    assert same.mean() > 0.95
    PL.check_out(res[0]["out"][same], res[1]["out"][same], "f32", "one kernel vs six")


def _skewed_small(seed, T, D, F, E, act, hot):
    """A small fp32 case whose router sends every token's first choice to
    expert `hot` (a large router bias), the rest by the logits."""
    d = dict(synth.random_case(seed, T, D, F, E, act=act, dtype="f32", weight_std=0.3))
    rb = np.zeros(E, dtype=np.float32) if d["router_bias"] is None else d["router_bias"].copy()
    rb[hot] += np.float32(40.0)
    d["router_bias"] = rb
    return d


SMALL_SPLIT_CASES = [
    # (seed, T, D, F, E, K, act, skew)
    (61, 64, 64, 128, 8, 2, "silu_gated", True),     # one expert takes every token
    (62, 64, 32, 64, 4, 2, "relu", True),
    (63, 1, 64, 128, 8, 2, "silu_gated", False),     # a single token
    (64, 32, 16, 32, 8, 8, "silu_gated", False),     # K = E: every expert, T*K = 256
    (65, 256, 16, 24, 3, 1, "relu", True),           # T*K = 256 on one expert
    (66, 40, 33, 47, 5, 2, "silu_gated", False),     # D, F not multiples of 4: 4-byte copies
    (67, 50, 8, 4, 2, 1, "silu_gated", True),        # F = 4: one column group, no split
    (68, 20, 12, 10, 1, 1, "relu", False),           # E = 1
    (69, 10, 3, 5, 3, 2, "relu", False),             # D = 3: one lane holds all of D
    (70, 16, 8, 1, 4, 2, "silu_gated", True),        # F = 1: a single column, never split
]


@pytest.mark.parametrize("cluster", [8, 16])
@pytest.mark.parametrize("seed,T,D,F,E,K,act,skew", SMALL_SPLIT_CASES)
def test_small_layer_split_over_the_cluster(seed, T, D, F, E, K, act, skew, cluster):
    """The one-kernel small layer splits each expert's hidden columns over
    CTAs in proportion to its rows.  Skewed routing (one expert with every
    token), a single token, K = E, column counts that do not split into
    4-column groups evenly or at all, and one expert: every token against
    the oracle, with clusters of 8 and of 16 CTAs, in one launch each."""
    from mixture_experts_ffn_09_b200 import moe
    d = _skewed_small(seed, T, D, F, E, act, seed % E) if skew else \
        synth.random_case(seed, T, D, F, E, act=act, dtype="f32", weight_std=0.3)
    prev = moe.set_small_cluster(cluster)
    try:
        n0 = moe.kernel_launches()
        g, _ = _full_check(d, E, K, True, act, "f32")
        assert moe.kernel_launches() - n0 == 1
    finally:
        moe.set_small_cluster(prev)
    if skew:
        assert (g["sel"][:, 0] == seed % E).all()


def _random_small_layers(n, seed):
    """Seeded small fp32 layers inside the one-kernel limits (E <= 8,
    T*K <= 256, widths up to 48 so that the shared memory of any such layer
    stays within the kernel's 200 KB), multiples of 4 or not."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        E = int(rng.integers(1, 9))
        K = int(rng.integers(1, E + 1))
        T = int(rng.integers(1, 256 // K + 1))
        D = int(rng.integers(1, 49))
        F = int(rng.integers(1, 49))
        act = "relu" if rng.random() < 0.4 else "silu_gated"
        skew = bool(rng.random() < 0.3)
        out.append((T, D, F, E, K, act, skew))
    return out


@pytest.mark.parametrize("cluster", [8, 16])
@pytest.mark.parametrize("T,D,F,E,K,act,skew", _random_small_layers(10, 4242))
def test_small_layer_random_sweep(T, D, F, E, K, act, skew, cluster):
    """Seeded random small fp32 layers through the one-kernel path, with
    clusters of 8 and 16 CTAs: every token against the oracle, one launch."""
    from mixture_experts_ffn_09_b200 import moe
    seed = 7000 + T + D + F + E
    d = _skewed_small(seed, T, D, F, E, act, seed % E) if skew else \
        synth.random_case(seed, T, D, F, E, act=act, dtype="f32", weight_std=0.3)
    prev = moe.set_small_cluster(cluster)
    try:
        n0 = moe.kernel_launches()
        _full_check(d, E, K, True, act, "f32")
        assert moe.kernel_launches() - n0 == 1
    finally:
        moe.set_small_cluster(prev)


@pytest.mark.parametrize("act", ["silu_gated", "relu"])
def test_split_last_wave(act):
    """Layers in the CTA-pair regime run their last wave as k-halves: the
    first half of a tile hands its fp32 accumulator to the second.  Here every
    tile is split (18 tiles, fewer than the pairs), the experts end in swapped
    tails, and every token is compared with the oracle; the result repeats
    bit for bit and equals the fused-gather variant's."""
    from mixture_experts_ffn_09_b200 import moe
    T, D, F, E, K = 1200, 256, 384, 2, 1       # 1200 routed rows >= 512 per expert
    d = synth.random_case(501, T, D, F, E, act=act, dtype="bf16", weight_std=0.05)
    g, _ = _full_check(d, E, K, True, act, "bf16")
    load = np.bincount(g["sel"].ravel(), minlength=E)
    assert (load % 256 > 0).all() and (load % 256 <= 128).any()   # a swapped tail
    dev = PL.to_device(d)
    a = PL.run_gpu(dev, E, K, True, act)
    b = PL.run_gpu(dev, E, K, True, act)
    prev = moe.set_fused_gather(True)
    try:
        c = PL.run_gpu(dev, E, K, True, act)
    finally:
        moe.set_fused_gather(prev)
    for k in ("out", "sel", "w"):
        np.testing.assert_array_equal(a[k], b[k])
        np.testing.assert_array_equal(a[k], c[k])
        np.testing.assert_array_equal(a[k], g[k])


def _random_shapes(n, seed):
    """Seeded layer shapes across the supported ranges: bf16 needs D and F
    multiples of 8, any sizes on float32."""
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        dtype = "bf16" if i % 3 else "f32"
        step = 8 if dtype == "bf16" else 1
        T = int(rng.integers(1, 700))
        D = int(rng.integers(1, 64)) * step
        F = int(rng.integers(1, 64)) * step
        E = int(rng.integers(1, 80))
        K = int(rng.integers(1, min(E, 10) + 1))
        act = "relu" if rng.random() < 0.3 else "silu_gated"
        out.append((T, D, F, E, K, act, dtype, int(rng.integers(1, 3))))
    return out


@pytest.mark.parametrize("tail_swap", [32, 128], indirect=True)
@pytest.mark.parametrize("T,D,F,E,K,act,dtype,mode", _random_shapes(12, 2026))
def test_random_shapes_sweep(T, D, F, E, K, act, dtype, mode, tail_swap):
    """Seeded random layers (token count, widths, expert count, top-k,
    activation, dtype, GEMM variant, tail swap): every token against the
    oracle."""
    from mixture_experts_ffn_09_b200 import moe
    if (mode == 1 or dtype == "f32") and tail_swap != 128:
        pytest.skip("the tail swap applies to the bf16 pair GEMM only")
    prev = moe.set_gemm_mode(mode)
    try:
        d = synth.random_case(3000 + T + E, T, D, F, E, act=act, dtype=dtype,
                              weight_std=0.3 if dtype == "f32" else 0.05)
        _full_check(d, E, K, True, act, dtype)
    finally:
        moe.set_gemm_mode(prev)
