"""The no-allocation forward, moe_ffn_forward_noalloc.

Some callers cannot allocate device memory at the moment they run the layer
(a plugin or callback inside another runtime that owns all device memory and
hands over only the tensors to read and write).  For them the library has
one more entry point that takes no workspace and uses a static scratch array
inside the library instead.  These tests run it through the C ABI and check
that it gives the ordinary entry point's results, on consecutive calls with
different shapes (the scratch keeps the previous call's contents), and that
sizes beyond the scratch are refused before anything runs.

This file is collected last on purpose, so a run that stops at the first
failure has run every other test before it.
"""
import numpy as np
import pytest

from mixture_experts_ffn_09_b200 import moe, synth

import parity_lib as PL


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixture_experts_ffn_09_b200 import build
    build.build()


def _both(d, E, K, act, dtype):
    import torch
    dev = PL.to_device(d)
    x = dev["x"]
    T, D = x.shape
    F = dev["down_proj"].shape[-1]
    code = moe.BF16 if dtype == "bf16" else moe.F32
    a = moe.ACT_NAMES[act]
    assert moe.workspace_size(T, D, F, E, K, code, a) <= moe.noalloc_scratch_bytes()
    res = []
    for noalloc in (False, True):
        out = torch.empty_like(x)
        sel = torch.empty(T, K, dtype=torch.int64, device="cuda")
        w = torch.empty(T, K, dtype=torch.float32, device="cuda")
        args = (x, dev["router"], dev["gate_up_proj"], dev["down_proj"], E, K, True, a, out, sel, w,
                dev["router_bias"], dev["b1"], dev["b2"])
        if noalloc:
            moe.ffn_forward_noalloc(*args)
        else:
            ws = torch.empty(moe.workspace_size(T, D, F, E, K, code, a), dtype=torch.uint8,
                             device="cuda")
            moe.ffn_forward(*args, None, ws)
        assert moe.device_status() == moe.MOE_OK
        res.append((out.float().cpu().numpy().astype(np.float64), sel.cpu().numpy(),
                    w.cpu().numpy()))
    (o_ref, s_ref, w_ref), (o, s, w) = res
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_allclose(w, w_ref, atol=1e-6, rtol=0)
    PL.check_out(o, o_ref, dtype, "no-allocation forward vs workspace forward")
    return s


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_forward_on_consecutive_calls():
    a = synth.random_case(41, 96, 512, 1024, 8, dtype="bf16", weight_std=0.05)
    b = synth.random_case(42, 300, 136, 200, 5, act="relu", dtype="bf16", weight_std=0.05)
    c = synth.random_case(43, 100, 33, 47, 6, dtype="f32", weight_std=0.3)
    _both(a, 8, 2, "silu_gated", "bf16")
    _both(b, 5, 2, "relu", "bf16")      # second call: other shapes over stale scratch
    _both(c, 6, 3, "silu_gated", "f32")
    _both(a, 8, 2, "silu_gated", "bf16")


def test_noalloc_refuses_sizes_beyond_its_scratch():
    # Rejected on the host before any device work; the pointers are never used.
    L = moe.lib()
    P = 0x10000
    st = L.moe_ffn_forward_noalloc(P, P, P, P, 8, 2, 1, 0, P, None, None, 4096, 4096, 14336,
                                   moe.BF16, None, None, None, None, None)
    assert st == moe.MOE_ERR_WORKSPACE
    assert "static scratch" in moe.last_error()
    st = L.moe_ffn_forward_noalloc(P, P, P, P, 8, 9, 1, 0, P, None, None, 32, 64, 64, moe.BF16,
                                   None, None, None, None, None)
    assert st == moe.MOE_ERR_INVALID_ARG


@pytest.mark.gpu
def test_noalloc_on_the_cta_pair_gemm():
    """The CTA-pair GEMM over the shared scratch: its short expert tails run
    with swapped operands (extra token views over the expert-sorted rows),
    longer tails as padded 256-row tiles whose pad rows hold whatever the
    previous call left there.  Both kinds, after calls with other shapes."""
    prev = moe.set_gemm_mode(moe.GEMM_2SM)
    try:
        long_tails = synth.random_case(44, 900, 512, 1024, 2, dtype="bf16", weight_std=0.05)
        short_tails = synth.random_case(45, 600, 256, 384, 6, dtype="bf16", weight_std=0.05)
        tails = []
        for d, E in ((long_tails, 2), (short_tails, 6), (long_tails, 2)):
            sel = _both(d, E, 1, "silu_gated", "bf16")
            rows = np.bincount(sel.ravel(), minlength=E)
            tails += [int(r) % 256 for r in rows if r % 256]
        assert any(1 <= t <= 128 for t in tails), tails      # swapped
        assert any(129 <= t <= 255 for t in tails), tails    # padded full tile
    finally:
        moe.set_gemm_mode(prev)


def test_noalloc_scratch_size_edge():
    """The scratch size the binding reports is the one the library enforces:
    the largest layer of this shape whose workspace fits gets past the size
    check, one token more is refused.  The pointers are misaligned on purpose,
    so a call that passes the size check is rejected on the host before any
    launch (MOE_ERR_ALIGNMENT; MOE_ERR_CUDA where no GPU is present)."""
    L = moe.lib()
    lim = moe.noalloc_scratch_bytes()
    D, F, E, K = 32, 32, 4, 1
    lo, hi = 1, 1 << 20                       # workspace(lo) <= lim < workspace(hi)
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if moe.workspace_size(mid, D, F, E, K, moe.BF16) <= lim:
            lo = mid
        else:
            hi = mid
    assert lim - moe.workspace_size(lo, D, F, E, K, moe.BF16) <= 8192
    P = 0x10001
    for T, refused in ((lo, False), (hi, True)):
        st = L.moe_ffn_forward_noalloc(P, P, P, P, E, K, 1, 0, P, None, None, T, D, F, moe.BF16,
                                       None, None, None, None, None)
        if refused:
            assert st == moe.MOE_ERR_WORKSPACE and "static scratch" in moe.last_error()
        else:
            assert st in (moe.MOE_ERR_ALIGNMENT, moe.MOE_ERR_CUDA, moe.MOE_ERR_DEVICE), st


def test_noalloc_rejects_a_non_contiguous_x():
    """A strided view of x would reach the C ABI as if it were a dense
    (T, D) matrix; the binding refuses it, as it does for the ordinary
    entry point."""
    import torch
    T, D, F, E, K = 8, 64, 32, 4, 2
    x = torch.zeros(T, 2 * D, dtype=torch.float32)[:, ::2]
    assert x.shape == (T, D) and not x.is_contiguous()
    router = torch.zeros(E, D)
    gu = torch.zeros(E, 2 * F, D)
    dn = torch.zeros(E, D, F)
    out = torch.zeros(T, D)
    for fn in (moe.ffn_forward_noalloc, moe.ffn_forward):
        with pytest.raises(ValueError, match="^x must be contiguous"):
            fn(x, router, gu, dn, E, K, True, "silu_gated", out)
