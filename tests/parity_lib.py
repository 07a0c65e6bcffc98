"""Shared helpers of the GPU parity tests: upload synthetic inputs, run the
CUDA path through the C ABI, run the oracle on the same inputs, compare.

Comparison rule (the selection is unique only up to rounding):

* selected_experts must equal the oracle's bit for bit on every token whose
  oracle K-th vs (K+1)-th probability gap exceeds 1e-5;
* on the other tokens the GPU's selection must be a valid top-K up to that
  gap (each kept expert's oracle probability within 1e-5 of the K-th), and
  the GPU's output is compared with the oracle evaluated on the GPU's
  selection (several selections are correct there);
* out: max |gpu - ref| <= tol * max |ref| with tol = 1e-4 (fp32 path) or
  2e-2 (bf16 path, fp32 accumulation).
"""
from __future__ import annotations

import numpy as np

from mixture_experts_ffn_09_b200 import synth

GAP = 1e-5
TOL = {"f32": 1e-4, "bf16": 2e-2}


class Bf16Experts:
    """Indexable float32 view of a bf16 (uint16 bits) weight stack, widened
    one expert at a time (keeps host memory bounded)."""

    def __init__(self, bits):
        self.bits = bits
        self.shape = bits.shape

    def __getitem__(self, e):
        return synth.bf16_bits_to_f32(self.bits[e])


def host_views(d: dict) -> dict:
    """Float views of the generator's arrays for the oracle."""
    out = {}
    for k, v in d.items():
        if v is None:
            out[k] = None
        elif v.dtype == np.uint16:
            out[k] = Bf16Experts(v) if k in ("gate_up_proj", "down_proj") else synth.bf16_bits_to_f32(v)
        else:
            out[k] = v
    return out


def to_device(d: dict, device="cuda"):
    """Device copies of the generator's (read-only) arrays; the host views
    are only read, so torch's warning about non-writable arrays is muted."""
    import warnings
    import torch
    out = {}
    with warnings.catch_warnings():
        warnings.filterwarnings("ignore", message="The given NumPy array is not writable")
        for k, v in d.items():
            if v is None:
                out[k] = None
            elif v.dtype == np.uint16:
                out[k] = torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).view(torch.bfloat16).to(device)
            else:
                out[k] = torch.from_numpy(np.ascontiguousarray(v)).to(device)
    return out


def run_gpu(dev: dict, E: int, K: int, norm: bool, act: str, with_logits: bool = True):
    """One forward through the C ABI; returns numpy out (float64), sel, w,
    logits."""
    import torch
    from mixture_experts_ffn_09_b200 import moe
    x = dev["x"]
    D = x.shape[-1]
    T = x.numel() // D
    F = dev["down_proj"].shape[-1]
    dt = moe.BF16 if x.dtype == torch.bfloat16 else moe.F32
    a = moe.ACT_NAMES[act]
    ws = torch.empty(moe.workspace_size(T, D, F, E, K, dt, a), dtype=torch.uint8, device=x.device)
    out = torch.empty_like(x)
    sel = torch.full((T, K), -1, dtype=torch.int64, device=x.device)
    w = torch.full((T, K), float("nan"), dtype=torch.float32, device=x.device)
    lg = torch.empty(T, E, dtype=torch.float32, device=x.device) if with_logits else None
    moe.ffn_forward(x, dev["router"], dev["gate_up_proj"], dev["down_proj"], E, K, norm, a, out,
                    sel, w, dev.get("router_bias"), dev.get("b1"), dev.get("b2"), lg, ws)
    assert moe.device_status() == moe.MOE_OK
    return {"out": out.float().cpu().numpy().astype(np.float64).reshape(T, D),
            "sel": sel.cpu().numpy(), "w": w.cpu().numpy().astype(np.float64),
            "logits": None if lg is None else lg.cpu().numpy().astype(np.float64)}


def oracle_route(h: dict, K: int, norm: bool):
    from oracle import moe_oracle as O
    x = h["x"].reshape(-1, h["x"].shape[-1])
    return O.moe_route(x, h["router"], K, norm, h["router_bias"])


def check_routing(g: dict, r: dict, K: int, norm: bool, tol_w: float = 1e-5):
    """Selections exact where the gap is clear, valid elsewhere; weights
    close.  Returns the boolean mask of clear tokens."""
    clear = r["gap"] > GAP
    np.testing.assert_array_equal(g["sel"][clear], r["selected_experts"][clear])
    p = r["probs"]
    T = p.shape[0]
    kth = np.sort(p, axis=1)[:, ::-1][:, K - 1]
    for t in np.nonzero(~clear)[0]:
        s = g["sel"][t]
        assert len(set(s.tolist())) == K and (s >= 0).all() and (s < p.shape[1]).all()
        assert (p[t, s] >= kth[t] - GAP).all()
    w_ref = np.take_along_axis(p, g["sel"], 1)
    if norm:
        w_ref = w_ref / (w_ref.sum(1, keepdims=True) + 1e-9)
    np.testing.assert_allclose(g["w"], w_ref, atol=tol_w, rtol=0)
    return clear


def check_out(g_out, ref_out, dtype: str, what: str = "out"):
    tol = TOL[dtype]
    scale = np.abs(ref_out).max()
    err = np.abs(g_out - ref_out).max()
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:g} * max|ref| {scale:.3e}"
    return err / scale


def oracle_out_for(h: dict, tokens, sel, K: int, norm: bool, act: str):
    """Oracle output of the given tokens under a given selection (the
    oracle's own weights for that selection)."""
    from oracle import moe_oracle as O
    x = h["x"].reshape(-1, h["x"].shape[-1])[tokens]
    r = O.moe_route(x, h["router"], K, norm, h["router_bias"])
    p = r["probs"]
    v = np.take_along_axis(p, sel, 1)
    w = O.routing_weights(v, norm)
    return O.moe_ffn_given_routing(x, sel, w, h["gate_up_proj"], h["down_proj"], act, h["b1"], h["b2"])


def tail_tokens(sel: np.ndarray, E: int) -> dict:
    """Tokens whose rows sit in each expert's last row blocks.

    The permutation sorts an expert's rows by token index, so the expert's
    last rows belong to its highest-index tokens.  For every expert this
    returns the token of its last row, and the first token of its last
    128-row and last 256-row block (the one-CTA and CTA-pair tiles: a pair
    GEMM's short last block runs with swapped operands).  Keyed by expert."""
    out = {}
    for e in range(E):
        toks = np.nonzero((sel == e).any(1))[0]
        n = len(toks)
        if n:
            out[e] = sorted({int(toks[-1]), int(toks[(n - 1) // 128 * 128]),
                             int(toks[(n - 1) // 256 * 256])})
    return out


def sample_tokens(sel_ref: np.ndarray, E: int, n: int, seed: int = 0, tails=None) -> np.ndarray:
    """A seeded token subset that covers every expert selected anywhere,
    plus the first and last token and the given tail tokens (see
    tail_tokens), topped up at random to n tokens."""
    rng = np.random.default_rng(seed)
    T = sel_ref.shape[0]
    order = rng.permutation(T)
    chosen = {0, T - 1}
    for e in range(E):
        hit = order[(sel_ref[order] == e).any(1)]
        if len(hit):
            chosen.add(int(hit[0]))
    for toks in (tails or {}).values():
        chosen.update(toks)
    for t in order:
        if len(chosen) >= n:
            break
        chosen.add(int(t))
    return np.array(sorted(chosen))
