"""Thin ctypes binding of libmoe (include/moe.h).

Argument marshalling only: every step of the forward runs in the CUDA
kernels of ``libmoe.so``.  torch is used for device memory and streams.
There is no fallback: if the library is missing, every call raises.

The functions keep the C names without the ``moe_`` prefix:

* :func:`ffn_forward`   - moe_ffn_forward (router, permutation, grouped GEMMs,
  combine), on caller-provided torch tensors;
* :func:`route`         - moe_route (router only);
* :func:`workspace_size`, :func:`device_status`, :func:`profile_enable`,
  :func:`profile_read`, :func:`status_string`, :func:`abi_version`.

:class:`MoEBlock` mirrors the interface of mojolearn.MoEBlock (forward,
load_state_dict, router_logits_, selected_experts_, routing_weights_) on
top of these calls.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED_ACT = 2
MOE_ERR_DTYPE = 3
MOE_ERR_SHAPE = 4
MOE_ERR_ALIGNMENT = 5
MOE_ERR_WORKSPACE = 6
MOE_ERR_CUDA = 7
MOE_ERR_TIMEOUT = 8
MOE_ERR_DEVICE = 9

ACT_SILU_GATED = 0
ACT_RELU = 1
ACT_NAMES = {"silu_gated": ACT_SILU_GATED, "silu": ACT_SILU_GATED, "relu": ACT_RELU}

F32 = 0
BF16 = 1
F64 = 2
NUM_STAGES = 6

SCORE_SOFTMAX = 0
SCORE_SIGMOID = 1
SCORE_NAMES = {"softmax": SCORE_SOFTMAX, "sigmoid": SCORE_SIGMOID}

_lock = threading.Lock()
_lib = None


class RouteOpts(ctypes.Structure):
    """moe_route_opts_t (include/moe.h)."""
    _fields_ = [("score", ctypes.c_int), ("selection_bias", ctypes.c_void_p),
                ("dynamic_threshold", ctypes.c_float), ("capacity_factor", ctypes.c_float),
                ("seq_len", ctypes.c_int64), ("slot_kept", ctypes.c_void_p),
                ("balance", ctypes.c_void_p)]


class MoEError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"libmoe status {status} ({status_string(status)}): {detail}")


def lib() -> ctypes.CDLL:
    """Loads libmoe.so (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with `python -m mixture_experts_ffn_09_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.moe_ffn_workspace_size.argtypes = [i64, i64, i64, i32, i32, i32, i32]
        L.moe_ffn_workspace_size.restype = sz
        L.moe_ffn_forward.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, i64, i64, i64,
                                      i32, vp, vp, vp, vp, vp, sz, vp]
        L.moe_ffn_forward.restype = i32
        L.moe_ffn_forward_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, i64,
                                              i64, i64, i32, vp, vp, vp, vp, vp]
        L.moe_ffn_forward_noalloc.restype = i32
        L.moe_ffn_forward_ex.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, i64, i64,
                                         i64, i32, vp, vp, vp, vp, vp, sz,
                                         ctypes.POINTER(RouteOpts), vp]
        L.moe_ffn_forward_ex.restype = i32
        L.moe_route_ex.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, i32, vp, vp, vp,
                                   ctypes.POINTER(RouteOpts), vp]
        L.moe_route_ex.restype = i32
        L.moe_route.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, i32, vp, vp, vp, vp]
        L.moe_route.restype = i32
        L.moe_status_string.argtypes = [i32]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_last_error.argtypes = []
        L.moe_last_error.restype = ctypes.c_char_p
        L.moe_abi_version.argtypes = []
        L.moe_abi_version.restype = i32
        L.moe_device_status.argtypes = [vp]
        L.moe_device_status.restype = i32
        L.moe_device_error_peek.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        L.moe_device_error_peek.restype = i32
        L.moe_kernel_launches.argtypes = []
        L.moe_kernel_launches.restype = ctypes.c_ulonglong
        L.moe_error_sites.argtypes = [ctypes.c_uint]
        L.moe_error_sites.restype = ctypes.c_char_p
        L.moe_profile_enable.argtypes = [i32]
        L.moe_profile_enable.restype = i32
        L.moe_profile_read.argtypes = [ctypes.POINTER(ctypes.c_float), i32]
        L.moe_profile_read.restype = i32
        L.moe_debug_bounded_wait.argtypes = [i32, vp]
        L.moe_debug_bounded_wait.restype = i32
        L.moe_set_pdl.argtypes = [i32]
        L.moe_set_pdl.restype = i32
        L.moe_set_debug_sync.argtypes = [i32]
        L.moe_set_debug_sync.restype = i32
        L.moe_set_fused_gather.argtypes = [i32]
        L.moe_set_fused_gather.restype = i32
        L.moe_set_gemm_mode.argtypes = [i32]
        L.moe_set_gemm_mode.restype = i32
        L.moe_set_small_cluster.argtypes = [i32]
        L.moe_set_small_cluster.restype = i32
        L.moe_stage_name.argtypes = [i32]
        L.moe_stage_name.restype = ctypes.c_char_p
        _lib = L
        return L


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def last_error() -> str:
    return lib().moe_last_error().decode()


def abi_version() -> int:
    return int(lib().moe_abi_version())


def _check(status: int) -> None:
    if status != MOE_OK:
        raise MoEError(status, last_error())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float64:
        return F64
    return -1


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _act_code(act) -> int:
    if isinstance(act, str):
        if act not in ACT_NAMES:
            return 99
        return ACT_NAMES[act]
    return int(act)


def workspace_size(T: int, D: int, F: int, E: int, K: int, dtype: int, act=ACT_SILU_GATED) -> int:
    return int(lib().moe_ffn_workspace_size(T, D, F, E, K, dtype, _act_code(act)))


def _expect(t, shape, name, dtype=None, required=True):
    """Shape / dtype / device / contiguity checks of one tensor argument."""
    if t is None:
        if required:
            raise ValueError(f"{name} is required")
        return
    if isinstance(t, int):
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def ffn_forward(x, router, gate_up_proj, down_proj, E: int, K: int, norm_topk_prob: bool, act,
                out, selected_experts=None, routing_weights=None, router_bias=None, b1=None,
                b2=None, router_logits=None, workspace=None, stream=None) -> None:
    """moe_ffn_forward on torch tensors.  x (..., D); out like x."""
    import torch
    D = int(x.shape[-1])
    T = int(x.numel() // D) if D else 0
    F = int(down_proj.shape[-1])
    dt = _dtype_code(x)
    a = _act_code(act)
    if dt in (F32, BF16) and a in (ACT_SILU_GATED, ACT_RELU) and 1 <= K <= E and T > 0:
        wdt = x.dtype
        gu_rows = 2 * F if a == ACT_SILU_GATED else F
        _expect(x, tuple(x.shape), "x", wdt)
        _expect(router, (E, D), "router", wdt)
        _expect(gate_up_proj, (E, gu_rows, D), "gate_up_proj", wdt)
        _expect(down_proj, (E, D, F), "down_proj", wdt)
        _expect(out, tuple(x.shape), "out", wdt)
        _expect(selected_experts, (T, K), "selected_experts", torch.int64, False)
        _expect(routing_weights, (T, K), "routing_weights", torch.float32, False)
        _expect(router_bias, (E,), "router_bias", torch.float32, False)
        _expect(b1, (E, F), "b1", torch.float32, False)
        _expect(b2, (E, D), "b2", torch.float32, False)
        _expect(router_logits, (T, E), "router_logits", torch.float32, False)
    ws_bytes = 0
    if workspace is not None and not isinstance(workspace, int):
        ws_bytes = workspace.numel() * workspace.element_size()
    elif isinstance(workspace, int):
        raise ValueError("pass the workspace as a tensor")
    st = lib().moe_ffn_forward(
        _ptr(x), _ptr(router), _ptr(gate_up_proj), _ptr(down_proj), E, K, int(bool(norm_topk_prob)),
        a, _ptr(out), _ptr(selected_experts), _ptr(routing_weights), T, D, F, dt,
        _ptr(router_bias), _ptr(b1), _ptr(b2), _ptr(router_logits), _ptr(workspace), ws_bytes,
        _stream(stream))
    _check(st)


def ffn_forward_noalloc(x, router, gate_up_proj, down_proj, E: int, K: int, norm_topk_prob: bool,
                        act, out, selected_experts=None, routing_weights=None, router_bias=None,
                        b1=None, b2=None, router_logits=None, stream=None) -> None:
    """moe_ffn_forward_noalloc: the same forward without a workspace, for
    callers that cannot allocate device memory when they run the layer (the
    library's static scratch of noalloc_scratch_bytes() is used instead)."""
    import torch
    D = int(x.shape[-1])
    T = int(x.numel() // D) if D else 0
    F = int(down_proj.shape[-1])
    dt = _dtype_code(x)
    a = _act_code(act)
    if dt in (F32, BF16) and a in (ACT_SILU_GATED, ACT_RELU) and 1 <= K <= E and T > 0:
        wdt = x.dtype
        gu_rows = 2 * F if a == ACT_SILU_GATED else F
        _expect(x, tuple(x.shape), "x", wdt)
        _expect(router, (E, D), "router", wdt)
        _expect(gate_up_proj, (E, gu_rows, D), "gate_up_proj", wdt)
        _expect(down_proj, (E, D, F), "down_proj", wdt)
        _expect(out, tuple(x.shape), "out", wdt)
        _expect(selected_experts, (T, K), "selected_experts", torch.int64, False)
        _expect(routing_weights, (T, K), "routing_weights", torch.float32, False)
        _expect(router_bias, (E,), "router_bias", torch.float32, False)
        _expect(b1, (E, F), "b1", torch.float32, False)
        _expect(b2, (E, D), "b2", torch.float32, False)
        _expect(router_logits, (T, E), "router_logits", torch.float32, False)
    st = lib().moe_ffn_forward_noalloc(
        _ptr(x), _ptr(router), _ptr(gate_up_proj), _ptr(down_proj), E, K, int(bool(norm_topk_prob)),
        a, _ptr(out), _ptr(selected_experts), _ptr(routing_weights), T, D, F, dt,
        _ptr(router_bias), _ptr(b1), _ptr(b2), _ptr(router_logits), _stream(stream))
    _check(st)


def noalloc_scratch_bytes() -> int:
    """Size of the static scratch behind ffn_forward_noalloc: the value of
    MOE_NOALLOC_SCRATCH_BYTES in include/moe.h (32 MiB).  A CPU test pins it
    against the library: sizes up to it pass the size check, one byte more
    of workspace is refused."""
    return 32 << 20


def _opts(score="softmax", selection_bias=None, dynamic_threshold=0.0, capacity_factor=0.0,
          seq_len=0, slot_kept=None, balance=None) -> RouteOpts:
    sc = SCORE_NAMES.get(score, score) if isinstance(score, str) else int(score)
    if isinstance(sc, str):
        sc = 99
    return RouteOpts(int(sc), _ptr(selection_bias), float(dynamic_threshold),
                     float(capacity_factor), int(seq_len), _ptr(slot_kept), _ptr(balance))


def ffn_forward_ex(x, router, gate_up_proj, down_proj, E: int, K: int, norm_topk_prob: bool, act,
                   out, selected_experts=None, routing_weights=None, router_bias=None, b1=None,
                   b2=None, router_logits=None, workspace=None, stream=None, **opts) -> None:
    """moe_ffn_forward_ex: the forward with routing options (score,
    selection_bias, dynamic_threshold, capacity_factor, seq_len, slot_kept,
    balance - see include/moe.h)."""
    import torch
    D = int(x.shape[-1])
    T = int(x.numel() // D) if D else 0
    F = int(down_proj.shape[-1])
    dt = _dtype_code(x)
    a = _act_code(act)
    if dt in (F32, BF16) and a in (ACT_SILU_GATED, ACT_RELU) and 1 <= K <= E and T > 0:
        wdt = x.dtype
        gu_rows = 2 * F if a == ACT_SILU_GATED else F
        _expect(x, tuple(x.shape), "x", wdt)
        _expect(router, (E, D), "router", wdt)
        _expect(gate_up_proj, (E, gu_rows, D), "gate_up_proj", wdt)
        _expect(down_proj, (E, D, F), "down_proj", wdt)
        _expect(out, tuple(x.shape), "out", wdt)
        _expect(selected_experts, (T, K), "selected_experts", torch.int64, False)
        _expect(routing_weights, (T, K), "routing_weights", torch.float32, False)
        _expect(router_bias, (E,), "router_bias", torch.float32, False)
        _expect(b1, (E, F), "b1", torch.float32, False)
        _expect(b2, (E, D), "b2", torch.float32, False)
        _expect(router_logits, (T, E), "router_logits", torch.float32, False)
        _expect(opts.get("selection_bias"), (E,), "selection_bias", torch.float32, False)
        _expect(opts.get("slot_kept"), (T, K), "slot_kept", torch.uint8, False)
        _expect(opts.get("balance"), (4,), "balance", torch.float32, False)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    o = _opts(**opts)
    st = lib().moe_ffn_forward_ex(
        _ptr(x), _ptr(router), _ptr(gate_up_proj), _ptr(down_proj), E, K, int(bool(norm_topk_prob)),
        a, _ptr(out), _ptr(selected_experts), _ptr(routing_weights), T, D, F, dt,
        _ptr(router_bias), _ptr(b1), _ptr(b2), _ptr(router_logits), _ptr(workspace), ws_bytes,
        ctypes.byref(o), _stream(stream))
    _check(st)


def route_ex(x, router, K: int, norm_topk_prob: bool, selected_experts, routing_weights,
             router_bias=None, router_logits=None, stream=None, **opts) -> None:
    """moe_route_ex: the router with options (not capacity or balance)."""
    import torch
    D = int(x.shape[-1])
    T = int(x.numel() // D) if D else 0
    E = int(router.shape[0])
    dt = _dtype_code(x)
    if dt in (F32, BF16) and 1 <= K <= E and T > 0:
        _expect(x, tuple(x.shape), "x", x.dtype)
        _expect(router, (E, D), "router", x.dtype)
        _expect(selected_experts, (T, K), "selected_experts", torch.int64)
        _expect(routing_weights, (T, K), "routing_weights", torch.float32)
        _expect(router_bias, (E,), "router_bias", torch.float32, False)
        _expect(router_logits, (T, E), "router_logits", torch.float32, False)
        _expect(opts.get("selection_bias"), (E,), "selection_bias", torch.float32, False)
        _expect(opts.get("slot_kept"), (T, K), "slot_kept", torch.uint8, False)
    o = _opts(**opts)
    st = lib().moe_route_ex(_ptr(x), _ptr(router), _ptr(router_bias), T, D, E, K,
                            int(bool(norm_topk_prob)), dt, _ptr(router_logits),
                            _ptr(selected_experts), _ptr(routing_weights), ctypes.byref(o),
                            _stream(stream))
    _check(st)


def route(x, router, K: int, norm_topk_prob: bool, selected_experts, routing_weights,
          router_bias=None, router_logits=None, stream=None) -> None:
    """moe_route on torch tensors."""
    import torch
    D = int(x.shape[-1])
    T = int(x.numel() // D) if D else 0
    E = int(router.shape[0])
    dt = _dtype_code(x)
    if dt in (F32, BF16) and 1 <= K <= E and T > 0:
        _expect(x, tuple(x.shape), "x", x.dtype)
        _expect(router, (E, D), "router", x.dtype)
        _expect(selected_experts, (T, K), "selected_experts", torch.int64)
        _expect(routing_weights, (T, K), "routing_weights", torch.float32)
        _expect(router_bias, (E,), "router_bias", torch.float32, False)
        _expect(router_logits, (T, E), "router_logits", torch.float32, False)
    st = lib().moe_route(_ptr(x), _ptr(router), _ptr(router_bias), T, D, E, K,
                         int(bool(norm_topk_prob)), dt, _ptr(router_logits),
                         _ptr(selected_experts), _ptr(routing_weights), _stream(stream))
    _check(st)


GEMM_AUTO, GEMM_1SM, GEMM_2SM = 0, 1, 2


def set_gemm_mode(mode: int) -> int:
    """Selects the bf16 grouped GEMM (GEMM_AUTO, GEMM_1SM, GEMM_2SM);
    returns the previous mode."""
    prev = int(lib().moe_set_gemm_mode(int(mode)))
    if prev < 0:
        raise ValueError(f"unknown GEMM mode {mode}")
    return prev


def set_tail_swap(max_rows: int) -> int:
    """An expert's last CTA-pair tile of at most max_rows rows (0..128)
    runs with swapped operands; 0 turns it off.  Returns the previous value."""
    prev = int(lib().moe_set_tail_swap(int(max_rows)))
    if prev < 0:
        raise ValueError(f"tail swap rows out of range: {max_rows}")
    return prev


SMALL_CLUSTER_AUTO = 0


def set_small_cluster(ctas: int) -> int:
    """Cluster size of the one-kernel float32 small layer: SMALL_CLUSTER_AUTO
    (16 where possible, else 8), 8 or 16.  Returns the previous value."""
    prev = int(lib().moe_set_small_cluster(int(ctas)))
    if prev < 0:
        raise ValueError(f"small-layer cluster size must be 0, 8 or 16, not {ctas}")
    return prev


def set_pdl(on: bool) -> bool:
    """Programmatic dependent launch between a forward's kernels (default
    off; see moe_set_pdl in include/moe.h); returns the previous setting."""
    return bool(lib().moe_set_pdl(int(bool(on))))


FUSED_GATHER_OFF, FUSED_GATHER_ON, FUSED_GATHER_AUTO = 0, 1, 2


def set_fused_gather(mode) -> int:
    """Selects whether the bf16 gate_up GEMM gathers its rows from x itself
    (TMA gather4) or reads an expert-sorted copy: False/"off", True/"on" or
    "auto" (the default; see moe_set_fused_gather in include/moe.h), or the
    FUSED_GATHER_* value.  Returns the previous value (an int)."""
    if isinstance(mode, str):
        mode = {"off": FUSED_GATHER_OFF, "on": FUSED_GATHER_ON, "auto": FUSED_GATHER_AUTO}[mode]
    elif isinstance(mode, bool):
        mode = FUSED_GATHER_ON if mode else FUSED_GATHER_OFF
    prev = int(lib().moe_set_fused_gather(int(mode)))
    if prev < 0:
        raise ValueError(f"fused gather mode must be 0, 1 or 2, not {mode}")
    return prev


def device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status."""
    return int(lib().moe_device_status(_stream(stream)))


def set_debug_sync(timeout_ms: int) -> int:
    """With timeout_ms > 0 every forward waits, bounded, after each kernel
    and fails naming the first kernel that did not finish; returns the
    previous setting."""
    return int(lib().moe_set_debug_sync(int(timeout_ms)))


def device_error_peek() -> int:
    """The device error word, read without waiting for any stream and
    without clearing it (for watchdogs)."""
    w = ctypes.c_uint(0)
    _check(lib().moe_device_error_peek(ctypes.byref(w)))
    return int(w.value)


def kernel_launches() -> int:
    """Kernels this library has launched in the process so far."""
    return int(lib().moe_kernel_launches())


def error_sites(word: int) -> str:
    """Names of the kernel roles whose bounded waits set bits in ``word``."""
    return lib().moe_error_sites(ctypes.c_uint(word)).decode()


def debug_bounded_wait(timeout_ms: int, stream=None) -> None:
    """Launches the failure-detection probe (a bounded wait that must time
    out); read the outcome with device_status()."""
    _check(lib().moe_debug_bounded_wait(int(timeout_ms), _stream(stream)))


def profile_enable(on: bool = True) -> None:
    _check(lib().moe_profile_enable(int(bool(on))))


def profile_read() -> tuple[dict, int]:
    """Per-stage milliseconds summed since enable/last read, and the number
    of forward calls they cover."""
    buf = (ctypes.c_float * NUM_STAGES)()
    calls = int(lib().moe_profile_read(buf, NUM_STAGES))
    names = [lib().moe_stage_name(i).decode() for i in range(NUM_STAGES)]
    return {n: float(buf[i]) for i, n in enumerate(names)}, calls


class MoEBlock:
    """Sparse MoE feed-forward block with mojolearn.MoEBlock's interface.

    Weights are device tensors in the Hugging Face layout: router (E, D),
    gate_up_proj (E, 2F, D), down_proj (E, D, F) (or W1 (E, F, D), W2
    (E, D, F) plus biases for the ReLU expert).  ``forward`` runs
    moe_ffn_forward and keeps ``router_logits_``, ``selected_experts_``
    (int64) and ``routing_weights_`` of the last call."""

    def __init__(self, router, gate_up_proj, down_proj, top_k: int = 2,
                 norm_topk_prob: bool = True, hidden_act: str = "silu", router_bias=None,
                 b1=None, b2=None):
        if hidden_act not in ACT_NAMES:
            raise NotImplementedError(f"hidden_act {hidden_act!r}")
        E = int(router.shape[0])
        if not (1 <= int(top_k) <= E):
            raise ValueError(f"top_k={top_k} outside [1, {E}]")
        self.router, self.gate_up_proj, self.down_proj = router, gate_up_proj, down_proj
        self.router_bias, self.b1, self.b2 = router_bias, b1, b2
        self.top_k = int(top_k)
        self.norm_topk_prob = bool(norm_topk_prob)
        self.act = ACT_NAMES[hidden_act]
        self._ws = None
        self.router_logits_ = self.selected_experts_ = self.routing_weights_ = None

    @property
    def num_experts(self) -> int:
        return int(self.router.shape[0])

    def load_state_dict(self, sd: dict) -> "MoEBlock":
        for k in ("router", "gate_up_proj", "down_proj"):
            cur = getattr(self, k)
            if tuple(sd[k].shape) != tuple(cur.shape):
                raise ValueError(f"{k}: shape {tuple(sd[k].shape)} != {tuple(cur.shape)}")
        for k in ("router", "gate_up_proj", "down_proj"):
            getattr(self, k).copy_(sd[k])
        return self

    def forward(self, x, stream=None):
        import torch
        if x.dtype == torch.float64:
            raise TypeError("float64 input is not supported")
        D = int(x.shape[-1])
        T = x.numel() // D
        E, K = self.num_experts, self.top_k
        F = int(self.down_proj.shape[-1])
        need = workspace_size(T, D, F, E, K, _dtype_code(x), self.act)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
        out = torch.empty_like(x)
        self.router_logits_ = torch.empty(T, E, dtype=torch.float32, device=x.device)
        self.selected_experts_ = torch.empty(T, K, dtype=torch.int64, device=x.device)
        self.routing_weights_ = torch.empty(T, K, dtype=torch.float32, device=x.device)
        ffn_forward(x, self.router, self.gate_up_proj, self.down_proj, E, K, self.norm_topk_prob,
                    self.act, out, self.selected_experts_, self.routing_weights_,
                    self.router_bias, self.b1, self.b2, self.router_logits_, self._ws, stream)
        return out

    __call__ = forward
