"""The C ABI on the CPU: the library loads, exports every function the header
declares, and rejects bad arguments on the host before touching the device.

No call here reaches a kernel: every call fails validation first, which is
the point (errors are caught before any launch)."""
import ctypes
import os
import re

import pytest

from mixture_experts_ffn_09_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")

P = 0x10000          # a 16-byte aligned stand-in for a device pointer (never dereferenced)
MIS = 0x10008        # misaligned


@pytest.fixture(scope="module")
def L():
    from mixture_experts_ffn_09_b200 import build
    build.build()
    return moe.lib()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("moe_ffn_forward", "moe_route", "moe_ffn_workspace_size", "moe_status_string",
              "moe_device_status", "moe_profile_enable", "moe_profile_read"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in declared_functions():
        assert hasattr(L, n), n
    out = os.popen(f"nm -D --defined-only {moe.LIB_PATH}").read()
    exported = set(re.findall(r" T (moe_\w+)", out))
    assert exported == set(declared_functions())


def test_abi_version_and_strings(L):
    assert moe.abi_version() == 1
    for s in range(10):
        assert moe.status_string(s) not in ("", "unknown status")
    assert moe.status_string(123) == "unknown status"


def test_process_wide_settings_validate_on_host(L):
    """The GEMM settings are host state: each setter returns the previous
    value, and refuses an out-of-range one without changing anything."""
    prev = L.moe_set_tail_swap(64)
    try:
        assert prev == 128                       # MOE_TAIL_SWAP_DEFAULT
        assert L.moe_set_tail_swap(129) == -1    # above MOE_TAIL_SWAP_MAX
        assert L.moe_set_tail_swap(-1) == -1
        assert L.moe_set_tail_swap(0) == 64
        assert L.moe_set_tail_swap(128) == 0
        with pytest.raises(ValueError):
            moe.set_tail_swap(200)
        assert moe.set_tail_swap(32) == 128 and moe.set_tail_swap(128) == 32
    finally:
        L.moe_set_tail_swap(prev)
    g = L.moe_set_gemm_mode(2)
    try:
        assert L.moe_set_gemm_mode(7) == -1
        assert L.moe_set_gemm_mode(1) == 2
    finally:
        L.moe_set_gemm_mode(g)
    f = L.moe_set_fused_gather(0)
    try:
        assert f == 2                              # MOE_FUSED_GATHER_AUTO
        for bad in (3, -1, 7):
            assert L.moe_set_fused_gather(bad) == -1
        assert L.moe_set_fused_gather(1) == 0
        assert moe.set_fused_gather("auto") == 1
        assert moe.set_fused_gather(False) == 2 and moe.set_fused_gather(True) == 0
        with pytest.raises(ValueError):
            moe.set_fused_gather(5)
    finally:
        L.moe_set_fused_gather(f)
    c = L.moe_set_small_cluster(8)
    try:
        assert c == 0                              # MOE_SMALL_CLUSTER_AUTO
        for bad in (1, 4, 12, 32, -1):
            assert L.moe_set_small_cluster(bad) == -1
        assert L.moe_set_small_cluster(16) == 8
        with pytest.raises(ValueError):
            moe.set_small_cluster(9)
        assert moe.set_small_cluster(moe.SMALL_CLUSTER_AUTO) == 16
    finally:
        L.moe_set_small_cluster(c)


C_CALLER = r'''
#include <stdio.h>
#include "moe.h"
int main(void) {
  size_t ws = moe_ffn_workspace_size(4096, 4096, 14336, 8, 2, MOE_BF16, MOE_ACT_SILU_GATED);
  int prev = moe_set_tail_swap(64);
  int back = moe_set_tail_swap(prev);
  printf("%d %s %zu %d %d\n", moe_abi_version(), moe_status_string(MOE_ERR_SHAPE), ws, prev, back);
  return 0;
}
'''


def test_header_serves_a_plain_c_caller(tmp_path):
    """The boundary is a C ABI: the header compiles as strict C99 without
    warnings, and a C program links against the library and calls its
    host-side entry points."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src, exe = tmp_path / "caller.c", tmp_path / "caller"
    src.write_text(C_CALLER)
    libdir = os.path.dirname(moe.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                        os.path.join(os.path.dirname(libdir), "include"), str(src), "-o", str(exe),
                        "-L", libdir, "-lmoe", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    abi, *words = out.stdout.split()
    assert abi == "1" and " ".join(words[:2]) == "unsupported shape"
    ws, prev, back = (int(v) for v in words[2:])
    assert ws == moe.workspace_size(4096, 4096, 14336, 8, 2, moe.BF16, "silu_gated")
    assert prev == 128 and back == 64


def _fwd(L, **kw):
    a = dict(x=P, router=P, gu=P, down=P, E=8, K=2, norm=1, act=0, out=P, sel=P, w=P, T=64, D=64,
             F=128, dt=0, rb=None, b1=None, b2=None, logits=None, ws=P, wsb=1 << 40, stream=None)
    a.update(kw)
    return L.moe_ffn_forward(a["x"], a["router"], a["gu"], a["down"], a["E"], a["K"], a["norm"],
                             a["act"], a["out"], a["sel"], a["w"], a["T"], a["D"], a["F"], a["dt"],
                             a["rb"], a["b1"], a["b2"], a["logits"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(K=0), moe.MOE_ERR_INVALID_ARG),          # top_k below 1
    (dict(K=9), moe.MOE_ERR_INVALID_ARG),          # top_k above E
    (dict(T=0), moe.MOE_ERR_INVALID_ARG),
    (dict(D=-1), moe.MOE_ERR_INVALID_ARG),
    (dict(F=0), moe.MOE_ERR_INVALID_ARG),
    (dict(E=0, K=0), moe.MOE_ERR_INVALID_ARG),
    (dict(dt=2), moe.MOE_ERR_DTYPE),               # float64 is rejected
    (dict(dt=7), moe.MOE_ERR_DTYPE),
    (dict(act=5), moe.MOE_ERR_UNSUPPORTED_ACT),    # anything but SiLU-gated / ReLU
    (dict(E=300, K=2), moe.MOE_ERR_SHAPE),         # beyond MOE_MAX_EXPERTS
    (dict(x=None), moe.MOE_ERR_INVALID_ARG),
    (dict(out=None), moe.MOE_ERR_INVALID_ARG),
    (dict(act=1), moe.MOE_ERR_INVALID_ARG),        # ReLU without biases
    (dict(act=0, b1=P, b2=P), moe.MOE_ERR_INVALID_ARG),   # SiLU with biases
    (dict(x=MIS), moe.MOE_ERR_ALIGNMENT),
    (dict(dt=1, D=60), moe.MOE_ERR_ALIGNMENT),     # bf16 rows need 16-byte strides
    (dict(dt=1, F=100), moe.MOE_ERR_ALIGNMENT),
    (dict(ws=None), moe.MOE_ERR_WORKSPACE),
    (dict(wsb=16), moe.MOE_ERR_WORKSPACE),
])
def test_forward_rejects_on_host(L, kw, code):
    assert _fwd(L, **kw) == code
    assert moe.last_error() != ""


def test_relu_with_all_biases_passes_validation_up_to_the_device(L):
    # With every argument valid the call reaches the device query, which
    # fails on a machine without a GPU (and nothing is launched).
    import torch
    st = _fwd(L, act=1, rb=P, b1=P, b2=P)
    if torch.cuda.is_available():
        pytest.skip("has a GPU")
    assert st in (moe.MOE_ERR_CUDA, moe.MOE_ERR_DEVICE)


def test_route_rejects_on_host(L):
    r = lambda **k: L.moe_route(k.get("x", P), P, None, k.get("T", 64), 64, 8, k.get("K", 2), 1,
                                k.get("dt", 0), None, k.get("sel", P), P, None)
    assert r(K=0) == moe.MOE_ERR_INVALID_ARG
    assert r(K=9) == moe.MOE_ERR_INVALID_ARG
    assert r(T=0) == moe.MOE_ERR_INVALID_ARG
    assert r(dt=2) == moe.MOE_ERR_DTYPE
    assert r(sel=None) == moe.MOE_ERR_INVALID_ARG
    assert r(x=MIS) == moe.MOE_ERR_ALIGNMENT


def test_workspace_size(L):
    ws = moe.workspace_size(64, 64, 128, 8, 2, moe.F32, moe.ACT_SILU_GATED)
    # 128 routed rows, padded to one 128-row tile: x_perm, H, Y dominate
    assert ws >= 128 * (64 + 128 + 64) * 4
    assert ws < 128 * (64 + 128 + 64) * 4 + 64 * 1024
    assert moe.workspace_size(64, 64, 128, 8, 9, moe.F32) == 0
    assert moe.workspace_size(64, 64, 128, 8, 2, moe.F64) == 0
    # a layer in the CTA-pair regime (>= 512 routed rows per expert) also
    # holds the split last wave's fp32 partial tiles: 148 CTAs x 128 x 256
    split = 148 * 128 * 256 * 4
    big = moe.workspace_size(4096, 4096, 14336, 8, 2, moe.BF16)
    assert big >= 8192 * (4096 + 14336 + 4096) * 2 + split
    assert big < 8192 * (4096 + 14336 + 4096) * 2 + split + 8 * 1024 * 1024
    # decode-sized layers take no partial tiles
    dec = moe.workspace_size(32, 4096, 14336, 8, 8, moe.BF16)
    assert dec < 256 * (4096 + 14336 + 4096) * 2 + 1024 * 1024


def test_route_opts_layout_matches_the_header(tmp_path):
    """The ctypes mirror of moe_route_opts_t has the C layout (gcc)."""
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "moe.h"\n'
                   'int main(void){printf("%zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(moe_route_opts_t),'
                   'offsetof(moe_route_opts_t, score), offsetof(moe_route_opts_t, selection_bias),'
                   'offsetof(moe_route_opts_t, dynamic_threshold), offsetof(moe_route_opts_t, capacity_factor),'
                   'offsetof(moe_route_opts_t, seq_len), offsetof(moe_route_opts_t, slot_kept),'
                   'offsetof(moe_route_opts_t, balance)); return 0;}\n')
    exe = tmp_path / "layout"
    import subprocess
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    R = moe.RouteOpts
    want = [ctypes.sizeof(R), R.score.offset, R.selection_bias.offset, R.dynamic_threshold.offset,
            R.capacity_factor.offset, R.seq_len.offset, R.slot_kept.offset, R.balance.offset]
    assert got == want


def test_route_opts_rejected_on_host(L):
    def fwd(**o):
        opts = moe._opts(**o)
        return L.moe_ffn_forward_ex(P, P, P, P, 8, 2, 1, 0, P, P, P, 64, 64, 128, 0, None, None,
                                    None, None, P, 1 << 40, ctypes.byref(opts), None)
    assert fwd(score=5) == moe.MOE_ERR_INVALID_ARG
    assert fwd(dynamic_threshold=-0.1) == moe.MOE_ERR_INVALID_ARG
    assert fwd(dynamic_threshold=float("nan")) == moe.MOE_ERR_INVALID_ARG
    assert fwd(capacity_factor=-1.0) == moe.MOE_ERR_INVALID_ARG
    assert fwd(capacity_factor=1.0, seq_len=48) == moe.MOE_ERR_INVALID_ARG   # not a multiple of 32
    assert fwd(selection_bias=MIS) == moe.MOE_ERR_ALIGNMENT
    opts = moe._opts(capacity_factor=1.0)
    assert L.moe_route_ex(P, P, None, 64, 64, 8, 2, 1, 0, None, P, P, ctypes.byref(opts),
                          None) == moe.MOE_ERR_INVALID_ARG


def test_error_sites_decode_on_host(L):
    """The site bits of the device error word name kernel roles."""
    assert moe.error_sites(0) == ""
    assert moe.error_sites(1) == ""
    assert moe.error_sites(1 | (1 << 16)) == "pair gemm epilogue"
    assert moe.error_sites((1 << 8) | (1 << 17)) == "router producer, bounded-wait probe"
    assert L.moe_device_error_peek(None) == moe.MOE_ERR_INVALID_ARG
