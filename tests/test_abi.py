"""Host-only checks of libgdn.so: it loads, exports every declared symbol and
rejects bad arguments before launching anything.  No GPU needed."""
import os
import re
import subprocess

import pytest

import chunked_gated_delta_14_b200 as gdn
from chunked_gated_delta_14_b200 import build as gbuild
from chunked_gated_delta_14_b200.gdn import (GDN_ERR_ALIGNMENT, GDN_ERR_FAULT_INJECTED,
                                             GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"GDN_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


def test_library_builds_and_loads():
    gbuild.build()
    assert gdn.abi_version() == 9


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert "gdn_chunk_fwd" in names and len(names) >= 5
    out = subprocess.check_output(["nm", "-D", "--defined-only", gbuild.LIB]).decode()
    exported = set(line.split()[-1] for line in out.splitlines() if " T " in line)
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    lib = gdn.lib()
    for n in names:
        getattr(lib, n)


def _args(**kw):
    base = dict(B=2, T=100, H=3, dk=128, dv=128, chunk=64, io_dtype=1, o_dtype=0,
                q=0x10000, k=0x20000, v=0x30000, o=0x40000)
    base.update(kw)
    return gdn.make_args(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), GDN_ERR_INVALID_ARG),
    (dict(T=0), GDN_ERR_INVALID_ARG),
    (dict(dk=48), GDN_ERR_INVALID_ARG),
    (dict(dv=256), GDN_ERR_INVALID_ARG),
    (dict(chunk=8), GDN_ERR_INVALID_ARG),
    (dict(chunk=96), GDN_ERR_INVALID_ARG),
    (dict(io_dtype=7), GDN_ERR_INVALID_ARG),
    (dict(q=None), GDN_ERR_INVALID_ARG),
    (dict(o=None), GDN_ERR_INVALID_ARG),
    (dict(o=0x10000), GDN_ERR_INVALID_ARG),             # o aliases q
    (dict(mode=1, neumann_N=64), GDN_ERR_INVALID_ARG),  # N > C - 1
    (dict(mode=5), GDN_ERR_INVALID_ARG),
    (dict(alpha_per_channel=1), GDN_ERR_INVALID_ARG),   # no alpha given
    (dict(erase=0x50000, beta=0x60000), GDN_ERR_INVALID_ARG),
    (dict(precond=1, rho_eps=0.0), GDN_ERR_INVALID_ARG),
    (dict(q=0x10008), GDN_ERR_ALIGNMENT),
    (dict(kernel=9), GDN_ERR_INVALID_ARG),
    (dict(kernel=2, dv=64), GDN_ERR_UNSUPPORTED),       # fused kernel: dk = dv = 128
    (dict(kernel=2, dv_split=2), GDN_ERR_UNSUPPORTED),  # fused kernel holds the whole head
    (dict(kernel=2, mode=2, neumann_N=3, residual_S=8), GDN_ERR_UNSUPPORTED),   # residual: split only
    (dict(kernel=4, mode=1, neumann_N=16), GDN_ERR_UNSUPPORTED),               # split: N <= 15
    (dict(dv_split=3), GDN_ERR_INVALID_ARG),
    (dict(kernel=2, io_dtype=0), GDN_ERR_UNSUPPORTED),  # tensor cores need bf16 io
    (dict(alpha=0x70000, alpha_per_channel=1, chunk=128, kernel=1, dv_split=8),
     GDN_ERR_UNSUPPORTED),                              # two-gate SIMT at C=128 too big
    (dict(mode=2, neumann_N=3, residual_S=65), GDN_ERR_INVALID_ARG),   # S > 64
    (dict(mode=2, neumann_N=3, residual_S=-1), GDN_ERR_INVALID_ARG),
    (dict(mode=2, neumann_N=64, residual_S=8), GDN_ERR_INVALID_ARG),   # N > C - 1
    (dict(mode=2, neumann_N=3, residual_S=8, kernel=1), GDN_ERR_UNSUPPORTED),  # SIMT has no residual
    (dict(mode=2, neumann_N=3, residual_S=8, io_dtype=0, dk=64, dv=64),
     GDN_ERR_UNSUPPORTED),                              # fp32 io: no tensor-core kernel
    (dict(kernel=3, dv=16), GDN_ERR_UNSUPPORTED),       # recurrent kernel needs dv % 32 == 0
    (dict(kernel=3, alpha=0x70000, alpha_per_channel=1), GDN_ERR_UNSUPPORTED),   # two-gate rule
    (dict(kernel=3, mode=1, neumann_N=3), GDN_ERR_UNSUPPORTED),
    (dict(precond=4, alpha=0x70000, alpha_per_channel=1), GDN_ERR_INVALID_ARG),
    (dict(precond=3, precond_x=1.0, alpha=0x70000, alpha_per_channel=1), GDN_ERR_INVALID_ARG),
    (dict(precond_query=1), GDN_ERR_INVALID_ARG),       # query placement needs a preconditioner
    (dict(precond=2, precond_query=2), GDN_ERR_INVALID_ARG),
])
def test_invalid_arguments_rejected_on_host(kw, status):
    a = _args(**kw)
    assert gdn.select_kernel(a) == -status, gdn.last_error()
    assert gdn.last_error()
    with pytest.raises(gdn.GDNError) as ei:
        gdn.call(a)  # returns before any CUDA call
    assert ei.value.status == status


def test_null_args_pointer():
    import ctypes
    assert gdn.lib().gdn_chunk_fwd(None, None) == GDN_ERR_INVALID_ARG


def test_valid_arguments_select_a_kernel():
    assert gdn.select_kernel(_args(kernel=1)) == 1
    assert gdn.select_kernel(_args()) == 4                                     # split tensor-core kernels
    assert gdn.select_kernel(_args(kernel=2)) == 2                             # the fused kernel on request
    assert gdn.select_kernel(_args(mode=1, neumann_N=63)) == 2                 # N > 15: the fused kernel
    assert gdn.select_kernel(_args(mode=2, neumann_N=3, residual_S=8)) == 4   # residual: split kernels
    assert gdn.select_kernel(_args(dv=64)) == 4                                # dv 64: split kernels
    assert gdn.select_kernel(_args(dv_split=2)) == 4                           # a value split: split kernels
    assert gdn.select_kernel(_args(dv_split=1)) == 2                           # one slice: the fused kernel
    assert gdn.select_kernel(_args(T=1)) == 3                                  # decode step
    assert gdn.select_kernel(_args(T=8, io_dtype=0, dk=64, dv=64)) == 3
    assert gdn.select_kernel(_args(T=9)) == 4                                  # chunked from T = 9
    assert gdn.select_kernel(_args(T=1, mode=1, neumann_N=3)) != 3             # series: chunked only
    assert gdn.select_kernel(_args(io_dtype=0, dk=64, dv=64)) == 1   # fp32 io -> SIMT
    # the two-gate rule: split tensor-core kernels (SIMT prep in fp16 rows + chain) at
    # chunk 64 with preconditioner forms 0 and 1; forms 2, 3, other chunks: SIMT
    two_gate = dict(alpha=0x70000, erase=0x50000, write=0x58000, alpha_per_channel=1)
    assert gdn.select_kernel(_args(precond=1, **two_gate)) == 4
    assert gdn.select_kernel(_args(precond=0, **two_gate)) == 4
    assert gdn.select_kernel(_args(precond=2, **two_gate)) == 1
    assert gdn.select_kernel(_args(precond=1, chunk=32, **two_gate)) == 1
    assert gdn.select_kernel(_args(precond=1, kernel=2, **two_gate)) < 0     # not on the fused kernel
    assert gdn.select_kernel(_args(S0=0x80000, S_T=0x80000)) in (1, 2, 4)  # S_T may alias S0
    # chunk 128: the masked series (N <= 15) on the split kernels as two 64-token
    # halves; wider bands on the SIMT kernel
    assert gdn.select_kernel(_args(chunk=128, mode=1, neumann_N=3)) == 4
    assert gdn.select_kernel(_args(chunk=128, mode=1, neumann_N=15)) == 4
    assert gdn.select_kernel(_args(chunk=128, mode=1, neumann_N=16)) == 1
    # exact inversion at chunk 128: the split kernels, as 64-token chunks (the same o, S_T)
    assert gdn.select_kernel(_args(chunk=128)) == 4
    assert gdn.workspace_bytes(_args(chunk=128)) == gdn.workspace_bytes(_args(chunk=64))
    assert gdn.select_kernel(_args(chunk=128, mode=2, neumann_N=3, residual_S=8)) < 0


def test_fault_injection_env(monkeypatch):
    monkeypatch.setenv("GDN_FAULT_INJECT", "1")
    with pytest.raises(gdn.GDNError) as ei:
        gdn.call(_args())
    assert ei.value.status == GDN_ERR_FAULT_INJECTED


def test_status_strings():
    for s in range(7):
        assert gdn.status_string(s).startswith("GDN_")


def test_python_wrapper_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 1, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        gdn.chunk_fwd(q, q, q)


# ------------------------------------------------------------------ backward

def _bwd_args(**kw):
    G = 1 << 32   # fake device addresses, far enough apart never to overlap
    base = dict(B=2, T=100, H=3, dk=128, dv=128, chunk=64, io_dtype=1, do_dtype=1,
                q=1 * G, k=2 * G, v=3 * G, alpha=4 * G, beta=5 * G, S0=6 * G, grad_o=7 * G,
                grad_S_T=8 * G, grad_q=9 * G, grad_k=10 * G, grad_v=11 * G, grad_alpha=12 * G,
                grad_beta=13 * G, grad_S0=14 * G)
    base.update(kw)
    return gdn.make_bwd_args(**base)


def _bwd_ws_expected(B, T, H, dk, dv, C):
    nch = B * H * -(-T // C)
    region = lambda f: (f * nch * 4 + 255) // 256 * 256
    return region(C) + 3 * region(C * C) + region(C * dk) + 2 * region(C * dv) + 3 * region(dk * dv)


@pytest.mark.parametrize("shape", [(2, 100, 3, 128, 128, 64), (1, 1, 1, 16, 32, 16),
                                   (4, 4096, 16, 128, 128, 64), (3, 77, 5, 32, 96, 32)])
def test_bwd_workspace_size(shape):
    B, T, H, dk, dv, C = shape
    a = _bwd_args(B=B, T=T, H=H, dk=dk, dv=dv, chunk=C)
    assert gdn.bwd_workspace_bytes(a) == _bwd_ws_expected(*shape), gdn.last_error()


def test_bwd_workspace_size_with_the_series():
    # the masked series (and its residual form) add one C x C region per chunk-head
    nch = 2 * 3 * 2
    extra = (64 * 64 * nch * 4 + 255) // 256 * 256
    base = _bwd_ws_expected(2, 100, 3, 128, 128, 64)
    assert gdn.bwd_workspace_bytes(_bwd_args(mode=1, neumann_N=3)) == base + extra
    assert gdn.bwd_workspace_bytes(_bwd_args(mode=2, neumann_N=3, residual_S=8)) == base + extra


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), GDN_ERR_INVALID_ARG),
    (dict(H=70000), GDN_ERR_INVALID_ARG),
    (dict(chunk=128), GDN_ERR_UNSUPPORTED),            # backward chunks: 16, 32, 64
    (dict(chunk=8), GDN_ERR_UNSUPPORTED),
    (dict(dk=48), GDN_ERR_UNSUPPORTED),
    (dict(dv=16), GDN_ERR_UNSUPPORTED),                # value slices of 32 columns
    (dict(io_dtype=3), GDN_ERR_INVALID_ARG),
    (dict(do_dtype=3), GDN_ERR_INVALID_ARG),
    (dict(grad_o=None), GDN_ERR_INVALID_ARG),
    (dict(grad_k=None), GDN_ERR_INVALID_ARG),
    (dict(alpha=None), GDN_ERR_INVALID_ARG),           # grad_alpha without alpha
    (dict(beta=None), GDN_ERR_INVALID_ARG),            # grad_beta without beta
    (dict(grad_q=(1 << 32) + 64), GDN_ERR_INVALID_ARG),  # grad_q overlaps q
    (dict(grad_v=10 * (1 << 32) + 4096), GDN_ERR_INVALID_ARG),  # grad_v overlaps grad_k
    (dict(grad_S0=6 * (1 << 32)), GDN_ERR_INVALID_ARG),  # grad_S0 aliases S0
    (dict(grad_q=9 * (1 << 32) + 8), GDN_ERR_ALIGNMENT),
    (dict(mode=7), GDN_ERR_INVALID_ARG),
    (dict(mode=1, neumann_N=64), GDN_ERR_INVALID_ARG),      # the series' order: 0 .. chunk - 1
    (dict(mode=2, neumann_N=3, residual_S=65), GDN_ERR_INVALID_ARG),
])
def test_bwd_invalid_arguments_rejected_on_host(kw, status):
    a = _bwd_args(**kw)
    assert gdn.bwd_workspace_bytes(a) == 0 and gdn.last_error()
    with pytest.raises(gdn.GDNError) as ei:
        gdn.call_bwd(a)   # returns before any CUDA call
    assert ei.value.status == status


def test_bwd_workspace_must_not_overlap_and_must_be_large_enough():
    a = _bwd_args()
    need = gdn.bwd_workspace_bytes(a)
    a.workspace, a.workspace_bytes = 20 << 32, need - 256
    with pytest.raises(gdn.GDNError) as ei:
        gdn.call_bwd(a)
    assert ei.value.status == GDN_ERR_INVALID_ARG and "workspace" in str(ei.value)
    a.workspace, a.workspace_bytes = (11 << 32) - 4096, need   # runs into grad_v
    with pytest.raises(gdn.GDNError) as ei:
        gdn.call_bwd(a)
    assert ei.value.status == GDN_ERR_INVALID_ARG


def test_bwd_optional_gradients_may_be_null():
    a = _bwd_args(alpha=None, beta=None, grad_alpha=None, grad_beta=None, grad_S0=None,
                  S0=None, grad_S_T=None)
    assert gdn.bwd_workspace_bytes(a) > 0, gdn.last_error()


def test_python_backward_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 1, 16, dtype=torch.bfloat16)
    v = torch.zeros(1, 4, 1, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        gdn.chunk_bwd(q, q, v, None, None, v)


def _c_layout(struct, fields, tmp_path):
    """sizeof and offsetof of every field of a struct in include/gdn.h, from gcc."""
    src = tmp_path / "layout.c"
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "gdn.h"', "int main(void) {",
             f'  printf("%zu\\n", sizeof({struct}));']
    lines += [f'  printf("%zu\\n", offsetof({struct}, {f}));' for f in fields]
    lines += ["  return 0;", "}"]
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    vals = [int(v) for v in subprocess.check_output([str(exe)]).decode().split()]
    return vals[0], vals[1:]


@pytest.mark.parametrize("struct,mirror", [("gdn_fwd_args", gdn.FwdArgs), ("gdn_bwd_args", gdn.BwdArgs)])
def test_ctypes_mirrors_match_the_c_structs(struct, mirror, tmp_path):
    import ctypes
    fields = [f[0] for f in mirror._fields_]
    size, offsets = _c_layout(struct, fields, tmp_path)
    assert ctypes.sizeof(mirror) == size
    for name, off in zip(fields, offsets):
        assert getattr(mirror, name).offset == off, name


def test_debug_chunk_T_rejects_on_host():
    """gdn_debug_chunk_T validates (b, h, n), T_out and the kernel before any launch."""
    import ctypes
    L = gdn.lib()
    fake = 0x90000
    for (b, h, n) in [(-1, 0, 0), (2, 0, 0), (0, 3, 0), (0, 0, 2)]:      # B=2, H=3, T=100: 2 chunks
        assert L.gdn_debug_chunk_T(ctypes.byref(_args()), b, h, n, ctypes.c_void_p(fake), None) == GDN_ERR_INVALID_ARG
    assert L.gdn_debug_chunk_T(ctypes.byref(_args()), 0, 0, 0, None, None) == GDN_ERR_INVALID_ARG
    assert L.gdn_debug_chunk_T(ctypes.byref(_args()), 0, 0, 0, ctypes.c_void_p(fake + 8), None) == GDN_ERR_ALIGNMENT
    assert L.gdn_debug_chunk_T(ctypes.byref(_args(kernel=1)), 0, 0, 0, ctypes.c_void_p(fake), None) == GDN_ERR_UNSUPPORTED
    assert L.gdn_debug_chunk_T(ctypes.byref(_args(dv=64)), 0, 0, 0, ctypes.c_void_p(fake), None) == GDN_ERR_UNSUPPORTED


def test_workspace_sizes_per_kernel():
    """The SIMT kernels keep, per chunk-head, the fp32 matrices TB, P (C x C), E, Q',
    K'' (C x dk) and the decay d (dk), padded to 16 bytes; the preconditioned two-gate
    rule adds three dk arrays per chunk-head.  The split tensor-core kernels keep
    24 KiB per chunk-head, the fused and the recurrent kernels nothing."""
    B, T, H, C, dk = 2, 100, 3, 64, 128
    chunks = B * H * (-(-T // C))
    per = 2 * C * C + 3 * C * dk + dk
    per = (per + 3) // 4 * 4
    assert gdn.workspace_bytes(_args(kernel=1)) == chunks * per * 4
    two_gate = _args(kernel=1, alpha=0x70000, alpha_per_channel=1, precond=1, erase=0x50000, write=0x58000)
    assert gdn.workspace_bytes(two_gate) == chunks * (per + 3 * dk) * 4
    # the two-gate rule on the split tensor-core kernels: fp16 rows of 128 B per
    # chunk-head (TB, P as hi + lo: 4 x 64; E, Q', K'': 128 each; U as hi + lo: 2 d_v;
    # d: 4), then the preconditioner's three running-average arrays
    two_gate_tc = _args(kernel=4, alpha=0x70000, alpha_per_channel=1, precond=1, erase=0x50000, write=0x58000)
    assert gdn.workspace_bytes(two_gate_tc) == chunks * ((640 + 2 * 128 + 4) * 128 + 3 * dk * 4)
    assert gdn.workspace_bytes(_args(kernel=4)) == chunks * 24576
    assert gdn.workspace_bytes(_args(kernel=2)) == 0
    assert gdn.workspace_bytes(_args(T=4, kernel=3)) == 0
    c128 = _args(kernel=1, chunk=128, mode=1, neumann_N=3)
    per128 = 2 * 128 * 128 + 3 * 128 * dk + dk
    assert gdn.workspace_bytes(c128) == B * H * 1 * per128 * 4
    # chunk 128 on the split kernels: per 64-token half the 24 KiB of T matrices and
    # the band corner's two parts (C2': 16 x dk, C1 V_a: 16 x dv, fp32)
    dv = 128
    assert gdn.workspace_bytes(_args(kernel=4, chunk=128, mode=1, neumann_N=3)) == \
        chunks * (24576 + 16 * (dk + dv) * 4)


def test_simt_call_without_workspace_rejected_on_host():
    a = _args(kernel=1)
    with pytest.raises(gdn.GDNError) as ei:
        gdn.call(a)   # returns before any CUDA call
    assert ei.value.status == GDN_ERR_INVALID_ARG and "workspace" in str(ei.value)
    a.workspace, a.workspace_bytes = 0x900000, gdn.workspace_bytes(a) - 16
    with pytest.raises(gdn.GDNError) as ei:
        gdn.call(a)
    assert ei.value.status == GDN_ERR_INVALID_ARG and "workspace" in str(ei.value)
