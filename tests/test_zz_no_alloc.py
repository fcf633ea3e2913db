"""gdn_chunk_fwd_static_scratch: the split tensor-core kernels with the
library's fixed scratch array instead of a caller workspace, for callers that
cannot allocate device memory per call.  Collected last on purpose, so that it
also runs after every other test has used the device."""
import ctypes

import numpy as np
import pytest
import torch

import chunked_gated_delta_14_b200 as gdn
import chunked_gated_delta_14_b200.gdn as G
from chunked_gated_delta_14_b200.inputs import make_inputs, workload
from gpu_util import TOL_BF16_REL_RMS


def _args(w, d, o, S):
    ptr = lambda t: None if t is None else t.data_ptr()
    return G.make_args(B=w.B, T=w.T, H=w.H, dk=w.dk, dv=w.dv, chunk=w.chunk, io_dtype=1, o_dtype=0,
                       q=ptr(d["q"]), k=ptr(d["k"]), v=ptr(d["v"]), alpha=ptr(d["alpha"]),
                       beta=ptr(d["beta"]), S0=ptr(d["S0"]), o=o.data_ptr(), S_T=S.data_ptr(),
                       mode=0, kernel=2)


def test_static_scratch_rejects_oversize_and_workspace():
    # host-side checks: they return before any device call
    w = workload("gdn_bf16", B=2, H=16, T=4096)          # 2048 chunk-heads: 48 MiB
    fake = 1 << 20
    a = G.make_args(B=w.B, T=w.T, H=w.H, dk=128, dv=128, chunk=64, io_dtype=1, o_dtype=0,
                    q=fake, k=fake, v=fake, alpha=fake, beta=fake, o=2 * fake, S_T=3 * fake,
                    mode=0, kernel=2)
    s = G.lib().gdn_chunk_fwd_static_scratch(ctypes.byref(a), None)
    assert s == G.GDN_ERR_INVALID_ARG
    msg = G.last_error()
    assert "scratch" in msg and str(48 << 20) in msg, msg
    a.B = 1                                                  # fits, but a workspace is passed
    a.workspace, a.workspace_bytes = 4 * fake, 24 << 20
    assert G.lib().gdn_chunk_fwd_static_scratch(ctypes.byref(a), None) == G.GDN_ERR_INVALID_ARG
    a.workspace, a.workspace_bytes = None, 0
    a.kernel = 1                                             # SIMT is not this entry point's kernel
    assert G.lib().gdn_chunk_fwd_static_scratch(ctypes.byref(a), None) == G.GDN_ERR_UNSUPPORTED
    a.kernel = 2
    a.T, a.H, a.seq_segments = 64 * 300, 1, 3                # sequence segments: not this entry point's
    assert G.lib().gdn_chunk_fwd_static_scratch(ctypes.byref(a), None) == G.GDN_ERR_UNSUPPORTED


def _free_bytes():
    free, _ = torch.cuda.mem_get_info()
    return free


@pytest.mark.gpu
@pytest.mark.parametrize("T", [4096, 1000])
def test_static_scratch_matches_workspace_entry(T):
    """The fixed-scratch entry runs the split tensor-core kernels on the
    library's array; the same kernels on a caller workspace must give the same
    bits, three times in a row, and no call may allocate device memory.
    T = 4096 fills the array exactly (1 x 16 heads x 64 chunks = 1024
    chunk-heads); T = 1000 ends in a ragged chunk."""
    w = workload("gdn_bf16", B=1, H=16, T=T, s0_std=0.02)
    assert w.B * w.H * (-(-w.T // 64)) * 24576 <= G.STATIC_SCRATCH_BYTES
    x = make_inputs(w, seed=21)
    d = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    o_ref, s_ref = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S0=d["S0"],
                                 o_dtype=torch.float32, kernel="tc_split")
    torch.cuda.synchronize()
    rms_o = float(o_ref.double().pow(2).mean().sqrt())
    stream = torch.cuda.current_stream().cuda_stream
    outs = [(torch.full_like(o_ref, float("nan")), torch.full_like(s_ref, float("nan"))) for _ in range(3)]
    torch.cuda.synchronize()
    # The scratch array is part of the library's device image.  With lazy module
    # loading (the CUDA default) the driver maps it when the entry point first
    # takes its address, so the first call may lower free memory by at most the
    # array (plus the image's code); later calls must change nothing.
    alloc0, free0 = torch.cuda.memory_allocated(), _free_bytes()
    G.call_static_scratch(_args(w, d, *outs[0]), stream)
    gdn.device_check(stream)
    torch.cuda.synchronize()
    free1 = _free_bytes()
    assert 0 <= free0 - free1 <= G.STATIC_SCRATCH_BYTES + (8 << 20), (free0, free1)
    for o, S in outs[1:]:                                   # two more calls in a row
        G.call_static_scratch(_args(w, d, o, S), stream)
        gdn.device_check(stream)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    assert _free_bytes() == free1, "a call after the first changed the device's free memory"
    for call, (o, S) in enumerate(outs):
        assert torch.equal(o, o_ref) and torch.equal(S, s_ref), call
    # and the split kernels meet the accuracy bar (against the fused kernel's result)
    o_f, _ = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S0=d["S0"],
                           o_dtype=torch.float32, kernel="tc")
    torch.cuda.synchronize()
    assert float((o_f.double() - o_ref.double()).abs().max()) <= TOL_BF16_REL_RMS * rms_o
