"""Sequence segments of the split tensor-core path (B = 1, scalar rule, chunk 64).

The state update is affine in the state, so over a run of chunks
h_end = M h_start + N: M is the run from h = I with v = 0, N the run from
h = 0.  With three segments the library runs s0 from S0, s1 from 0 (N) and s1
with v = 0 from I (M) side by side, composes h at s2's start, then reruns s1
and s2 from their true starts.

CPU checks (no GPU): the decomposition itself on the fp64 token recurrence
(the reading of "M" and "N" the schedule relies on, with alpha == 1 so that M
is far from 0), and the host-side selection rules.

GPU checks: the segment schedule against the fp64 oracle at the bf16 bar
(max|err| <= 2e-2 * rms on fp32 o and on S_T), for the workload's strong
decay, weak decay and alpha == 1 (where M carries the state across segments),
with ragged tails, S0, S_T aliasing S0, the masked Neumann mode against its
chunk model, repeated calls, and against the one-pass schedule.
"""
import numpy as np
import pytest
import torch

import chunked_gated_delta_14_b200 as gdn
import oracle
from chunked_gated_delta_14_b200.inputs import make_inputs, workload
from oracle import chunk_forms as cf

from gpu_util import TOL_BF16_REL_RMS, report, stats

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _args(**kw):
    base = dict(B=1, T=64 * 300, H=16, dk=128, dv=128, chunk=64, io_dtype=1, o_dtype=1,
                q=1 << 20, k=2 << 20, v=3 << 20, o=4 << 20, alpha=5 << 20, beta=6 << 20,
                kernel=gdn.gdn.KERNELS["tc_split"])
    base.update(kw)
    return gdn.make_args(**base)


# ------------------------------------------------------------------ CPU checks

@pytest.mark.parametrize("decay", ["none", "weak"])
def test_affine_state_map_on_the_recurrence(decay):
    """h_end(h0) = M h0 + N on the fp64 token recurrence, M from (h0 = I, v = 0)
    and N from h0 = 0, for a random h0: the identity the segment schedule uses."""
    w = workload("gdn_bf16", B=1, H=2, T=40, dk=32, dv=8, decay=decay, s0_std=0.5)
    x = make_inputs(w, seed=3)
    q, k, v, a, b, h0 = x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"]
    _, S_full = oracle.gated_delta_fwd(q, k, v, a, b, h0)
    _, N = oracle.gated_delta_fwd(q, k, v, a, b, None)
    eye = torch.eye(32, dtype=torch.float32).expand(1, 2, 32, 32).contiguous()
    v0 = torch.zeros((1, 40, 2, 32), dtype=v.dtype)
    _, M = oracle.gated_delta_fwd(q, k, v0, a, b, eye)
    h0d = h0.double().numpy()
    comp = np.einsum("bhij,bhjc->bhic", M, h0d) + N
    assert np.abs(comp - S_full).max() <= 1e-10 * max(1.0, np.abs(S_full).max())
    if decay == "none":
        # the linear part is far from 0 here, so the check above has teeth
        assert np.abs(M).max() > 0.1


def test_segment_selection_rules():
    # long sequence, chains fill under a third of the SMs: three segments by default
    assert gdn.select_segments(_args(T=65536)) == 3
    assert gdn.select_segments(_args(T=65536, seq_segments=1)) == 1
    # below the default length, or with too many chains per pass: one pass
    assert gdn.select_segments(_args(T=64 * 255)) == 1
    assert gdn.select_segments(_args(T=65536, H=25)) == 1
    assert gdn.select_segments(_args(B=4, T=4096)) == 1
    # forced: any B = 1 call of the scalar rule at chunk 64 with >= 3 chunks
    assert gdn.select_segments(_args(T=129, H=2, seq_segments=3)) == 3
    assert gdn.select_segments(_args(T=128, H=2, seq_segments=3)) == -gdn.gdn.GDN_ERR_UNSUPPORTED
    assert gdn.select_segments(_args(B=2, T=4096, seq_segments=3)) == -gdn.gdn.GDN_ERR_UNSUPPORTED
    assert gdn.select_segments(_args(T=4096, chunk=128, mode=1, neumann_N=3,
                                     seq_segments=3)) == -gdn.gdn.GDN_ERR_UNSUPPORTED
    assert gdn.select_segments(_args(T=4096, seq_segments=2)) == -gdn.gdn.GDN_ERR_INVALID_ARG
    assert gdn.select_segments(_args(T=4096, seq_segments=3,
                                     kernel=gdn.gdn.KERNELS["simt"])) == -gdn.gdn.GDN_ERR_UNSUPPORTED
    # the segment path keeps the kernel choice
    assert gdn.select_kernel(_args(T=65536)) == gdn.gdn.KERNELS["tc_split"]


def test_segment_workspace_size():
    one = gdn.workspace_bytes(_args(T=4096, seq_segments=1))
    three = gdn.workspace_bytes(_args(T=4096, seq_segments=3))
    assert one == 16 * 64 * 24576
    assert three == one + 16 * 128 * (2 * 128 + 3 * 128) * 4
    # the fixed-scratch entry point always runs one pass; its limit is unchanged
    assert gdn.workspace_bytes(_args(T=4096, H=4, seq_segments=1)) <= gdn.gdn.STATIC_SCRATCH_BYTES


# ------------------------------------------------------------------ GPU checks

def _run(x, w, segments, mode="exact", N=3, out=None, S_T=None, S0=None):
    d = {k: (None if v is None else v.to("cuda").contiguous()) for k, v in x.items()}
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S0=d["S0"] if S0 is None else S0,
                         chunk=64, mode=mode, N=N, o_dtype=torch.float32, kernel="tc_split",
                         segments=segments, out=out, S_T=S_T)
    torch.cuda.synchronize()
    return o, S


def _check(name, o, S, o_ref, s_ref):
    so = stats(o.double().cpu().numpy(), o_ref)
    ss = stats(S.double().cpu().numpy(), s_ref)
    report(name, o=so, S_T=ss)
    assert so["max_rel_rms"] <= TOL_BF16_REL_RMS, so
    assert ss["max_rel_rms"] <= TOL_BF16_REL_RMS, ss


@pytest.mark.gpu
@needs_cuda
@pytest.mark.parametrize("decay", ["scalar", "weak", "none"])
@pytest.mark.parametrize("T", [64 * 30 + 17, 64 * 96])
def test_segments_match_oracle(decay, T):
    w = workload("gdn_bf16", B=1, H=4, T=T, decay=decay, s0_std=0.02)
    x = make_inputs(w, seed=41)
    a = _args(T=T, H=4, seq_segments=3, beta=6 << 20, alpha=(5 << 20) if x["alpha"] is not None else None)
    assert gdn.select_segments(a) == 3
    o_ref, s_ref = oracle.gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"])
    o, S = _run(x, w, 3)
    _check(f"segments_{decay}_{T}", o, S, o_ref, s_ref)


@pytest.mark.gpu
@needs_cuda
@pytest.mark.parametrize("T", [192, 193, 64 * 7 + 1])
def test_segments_short_and_ragged(T):
    """The shortest schedules: one chunk per segment, and a tail chunk in s2."""
    w = workload("gdn_bf16", B=1, H=2, T=T, decay="none", s0_std=0.02)
    x = make_inputs(w, seed=42)
    o_ref, s_ref = oracle.gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"])
    o, S = _run(x, w, 3)
    _check(f"segments_short_{T}", o, S, o_ref, s_ref)


@pytest.mark.gpu
@needs_cuda
def test_segments_neumann_against_chunk_model():
    w = workload("gdn_bf16", B=1, H=4, T=64 * 40 + 5, decay="weak", s0_std=0.02)
    x = make_inputs(w, seed=43)
    o_ref, s_ref = cf.chunked_gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"],
                                              chunk=64, inverse=cf.neumann_inverse(3))
    o, S = _run(x, w, 3, mode="neumann", N=3)
    _check("segments_neumann3", o, S, o_ref, s_ref)


@pytest.mark.gpu
@needs_cuda
def test_segments_repeat_alias_and_one_pass():
    """Two calls in a row give identical results (the library's streams and events
    are reused); S_T may alias S0; the one-pass schedule agrees within the bar."""
    w = workload("gdn_bf16", B=1, H=16, T=64 * 60 + 33, decay="none", s0_std=0.02)
    x = make_inputs(w, seed=44)
    o1, S1 = _run(x, w, 3)
    o2, S2 = _run(x, w, 3)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    state = x["S0"].to("cuda").contiguous().clone()
    o3, S3 = _run(x, w, 3, S0=state, S_T=state)
    assert S3.data_ptr() == state.data_ptr()
    assert torch.equal(o3, o1) and torch.equal(S3, S1)
    op, Sp = _run(x, w, 1)
    _check("segments_vs_one_pass", o1, S1, op.double().cpu().numpy(), Sp.double().cpu().numpy())
    o_ref, s_ref = oracle.gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"])
    _check("segments_alias", o3, S3, o_ref, s_ref)


@pytest.mark.gpu
@needs_cuda
def test_segments_long_context_bf16_output():
    """The timed long-context configuration (bf16 o, the library's choice of
    segments) against the fp64 oracle: every element within the bar plus one bf16
    rounding of the reference, and S_T (fp32) at the bar."""
    from gpu_util import bf16_allowance_ok
    w = workload("long_context")
    x = make_inputs(w)
    d = {k: (None if v is None else v.to("cuda").contiguous()) for k, v in x.items()}
    a = _args(T=w.T, H=w.H, o_dtype=1)
    assert gdn.select_segments(a) == 3
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S0=d["S0"], chunk=64)
    torch.cuda.synchronize()
    assert o.dtype == torch.bfloat16
    o_ref, s_ref = oracle.gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"])
    got = o.double().cpu().numpy()
    report("segments_long_context_bf16_o", o=stats(got, o_ref), S_T=stats(S.double().cpu().numpy(), s_ref))
    assert bf16_allowance_ok(got, o_ref)
    assert stats(S.double().cpu().numpy(), s_ref)["max_rel_rms"] <= TOL_BF16_REL_RMS


@pytest.mark.gpu
@needs_cuda
def test_segments_residual_mode_and_narrow_values():
    """The residual-corrected series through the segments (against its chunk model),
    and d_v = 64 (one value slice per head) without a final state."""
    w = workload("gdn_bf16", B=1, H=3, T=64 * 33 + 9, decay="weak", s0_std=0.02)
    x = make_inputs(w, seed=45)
    d = {k: (None if v is None else v.to("cuda").contiguous()) for k, v in x.items()}
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S0=d["S0"], chunk=64, mode="residual",
                         N=3, S=8, o_dtype=torch.float32, kernel="tc_split", segments=3)
    torch.cuda.synchronize()
    o_ref, s_ref = cf.chunked_gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"], chunk=64,
                                              inverse=cf.residual_inverse(3, 8))
    _check("segments_residual", o, S, o_ref, s_ref)

    w64 = workload("gdn_bf16", B=1, H=5, T=64 * 40, dv=64, decay="none", s0_std=0.02)
    x = make_inputs(w64, seed=46)
    d = {k: (None if v is None else v.to("cuda").contiguous()) for k, v in x.items()}
    a = _args(T=w64.T, H=5, dv=64, seq_segments=3)
    assert gdn.select_segments(a) == 3
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S0=d["S0"], chunk=64,
                         o_dtype=torch.float32, kernel="tc_split", segments=3, final_state=False)
    torch.cuda.synchronize()
    assert S is None
    o_ref, _ = oracle.gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"])
    so = stats(o.double().cpu().numpy(), o_ref)
    report("segments_dv64_no_state", o=so)
    assert so["max_rel_rms"] <= TOL_BF16_REL_RMS, so
