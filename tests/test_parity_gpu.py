"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Every workload is drawn by the shared seeded generator, so both sides see the
same bits.  The full-size cases run in the launch configuration the benchmark
times (kernel selection "auto", default value-axis split).
"""
import numpy as np
import pytest
import torch

from chunked_gated_delta_14_b200.inputs import make_inputs, workload
from oracle import chunk_forms as cf

from gpu_util import (TOL_BF16_REL_RMS, TOL_F32_ABS, bf16_allowance_ok, report, run_gpu,
                      run_oracle, stats)

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _check_bf16(name, w, x, o_ref, s_ref, **kw):
    o, s = run_gpu(x, w, o_dtype=torch.float32, **kw)
    so, ss = stats(o, o_ref), stats(s, s_ref)
    report(name, o=so, S_T=ss, **{k: str(v) for k, v in kw.items()})
    assert so["max_rel_rms"] <= TOL_BF16_REL_RMS, so
    assert ss["max_rel_rms"] <= TOL_BF16_REL_RMS, ss
    return o, s


# ------------------------------------------------------------ configuration 1

@needs_cuda
def test_plain_delta_rule_fp32():
    w = workload("plain_fp32")
    x = make_inputs(w)
    o_ref, s_ref = run_oracle(x, w)
    o, s = run_gpu(x, w)
    report("plain_fp32", o=stats(o, o_ref), S_T=stats(s, s_ref))
    assert np.abs(o - o_ref).max() <= TOL_F32_ABS
    assert np.abs(s - s_ref).max() <= TOL_F32_ABS


# ------------------------------------------------------------ configuration 2

@needs_cuda
@pytest.mark.parametrize("kernel", ["auto", "simt"])
def test_gdn_bf16_small_ragged(kernel):
    w = workload("gdn_bf16", B=2, H=3, T=1000)
    x = make_inputs(w, seed=3)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16(f"gdn_small_{kernel}", w, x, o_ref, s_ref, kernel=kernel)


@needs_cuda
def test_gdn_bf16_full_size():
    w = workload("gdn_bf16")
    x = make_inputs(w)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16("gdn_full_auto", w, x, o_ref, s_ref)
    # bf16 output: the bar plus one bf16 ulp of the reference
    o16, _ = run_gpu(x, w, o_dtype=torch.bfloat16)
    report("gdn_full_auto_o_bf16", o=stats(o16, o_ref))
    assert bf16_allowance_ok(o16, o_ref)


# ------------------------------------------------------------ configuration 3

@needs_cuda
def test_long_context_state_carry():
    w = workload("long_context")
    x = make_inputs(w)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16("long_context_full_auto", w, x, o_ref, s_ref)


# ------------------------------------------------------------ configuration 4

@needs_cuda
@pytest.mark.parametrize("chunk", [64, 128])
@pytest.mark.parametrize("N", [2, 3, 4])
def test_neumann_sweep(chunk, N):
    w = workload("neumann", B=1, H=4, chunk=chunk, neumann_N=N)
    x = make_inputs(w)
    o_ref, s_ref = run_oracle(x, w)               # chunk model with the masked series
    o, s = _check_bf16(f"neumann_C{chunk}_N{N}", w, x, o_ref, s_ref)
    ex = w.replace(mode="exact")
    o_ex, s_ex = run_oracle(x, ex)
    report(f"neumann_C{chunk}_N{N}_vs_exact_oracle", o=stats(o, o_ex), S_T=stats(s, s_ex))


@needs_cuda
@pytest.mark.parametrize("T,N,s0", [(1000, 15, 0.02), (900, 1, 0.0), (129, 7, 0.02), (640, 0, 0.02),
                                    (4096, 3, 0.02), (64, 3, 0.02), (65, 2, 0.02), (128, 15, 0.0)])
def test_neumann_chunk128_halves_ragged(T, N, s0):
    """Chunk 128 of the masked series on the split tensor-core kernels: each
    128-token chunk runs as two 64-token halves plus the band's corner between
    them.  Ragged ends (a partial second half; a lone first half), a sequence of one
    half (T = 64: no corner launch), a one-token second half (T = 65), exactly one
    128-token chunk, the widest band (N = 15), N = 0 (T = I: no corner) and a
    nonzero initial state."""
    w = workload("neumann", B=2, H=2, T=T, chunk=128, neumann_N=N, s0_std=s0)
    x = make_inputs(w, seed=40 + N)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16(f"neumann_C128_halves_T{T}_N{N}", w, x, o_ref, s_ref, kernel="tc_split")


# ------------------------------------------- residual correction (next row 1)

@needs_cuda
@pytest.mark.parametrize("N,S", [(3, 8), (2, 2), (3, 0), (1, 31)])
def test_residual_correction_small(N, S):
    """T0 = masked series to order N, corrected with S residual terms, on a ragged
    sequence with S0; S = 0 is the masked series itself, (N+1)(S+1) >= C exact."""
    w = workload("gdn_bf16", B=1, H=2, T=300, s0_std=0.02)
    x = make_inputs(w, seed=17)
    o_ref, s_ref = cf.chunked_gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"],
                                              chunk=64, inverse=cf.residual_inverse(N, S))
    _check_bf16(f"residual_N{N}_S{S}", w, x, o_ref, s_ref, mode="residual", N=N, S=S)


@needs_cuda
def test_residual_correction_full_size():
    """N = 3, S = 8 on the bench workload: parity against the chunk model with the
    same correction; the error against the exact recurrence is reported."""
    w = workload("gdn_bf16")
    x = make_inputs(w)
    o_ref, s_ref = cf.chunked_gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"],
                                              chunk=64, inverse=cf.residual_inverse(3, 8))
    o, s = _check_bf16("residual_N3_S8_full", w, x, o_ref, s_ref, mode="residual", N=3, S=8)
    o_ex, s_ex = run_oracle(x, w)
    report("residual_N3_S8_vs_exact_oracle", o=stats(o, o_ex), S_T=stats(s, s_ex))


# ---------------------------------------------------- decode steps (next row 4)

@needs_cuda
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (32, 32), (16, 32), (128, 64)])
def test_recurrent_decode_step(dk, dv):
    """One token per call with a carried state: the token-by-token kernel (chosen
    automatically for short T) against the oracle, bf16 and fp32 inputs."""
    import chunked_gated_delta_14_b200 as gdn
    for io in ("bf16", "f32"):
        w = workload("gdn_bf16", B=3, H=4, T=1, dk=dk, dv=dv, io=io, s0_std=0.02)
        x = make_inputs(w, seed=18)
        o_ref, s_ref = run_oracle(x, w)
        o, s = run_gpu(x, w, o_dtype=torch.float32)
        if io == "f32":
            assert np.abs(o - o_ref).max() <= TOL_F32_ABS and np.abs(s - s_ref).max() <= TOL_F32_ABS
        else:
            so, ss = stats(o, o_ref), stats(s, s_ref)
            report(f"decode_{dk}_{dv}", o=so, S_T=ss)
            assert so["max_rel_rms"] <= TOL_BF16_REL_RMS and ss["max_rel_rms"] <= TOL_BF16_REL_RMS
        a = gdn.make_args(B=w.B, T=w.T, H=w.H, dk=dk, dv=dv, chunk=64, io_dtype=int(io == "bf16"),
                          o_dtype=0, q=1 << 20, k=2 << 20, v=3 << 20, o=4 << 20)
        assert gdn.select_kernel(a) == 3


@needs_cuda
def test_recurrent_decode_chain_equals_one_call():
    """Six decode calls with the state updated in place (S_T aliases S0) equal one
    chunked call over the six tokens (SIMT kernel), fp32."""
    import chunked_gated_delta_14_b200 as gdn
    w = workload("plain_fp32", B=2, H=3, T=6, dk=64, dv=64, decay="scalar", s0_std=0.02)
    x = make_inputs(w, seed=19)
    d = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    o_all, s_all = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S0=d["S0"], kernel="simt")
    state = d["S0"].clone()
    outs = []
    for t in range(w.T):
        sl = lambda z: z[:, t:t + 1].contiguous()
        o_t, _ = gdn.chunk_fwd(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["alpha"]), sl(d["beta"]),
                               S0=state, S_T=state, kernel="recurrent")
        outs.append(o_t)
    torch.cuda.synchronize()
    o_cat = torch.cat(outs, dim=1)
    assert (o_cat - o_all).abs().max().item() <= TOL_F32_ABS
    assert (state - s_all).abs().max().item() <= TOL_F32_ABS


@needs_cuda
def test_recurrent_short_sequence_bf16():
    """T = 8, the longest sequence the automatic choice sends to the token kernel,
    with S0: against the oracle."""
    w = workload("gdn_bf16", B=2, H=16, T=8, s0_std=0.02)
    x = make_inputs(w, seed=20)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16("recurrent_T8", w, x, o_ref, s_ref, kernel="recurrent")


# ------------------------------------------------------------ configuration 5

@needs_cuda
@pytest.mark.parametrize("kernel", ["auto", "simt", "tc_split"])
def test_precond_two_gate_small(kernel):
    """auto and tc_split: the SIMT prep writes fp16 rows for the tensor-core chain;
    simt: the fp32 chain."""
    w = workload("precond_two_gate", B=1, H=2, T=300)
    x = make_inputs(w, seed=5)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16(f"precond_small_{kernel}", w, x, o_ref, s_ref, kernel=kernel)


@needs_cuda
@pytest.mark.parametrize("kernel", ["auto", "simt"])
def test_precond_two_gate_full_size(kernel):
    w = workload("precond_two_gate")
    x = make_inputs(w)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16(f"precond_full_{kernel}", w, x, o_ref, s_ref, kernel=kernel)


@needs_cuda
@pytest.mark.parametrize("T,s0,dv", [(1000, 0.02, 128), (4096, 0.0, 64), (65, 0.02, 128), (1, 0.02, 128),
                                     (64, 0.0, 64)])
def test_precond_two_gate_tensor_cores(T, s0, dv):
    """The two-gate rule on the tensor-core chain: ragged tails (a one-token last
    chunk), a single token, one full chunk, an initial state, d_v 64 (one value
    slice), against the oracle."""
    w = workload("precond_two_gate", B=2, H=2, T=T, s0_std=s0, dv=dv)
    x = make_inputs(w, seed=30 + T)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16(f"precond_tc_T{T}_dv{dv}", w, x, o_ref, s_ref, kernel="tc_split")


@needs_cuda
@pytest.mark.parametrize("chunk,T", [(16, 301), (32, 1000), (64, 65)])
def test_precond_two_gate_chunks_ragged(chunk, T):
    """The preconditioner's running average crosses every chunk boundary (chunk
    sums chained over many chunks, a ragged last chunk); the chain kernel runs
    with several value slices."""
    w = workload("precond_two_gate", B=1, H=2, T=T, chunk=chunk)
    x = make_inputs(w, seed=6 + chunk)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16(f"precond_C{chunk}_T{T}", w, x, o_ref, s_ref)


# ------------------------------ page-form preconditioner variants (next row 3)

def _precond_case(w, x, **kw):
    import chunked_gated_delta_14_b200 as gdn
    import oracle
    o_ref, s_ref = oracle.precond_two_gate_fwd(x["q"], x["k"], x["v"], x["alpha"], x["erase"],
                                               x["write"], h0=x["S0"], **kw)
    d = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    o, s = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], None, erase=d["erase"], write=d["write"],
                         S0=d["S0"], o_dtype=torch.float32, **kw)
    torch.cuda.synchronize()
    return o.double().cpu().numpy(), s.double().cpu().numpy(), o_ref, s_ref


@needs_cuda
@pytest.mark.parametrize("form,query", [(2, False), (3, False), (2, True), (3, True), (1, True)])
def test_page_form_preconditioners(form, query):
    """P_t = Diag(A_t)^-1 with the plain running sum (form 2; eps 1 keeps it
    bounded), its squash into [1/2, 2] (form 3), on the write key (ATK) or the
    query (ATQ), on the two-gate engine with per-channel decay and S0."""
    w = workload("precond_two_gate", B=1, H=2, T=300, s0_std=0.02)
    x = make_inputs(w, seed=21)
    kw = dict(precond=form, rho_decay=1.0, rho_eps=1.0 if form == 2 else 1e-6, precond_x=2.0,
              precond_query=query)
    o, s, o_ref, s_ref = _precond_case(w, x, **kw)
    so, ss = stats(o, o_ref), stats(s, s_ref)
    report(f"precond_form{form}_{'atq' if query else 'atk'}", o=so, S_T=ss)
    assert so["max_rel_rms"] <= TOL_BF16_REL_RMS and ss["max_rel_rms"] <= TOL_BF16_REL_RMS


@needs_cuda
def test_squashed_preconditioner_full_size():
    w = workload("precond_two_gate")
    x = make_inputs(w)
    o, s, o_ref, s_ref = _precond_case(w, x, precond=3, rho_decay=1.0, rho_eps=1e-6, precond_x=2.0)
    so, ss = stats(o, o_ref), stats(s, s_ref)
    report("precond_form3_full", o=so, S_T=ss)
    assert so["max_rel_rms"] <= TOL_BF16_REL_RMS and ss["max_rel_rms"] <= TOL_BF16_REL_RMS


# ------------------------------------------------------------------ edges

@needs_cuda
@pytest.mark.parametrize("T", [1, 15, 63, 64, 65, 130])
@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
def test_ragged_lengths_and_chunk_sizes_fp32(T, chunk):
    w = workload("plain_fp32", T=T, chunk=chunk, decay="scalar", s0_std=0.02, H=2)
    x = make_inputs(w, seed=11)
    o_ref, s_ref = run_oracle(x, w)
    o, s = run_gpu(x, w)
    assert np.abs(o - o_ref).max() <= TOL_F32_ABS
    assert np.abs(s - s_ref).max() <= TOL_F32_ABS


@needs_cuda
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128), (32, 16)])
def test_head_dims(dk, dv):
    w = workload("gdn_bf16", B=1, H=2, T=200, dk=dk, dv=dv, s0_std=0.02)
    x = make_inputs(w, seed=12)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16(f"dims_{dk}_{dv}", w, x, o_ref, s_ref)


@needs_cuda
@pytest.mark.parametrize("kernel", ["auto", "simt"])
def test_state_chaining_and_in_place_state(kernel):
    """S_T of the first half fed as S0 of the second equals one call; S_T may alias S0."""
    w = workload("gdn_bf16", B=1, H=4, T=640, s0_std=0.02)
    x = make_inputs(w, seed=13)
    d = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    import chunked_gated_delta_14_b200 as gdn
    o_full, s_full = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S0=d["S0"],
                                   o_dtype=torch.float32, kernel=kernel)
    half = 320
    sl = lambda t: t[:, :half].contiguous()
    sr = lambda t: t[:, half:].contiguous()
    state = d["S0"].clone()
    o1, _ = gdn.chunk_fwd(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["alpha"]), sl(d["beta"]),
                          S0=state, S_T=state, o_dtype=torch.float32, kernel=kernel)
    o2, _ = gdn.chunk_fwd(sr(d["q"]), sr(d["k"]), sr(d["v"]), sr(d["alpha"]), sr(d["beta"]),
                          S0=state, S_T=state, o_dtype=torch.float32, kernel=kernel)
    torch.cuda.synchronize()
    o_cat = torch.cat([o1, o2], dim=1)
    rms = o_full.double().pow(2).mean().sqrt().item()
    assert (o_cat - o_full).abs().max().item() <= 1e-2 * rms
    srms = s_full.double().pow(2).mean().sqrt().item()
    assert (state - s_full).abs().max().item() <= 1e-2 * srms


@needs_cuda
def test_two_gate_engine_reduces_to_gated_delta():
    """Per-channel alpha_t 1, erase alpha_t beta_t, write beta_t, no preconditioner
    on the two-gate path equals the gated delta rule (fp32 io)."""
    w = workload("plain_fp32", B=1, H=2, T=150, decay="scalar", s0_std=0.02)
    x = make_inputs(w, seed=14)
    dk, dv = w.dk, w.dv
    o_ref, s_ref = run_oracle(x, w)
    a = x["alpha"]
    y = dict(x)
    y["alpha"] = a[..., None].expand(*a.shape, dk).contiguous()
    y["erase"] = (a * x["beta"])[..., None].expand(*a.shape, dk).contiguous()
    y["write"] = x["beta"][..., None].expand(*a.shape, dv).contiguous()
    y["beta"] = None
    o, s = run_gpu(y, None, precond=False)
    assert np.abs(o - o_ref).max() <= TOL_F32_ABS
    assert np.abs(s - s_ref).max() <= TOL_F32_ABS


@needs_cuda
def test_neumann_full_series_equals_exact():
    """Neumann mode with N = C - 1 is the exact inverse (Lemma 3.1)."""
    w = workload("gdn_bf16", B=1, H=2, T=256, chunk=32)
    x = make_inputs(w, seed=15)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16("neumann_N_eq_C_minus_1", w.replace(mode="neumann", neumann_N=31), x,
                o_ref, s_ref)


@needs_cuda
@pytest.mark.parametrize("split", [1, 2, 4, 8])
def test_value_split_invariance(split):
    w = workload("gdn_bf16", B=1, H=2, T=300, s0_std=0.02)
    x = make_inputs(w, seed=16)
    o_ref, s_ref = run_oracle(x, w)
    _check_bf16(f"split_{split}", w, x, o_ref, s_ref, dv_split=split)


@needs_cuda
@pytest.mark.parametrize("tc_kernel", ["tc_split", "tc"])
def test_tensor_core_repeatable_after_other_kernels(tc_kernel):
    """Repeated tensor-core calls, each after a SIMT call that leaves other data in
    shared memory, give bit-identical results within the bar: no value may be read
    before it is written, whatever a previous kernel left behind."""
    w = workload("gdn_bf16", B=1, H=2, T=300, s0_std=0.02)
    x = make_inputs(w, seed=16)
    o_ref, s_ref = run_oracle(x, w)
    first = None
    for _ in range(6):
        run_gpu(x, w, o_dtype=torch.float32, kernel="simt", dv_split=1)
        o, s = run_gpu(x, w, o_dtype=torch.float32, kernel=tc_kernel)
        if first is None:
            first = (o, s)
            so = stats(o, o_ref)
            assert so["max_rel_rms"] <= TOL_BF16_REL_RMS, so
        else:
            assert np.array_equal(o, first[0]) and np.array_equal(s, first[1])
