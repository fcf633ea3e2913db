"""GPU parity of the fused tensor-core kernel (one 2-CTA cluster per head).

The key-side CTA of each cluster ships the per-chunk inverses to the chain
CTA through shared memory, so these cases exercise what is particular to it:
ragged lengths (a tail chunk, one chunk, one token), one key-side group idle
(a single chunk), more clusters than fit on the GPU at once, the Neumann
series up to N = C - 1 (Lemma 3.1 of "Quando o 'Bom o Suficiente' e Otimo
...", section "Metodologia": the series is then the exact inverse), agreement
with the split kernels, and bit-identical reruns.  Bar: max |err| <= 2e-2 *
rms(oracle) on o (fp32) and S_T.
"""
import numpy as np
import pytest
import torch

import chunked_gated_delta_14_b200 as gdn
from chunked_gated_delta_14_b200.inputs import make_inputs, workload
from oracle import chunk_forms as cf

from gpu_util import TOL_BF16_REL_RMS, report, run_gpu, run_oracle, stats

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _fused(w):
    """The fused kernel supports the call (forced, as the tests run it; AUTO picks
    the token kernel for T <= 8 instead)."""
    a = gdn.make_args(B=w.B, T=w.T, H=w.H, dk=w.dk, dv=w.dv, chunk=w.chunk, io_dtype=1, o_dtype=0,
                      q=1 << 20, k=2 << 20, v=3 << 20, o=4 << 20, alpha=5 << 20, beta=6 << 20,
                      mode={"exact": 0, "neumann": 1}[w.mode], neumann_N=w.neumann_N, kernel=2)
    return gdn.select_kernel(a) == 2


def _check(name, w, x, o_ref, s_ref, **kw):
    o, s = run_gpu(x, w, o_dtype=torch.float32, kernel="tc", **kw)
    gdn.device_check()
    so, ss = stats(o, o_ref), stats(s, s_ref)
    report(name, o=so, S_T=ss)
    assert so["max_rel_rms"] <= TOL_BF16_REL_RMS, so
    assert ss["max_rel_rms"] <= TOL_BF16_REL_RMS, ss
    return o, s


@needs_cuda
@pytest.mark.parametrize("T", [1, 9, 63, 64, 65, 129, 1000])
def test_fused_ragged_lengths(T):
    w = workload("gdn_bf16", B=2, H=3, T=T, s0_std=0.02)
    assert _fused(w)
    x = make_inputs(w, seed=40 + T)
    o_ref, s_ref = run_oracle(x, w)
    _check(f"fused_T{T}", w, x, o_ref, s_ref)


@needs_cuda
def test_fused_more_clusters_than_fit_at_once():
    """B * H = 160 clusters of two CTAs: more than one wave on 148 SMs."""
    w = workload("gdn_bf16", B=10, H=16, T=300)
    x = make_inputs(w, seed=50)
    o_ref, s_ref = run_oracle(x, w)
    _check("fused_waves", w, x, o_ref, s_ref)


@needs_cuda
@pytest.mark.parametrize("N", [2, 3, 4, 15, 16])
def test_fused_neumann_against_chunk_model(N):
    w = workload("gdn_bf16", B=1, H=4, T=700, s0_std=0.02, mode="neumann", neumann_N=N)
    assert _fused(w)
    x = make_inputs(w, seed=51)
    o_ref, s_ref = run_oracle(x, w)          # chunk model with the masked series
    _check(f"fused_neumann_N{N}", w, x, o_ref, s_ref)


@needs_cuda
def test_fused_neumann_full_series_equals_exact():
    """N = C - 1 = 63: the masked series is the exact inverse (A^C = 0), so the
    fused kernel in Neumann mode meets the bar against the exact recurrence."""
    w = workload("gdn_bf16", B=1, H=2, T=256, mode="neumann", neumann_N=63, decay="weak")
    assert _fused(w)
    x = make_inputs(w, seed=52)
    o_ref, s_ref = run_oracle(x, w.replace(mode="exact"))
    _check("fused_neumann_N63_vs_exact", w, x, o_ref, s_ref)


@needs_cuda
def test_fused_and_split_kernels_agree():
    """The fused kernel and the split kernels compute the same chunk algebra in
    the same operand precision; both meet the bar and stay close to each other."""
    w = workload("gdn_bf16", B=2, H=4, T=1000, s0_std=0.02)
    x = make_inputs(w, seed=53)
    o_ref, s_ref = run_oracle(x, w)
    o_f, s_f = _check("fused_vs_split_fused", w, x, o_ref, s_ref)
    o_s, s_s = run_gpu(x, w, o_dtype=torch.float32, kernel="tc_split")
    so, ss = stats(o_s, o_ref), stats(s_s, s_ref)
    report("fused_vs_split_split", o=so, S_T=ss)
    assert so["max_rel_rms"] <= TOL_BF16_REL_RMS and ss["max_rel_rms"] <= TOL_BF16_REL_RMS
    rms = np.sqrt(np.mean(o_ref ** 2))
    assert np.abs(o_f - o_s).max() <= TOL_BF16_REL_RMS * rms


@needs_cuda
def test_fused_repeatable_bit_identical():
    """No atomics and a fixed order of operations: reruns are bit-identical, also
    after other kernels have left other data in shared memory and TMEM."""
    w = workload("gdn_bf16", B=1, H=4, T=640, s0_std=0.02)
    x = make_inputs(w, seed=54)
    first = None
    for _ in range(5):
        run_gpu(x, w, o_dtype=torch.float32, kernel="simt", dv_split=1)
        run_gpu(x, w, o_dtype=torch.float32, kernel="tc_split")
        o, s = run_gpu(x, w, o_dtype=torch.float32, kernel="tc")
        if first is None:
            first = (o, s)
        else:
            assert np.array_equal(o, first[0]) and np.array_equal(s, first[1])
    gdn.device_check()


@needs_cuda
def test_fused_bf16_output_and_no_final_state():
    """bf16 o (the benchmark's output type) and S_T = NULL."""
    w = workload("gdn_bf16", B=1, H=4, T=500)
    x = make_inputs(w, seed=55)
    o_ref, _ = run_oracle(x, w)
    d = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], o_dtype=torch.bfloat16,
                         kernel="tc", final_state=False)
    torch.cuda.synchronize()
    assert S is None
    from gpu_util import bf16_allowance_ok
    assert bf16_allowance_ok(o.double().cpu().numpy(), o_ref)
