"""Helpers for the GPU parity tests: run the CUDA path, compare with the oracle."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import chunked_gated_delta_14_b200 as gdn
import oracle
from oracle import chunk_forms as cf

# Tolerances from the method's accuracy bar: fp32 configurations must match
# the fp64 oracle to 1e-4 absolute; bf16 configurations to 2e-2 of the
# oracle's RMS in the maximum absolute error, for o and for S_T.
TOL_F32_ABS = 1e-4
TOL_BF16_REL_RMS = 2e-2
# A bf16 output cannot be closer to the oracle than its own rounding: the
# bf16-o checks allow one bf16 ulp of |reference| on top of the bar.
BF16_ULP_REL = 2.0 ** -8


def to_dev(x):
    return None if x is None else x.to("cuda").contiguous()


def run_gpu(x, w=None, **kw):
    """Call the CUDA path on inputs ``x`` (CPU tensors). Returns float64 numpy o, S_T."""
    d = {k: to_dev(v) for k, v in x.items()}
    args = dict(chunk=w.chunk if w else 64)
    if w is not None:
        args.update(mode=w.mode, N=w.neumann_N)
        if w.precond or w.gates or w.decay == "channel":
            args.update(precond=w.precond)
    args.update(kw)
    o, S = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], erase=d["erase"],
                         write=d["write"], S0=d["S0"], **args)
    torch.cuda.synchronize()
    return o.double().cpu().numpy(), S.double().cpu().numpy()


def run_oracle(x, w):
    if w.gates or w.precond or w.decay == "channel":
        return oracle.precond_two_gate_fwd(x["q"], x["k"], x["v"], x["alpha"], x["erase"],
                                           x["write"], precond=w.precond, h0=x["S0"])
    if w.mode == "neumann":
        return cf.chunked_gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"],
                                          x["S0"], chunk=w.chunk,
                                          inverse=cf.neumann_inverse(w.neumann_N))
    return oracle.gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"])


def stats(got, ref):
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    e2 = float(np.sum(err ** 2))
    return dict(max_abs=float(err.max()), rms_ref=rms,
                max_rel_rms=float(err.max() / rms) if rms > 0 else float(err.max()),
                rms_rel=float(np.sqrt(np.mean(err ** 2)) / rms) if rms > 0 else 0.0,
                snr_db=float(10 * np.log10(np.sum(ref ** 2) / e2)) if e2 > 0 else float("inf"))


def bf16_allowance_ok(got, ref, rel_rms=TOL_BF16_REL_RMS):
    rms = np.sqrt(np.mean(ref ** 2))
    return bool(np.all(np.abs(got - ref) <= rel_rms * rms + BF16_ULP_REL * np.abs(ref)))


def report(name, **fields):
    path = os.environ.get("GDN_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(dict(test=name, **fields)) + "\n")
