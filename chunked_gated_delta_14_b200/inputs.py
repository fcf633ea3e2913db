"""Seeded synthetic workloads for the chunked gated delta-rule forward.

This module only draws and shapes random tensors; it holds none of the
method's arithmetic.  Both the CUDA path and the fp64 oracle are fed from
here, so the two sides always see bit-identical inputs.

Recipe (one ``numpy.random.Generator(PCG64(seed))`` per workload, every draw
fp32 standard normal; draw order q, k, v, beta, alpha-noise, S0, erase, write,
skipping the ones a workload does not use):

* q, k: N(0, 1), then L2-normalised per (token, head) over d_k in fp32
  (x / ||x||_2, no epsilon), then rounded to the io dtype (round to nearest
  even for bf16).
* v: N(0, 1), rounded to the io dtype.
* beta = sigmoid(N(0, 1)), fp32, shape [B, T, H].
* alpha = exp(-softplus(N(0, 1) + 2)), fp32, shape [B, T, H] (scalar decay)
  or [B, T, H, d_k] (per key channel).  ``None`` means alpha == 1.  The
  "weak" scalar decay, the regime of trained Gated DeltaNet layers whose gates
  sit close to 1, draws alpha = 0.9 + 0.1 U[0, 1) (fp32 uniform) in the same
  slot instead.
* S0 ~ N(0, 0.02^2) (0.02 is the standard deviation), fp32 [B, H, d_k, d_v].
* erase gate b and write gate w = sigmoid(N(0, 1)) in the io dtype,
  shapes [B, T, H, d_k] and [B, T, H, d_v].

Cotangents for the backward pass (``make_cotangents``) come from a second
generator, ``PCG64([seed, 1])``, so drawing them never shifts the forward
inputs: grad_o ~ N(0, 1) rounded to the io dtype, [B, T, H, d_v]; grad_S_T ~
N(0, 0.02^2), fp32 [B, H, d_k, d_v] (the scale of S0).

The workloads are the Gated DeltaNet layer shapes the pages discuss
(1.3B-class head geometry: H=16, d_k=d_v=128); no dataset is involved.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "make_cotangents", "make_inputs", "workload"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int
    io: str                 # "f32" or "bf16"
    decay: str              # "none" | "scalar" | "weak" | "channel"
    beta: bool              # scalar write strength beta_t present
    s0_std: float           # 0 -> no initial state
    gates: bool             # erase/write channel gates present
    precond: bool           # diagonal curvature preconditioned write key
    mode: str = "exact"     # "exact" | "neumann"
    neumann_N: int = 3

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.H


WORKLOADS = {
    # Plain delta rule, fp32, alpha == 1, no initial state.
    "plain_fp32": Workload("plain_fp32", B=1, H=1, T=256, dk=64, dv=64, chunk=64,
                           io="f32", decay="none", beta=True, s0_std=0.0,
                           gates=False, precond=False),
    # Gated DeltaNet layer, 1.3B-class head shape.
    "gdn_bf16": Workload("gdn_bf16", B=4, H=16, T=4096, dk=128, dv=128, chunk=64,
                         io="bf16", decay="scalar", beta=True, s0_std=0.0,
                         gates=False, precond=False),
    # Long-context state carry with a random initial state.
    "long_context": Workload("long_context", B=1, H=16, T=65536, dk=128, dv=128,
                             chunk=64, io="bf16", decay="scalar", beta=True,
                             s0_std=0.02, gates=False, precond=False),
    # Truncated Neumann inverse on the gdn_bf16 inputs (chunk and N are swept).
    "neumann": Workload("neumann", B=4, H=16, T=4096, dk=128, dv=128, chunk=64,
                        io="bf16", decay="scalar", beta=True, s0_std=0.0,
                        gates=False, precond=False, mode="neumann", neumann_N=3),
    # Preconditioned write key, per-channel decay, erase/write channel gates.
    "precond_two_gate": Workload("precond_two_gate", B=2, H=16, T=4096, dk=128,
                                 dv=128, chunk=64, io="bf16", decay="channel",
                                 beta=False, s0_std=0.0, gates=True, precond=True),
}


def workload(name: str, **overrides) -> Workload:
    return WORKLOADS[name].replace(**overrides)


def _round_io(x: np.ndarray, io: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if io == "bf16":
        return t.to(torch.bfloat16)
    if io == "f32":
        return t
    raise ValueError(f"unknown io dtype {io!r}")


def _l2_normalise(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float32) ** 2, axis=-1, keepdims=True, dtype=np.float32))
    return (x / n).astype(np.float32)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float32)))).astype(np.float32)


def _decay(x: np.ndarray) -> np.ndarray:
    # exp(-softplus(x + 2)) == 1 / (1 + exp(x + 2)), evaluated stably in fp32.
    z = x.astype(np.float32) + np.float32(2.0)
    sp = np.logaddexp(np.float32(0.0), z).astype(np.float32)
    return np.exp(-sp).astype(np.float32)


def make_inputs(w: Workload, seed: int = 0) -> dict:
    """Draw the tensors of workload ``w`` on the CPU.

    Returns a dict of CPU torch tensors: q, k, v (io dtype), alpha (fp32 or
    None), beta (fp32 or None), S0 (fp32 or None), erase, write (io dtype or
    None).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv

    def normal(shape):
        return rng.standard_normal(size=shape, dtype=np.float32)

    q = _round_io(_l2_normalise(normal((B, T, H, dk))), w.io)
    k = _round_io(_l2_normalise(normal((B, T, H, dk))), w.io)
    v = _round_io(normal((B, T, H, dv)), w.io)
    beta = torch.from_numpy(_sigmoid(normal((B, T, H)))) if w.beta else None
    alpha: Optional[torch.Tensor]
    if w.decay == "none":
        alpha = None
    elif w.decay == "scalar":
        alpha = torch.from_numpy(_decay(normal((B, T, H))))
    elif w.decay == "weak":
        u = rng.random(size=(B, T, H), dtype=np.float32)
        alpha = torch.from_numpy((np.float32(0.9) + np.float32(0.1) * u).astype(np.float32))
    elif w.decay == "channel":
        alpha = torch.from_numpy(_decay(normal((B, T, H, dk))))
    else:
        raise ValueError(w.decay)
    S0 = (torch.from_numpy(normal((B, H, dk, dv)) * np.float32(w.s0_std))
          if w.s0_std > 0 else None)
    erase = write = None
    if w.gates:
        erase = _round_io(_sigmoid(normal((B, T, H, dk))), w.io)
        write = _round_io(_sigmoid(normal((B, T, H, dv))), w.io)
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta, S0=S0, erase=erase, write=write)


def make_cotangents(w: Workload, seed: int = 0, grad_state: bool = True) -> dict:
    """Draw dL/do (io dtype) and dL/dS_T (fp32, or None) for workload ``w``."""
    rng = np.random.Generator(np.random.PCG64([seed, 1]))
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    do = _round_io(rng.standard_normal(size=(B, T, H, dv), dtype=np.float32), w.io)
    dS = (torch.from_numpy(rng.standard_normal(size=(B, H, dk, dv), dtype=np.float32)
                           * np.float32(0.02)) if grad_state else None)
    return dict(grad_o=do, grad_S_T=dS)
