"""Host-side check of bench.py's JSON lines, without a GPU.

torch.cuda is replaced by stand-ins (events that report a fixed time, a
no-op synchronize, CPU tensors in place of device ones) and the kernel calls
by stubs that only ask the real library to validate their arguments.  What
is tested is the line's assembly: every key of the contract is present and
of the right kind, in the forward line (with its backward object) and in the
backward line.  Nothing here measures anything.
"""
import contextlib
import io
import json
import types

import pytest
import torch

import chunked_gated_delta_14_b200 as gdn
import chunked_gated_delta_14_b200.gdn as gmod

CONTRACT = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "clocks",
            "e2e", "gpu_launches", "roofline", "cpu_baseline")


@pytest.fixture
def fake_cuda(monkeypatch):
    class Event:
        def __init__(self, **kw):
            pass

        def record(self, stream=None):
            pass

        def elapsed_time(self, other):
            return 10.0

    class Stream:
        cuda_stream = 0

        def __init__(self, *a, **kw):
            pass

        def wait_event(self, ev):
            pass

    calls = dict(fwd=0, bwd=0)

    def fwd(a, s=None):
        assert gmod.lib().gdn_select_kernel(a) > 0, gmod.last_error()
        calls["fwd"] += 1

    def bwd(a, s=None):
        assert gmod.lib().gdn_bwd_workspace_bytes(a) > 0, gmod.last_error()
        calls["bwd"] += 1

    real_device, real_empty = torch.device, torch.empty

    def empty(*a, **kw):
        kw.pop("pin_memory", None)
        return real_empty(*a, **kw)

    monkeypatch.setattr(torch.cuda, "Event", Event)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda dev=None: Stream())
    monkeypatch.setattr(torch.cuda, "Stream", Stream)
    monkeypatch.setattr(torch.cuda, "stream", lambda st: contextlib.nullcontext())
    monkeypatch.setattr(torch.Tensor, "record_stream", lambda self, st: None)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    monkeypatch.setattr(torch, "device",
                        lambda *a, **k: real_device("cpu") if a and a[0] == "cuda" else real_device(*a, **k))
    monkeypatch.setattr(torch, "empty", empty)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self, *a, **k: self)
    monkeypatch.setattr(gmod, "call", fwd)
    monkeypatch.setattr(gdn, "call", fwd)
    monkeypatch.setattr(gmod, "call_bwd", bwd)
    monkeypatch.setattr(gdn, "call_bwd", bwd)
    monkeypatch.setattr(gmod, "_check", lambda *a, **k: None)
    monkeypatch.setattr(gmod, "device_check", lambda *a, **k: None)
    monkeypatch.setattr(gdn, "device_check", lambda *a, **k: None)
    return calls


def _line(fn, **over):
    import bench
    args = types.SimpleNamespace(steps=2, warmup=3, e2e_steps=4, cpu_budget=0.2, no_cpu_baseline=False,
                                 workload="gdn_bf16", kernel="auto",
                                 batch=1, mode="exact", N=3, S=8, bwd_steps=2, ref_budget=1.0)
    for k, v in over.items():
        setattr(args, k, v)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        getattr(bench, fn)(args, 0, 1, 0)
    return json.loads(buf.getvalue().strip().splitlines()[-1])


def _lines(fn, **over):
    import bench
    args = types.SimpleNamespace(steps=2, warmup=3, e2e_steps=4, cpu_budget=0.2, no_cpu_baseline=False,
                                 workload="gdn_bf16", kernel="auto", batch=1, mode="exact", N=3, S=8,
                                 bwd_steps=0, ref_budget=1.0)
    for k, v in over.items():
        setattr(args, k, v)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        getattr(bench, fn)(args, 0, 1, 0)
    return [json.loads(x) for x in buf.getvalue().strip().splitlines() if x.startswith("{")]


def _check_contract(line):
    for k in CONTRACT:
        assert k in line, k
    assert line["value"] > 0 and line["ms_per_step"] > 0 and line["n_gpus"] == 1
    assert isinstance(line["config"], dict) and "workload" in line["config"]
    r = line["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    e = line["e2e"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0 and e["unit"] == line["unit"]
    assert e["value"] > 0 and e["ms_per_step"] > 0
    c = line["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0 and c["sample"]
    assert line["gpu_launches"] > 0


def test_forward_line_with_backward_object(fake_cuda):
    line = _line("run_gpu")
    _check_contract(line)
    assert line["roofline"]["bound"] == "hbm" and line["gpu_launches"] == 2 * 2  # split kernels: two a step
    b = line["backward"]
    assert "error" not in b, b
    assert b["value"] > 0 and b["gpu_launches"] == 4 * 2 and b["roofline"]["bound"] == "alu"
    assert fake_cuda["fwd"] > 0 and fake_cuda["bwd"] > 0


def test_forward_line_forced_fused_kernel(fake_cuda):
    line = _line("run_gpu", kernel="tc", bwd_steps=0)
    _check_contract(line)
    assert line["config"]["kernel"] == "fused_kernel" and line["gpu_launches"] == 2  # one launch a step


def test_backward_line(fake_cuda):
    line = _line("run_bwd")
    _check_contract(line)
    assert line["roofline"]["bound"] == "alu" and line["gpu_launches"] == 4 * 2
    assert line["dtype"] == "f32"


@pytest.mark.parametrize("mode", ["neumann", "residual"])
def test_backward_line_of_the_series(fake_cuda, mode):
    line = _line("run_bwd", mode=mode, S=2)
    _check_contract(line)
    assert line["gpu_launches"] == 5 * 2 and "bwd_neumann_kernel" in line["config"]["kernel"]
    assert "masked truncated Neumann inverse N=3" in line["config"]["workload"]
    assert ("residual" in line["config"]["workload"]) == (mode == "residual")
    assert line["roofline"]["traffic"] is None          # the committed capture is of the exact mode
    assert "autograd" in line["cpu_baseline"]["sample"]


def test_backward_object_can_be_skipped(fake_cuda):
    line = _line("run_gpu", bwd_steps=0, no_cpu_baseline=True)
    assert line.get("backward") is None and line["cpu_baseline"] is None


def test_decode_line(fake_cuda):
    line = _line("run_decode", batch=8)
    _check_contract(line)
    assert line["roofline"]["bound"] == "hbm" and line["config"]["seq_len"] == 1


def test_e2e_falls_back_to_one_stream(fake_cuda, monkeypatch):
    import bench

    def broken(*a, **k):
        raise RuntimeError("stand-in failure")
    monkeypatch.setattr(bench, "pipelined_e2e", broken)
    line = _line("run_gpu", bwd_steps=0, no_cpu_baseline=True)
    assert line["e2e"]["value"] > 0 and line["e2e"]["pipeline"].startswith("one stream")


@pytest.mark.parametrize("name,kernel,launches", [("plain_fp32", "simt_prep_kernel+simt_chain_kernel", 2),
                                                  ("long_context", "keyside_kernel+chain_kernel", 2),
                                                  ("precond_two_gate", "simt_prep_kernel+chain_kernel", 4)])
def test_other_workload_lines(fake_cuda, monkeypatch, name, kernel, launches):
    import bench
    # the line's assembly only: a stand-in for the oracle timing of a whole long sequence
    from chunked_gated_delta_14_b200 import inputs
    monkeypatch.setattr(bench, "cpu_baseline", lambda w, x, budget_s=0: dict(
        value=1.0, unit="tokens/s", cores=1, kind="oracle", sample="stand-in"))
    if name == "long_context":   # the same line at a shorter length: host memory and time
        monkeypatch.setitem(inputs.WORKLOADS, name, inputs.WORKLOADS[name].replace(T=2048))
    (line,) = _lines("run_gpu", workload=name, cpu_budget=0.05)
    _check_contract(line)
    assert line["config"]["kernel"] == kernel
    assert line["gpu_launches"] == launches * line["steps"]
    assert line["config"]["workload"].startswith(name)
    assert line["metric"] != _line("run_gpu", bwd_steps=0, no_cpu_baseline=True)["metric"]


def test_neumann_sweep_lines(fake_cuda, monkeypatch):
    """One line per chunk 64 / 128 and N 2 / 3 / 4, each with its error against
    exact inversion and against the oracle."""
    import bench
    import numpy as np
    monkeypatch.setattr(bench, "oracle_reference", lambda w, x: (
        np.ones((w.B, w.T, w.H, w.dv)), np.ones((w.B, w.H, w.dk, w.dv))))
    lines = _lines("run_gpu", workload="neumann", cpu_budget=0.05, e2e_steps=0, no_cpu_baseline=True)
    assert len(lines) == 6
    seen = set()
    for ln in lines:
        acc = ln["accuracy"]
        assert set(acc) >= {"vs_exact_inverse", "vs_exact_oracle", "note"}
        seen.add((ln["config"]["workload"].split("chunk=")[1].split()[0],
                  ln["config"]["workload"].split("N=")[1].split(",")[0]))
    assert seen == {(c, n) for c in ("64", "128") for n in ("2", "3", "4")}
