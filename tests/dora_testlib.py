"""Helpers shared by the GPU tests: move generated inputs to the device, run the
library's three calls, run the oracle on the same values, compare.

Tolerances (per output tensor):
  norm C and g          max_i |gpu - ref| / |ref| <= 1e-4   (fp32 outputs)
  g - 1                 max |gpu - ref| <= 1e-3 * max |ref| (near-unity check)
  bf16 y, dm, dA, dB, dx  ||gpu - ref||_F / ||ref||_F <= 2e-2 and cosine >= 0.9999
  fp32 y, dm, dA, dB, dx  ||gpu - ref||_F / ||ref||_F <= 1e-4 and cosine >= 0.9999
  merged weight         element-wise, in tests/test_merge_gpu.py
"""
from __future__ import annotations

import numpy as np

import oracle
from dora_inputs import make_inputs, near_unity_magnitude

NORM_RTOL = 1e-4
GM1_TOL = 1e-3
BF16_RTOL = 2e-2
F32_RTOL = 1e-4
MIN_COSINE = 0.9999


def to_device(inp: dict, device="cuda"):
    import torch
    wl = inp["workload"]
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    out = {}
    for k in ("W0", "A", "B", "x", "dy"):
        if inp.get(k) is not None:
            out[k] = torch.from_numpy(inp[k]).to(device=device).to(dt).contiguous()
    out["m"] = torch.from_numpy(np.asarray(inp["m"], dtype=np.float32)).to(device)
    return out


def prepare(wl, with_backward=True):
    """Generate inputs; for near-unity workloads set m = C (1 + delta) from the oracle's C."""
    inp = make_inputs(wl, with_backward=with_backward)
    if inp["m"] is None:
        C, _, _ = oracle.norm(inp["W0"], inp["A"], inp["B"], np.ones(wl.d_out), inp["s"])
        inp["m"] = near_unity_magnitude(C, inp["delta"])
    return inp


def run_gpu(dev: dict, s: float, need_dx=True):
    import dora_weight_decomposed_b200 as dw
    norm, g, gm1 = dw.dora_norm(dev["W0"], dev["A"], dev["B"], dev["m"], s)
    y, su, pre = dw.dora_forward(dev["x"], dev["W0"], dev["A"], dev["B"], gm1, s)
    out = {"C": norm, "g": g, "gm1": gm1, "y": y, "su": su, "pre": pre}
    if "dy" in dev:
        dm, dA, dB, dx = dw.dora_backward(dev["dy"], dev["x"], dev["W0"], dev["A"], dev["B"], norm, g, su, pre, s,
                                          need_dx=need_dx)
        out.update(dm=dm, dA=dA, dB=dB, dx=dx)
    return out


def run_oracle(inp: dict, with_backward=True):
    W0, A, B, m, s, x = (inp[k] for k in ("W0", "A", "B", "m", "s", "x"))
    C, g, gm1 = oracle.norm(W0, A, B, m, s)
    ref = {"C": C, "g": g, "gm1": gm1, "y": oracle.forward(x, W0, A, B, m, s)}
    if with_backward:
        ref.update(oracle.backward(inp["dy"], x, W0, A, B, m, s))
    return ref


def host(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_fro(a, b) -> float:
    den = float(np.linalg.norm(b))
    return float(np.linalg.norm(a - b)) / (den if den > 0 else 1.0)


def cosine(a, b) -> float:
    na, nb = float(np.linalg.norm(a)), float(np.linalg.norm(b))
    if na == 0 and nb == 0:
        return 1.0
    return float(np.dot(a.ravel(), b.ravel()) / (na * nb))


def check_norms(out: dict, ref: dict, what=""):
    for k in ("C", "g"):
        a, b = host(out[k]), ref[k]
        err = float(np.max(np.abs(a - b) / np.abs(b)))
        assert err <= NORM_RTOL, f"{what} {k}: max rel err {err:.3e} > {NORM_RTOL}"
    a, b = host(out["gm1"]), ref["gm1"]
    err = float(np.max(np.abs(a - b)))
    assert err <= GM1_TOL * float(np.max(np.abs(b))), f"{what} gm1: max abs err {err:.3e}"


def check_tensor(name, gpu_t, ref, dtype: str, what=""):
    a = host(gpu_t)
    b = np.asarray(ref, dtype=np.float64)
    assert a.shape == b.shape, f"{what} {name}: shape {a.shape} vs {b.shape}"
    assert np.all(np.isfinite(a)), f"{what} {name}: non-finite values"
    rtol = BF16_RTOL if dtype == "bf16" else F32_RTOL
    e = rel_fro(a, b)
    c = cosine(a, b)
    assert e <= rtol and c >= MIN_COSINE, f"{what} {name}: rel err {e:.3e} (tol {rtol}), cosine {c:.6f}"
    return e, c


def check_all(out: dict, ref: dict, dtype: str, what="", backward=True):
    check_norms(out, ref, what)
    report = {"y": check_tensor("y", out["y"], ref["y"], dtype, what)}
    if backward:
        for k in ("dm", "dA", "dB", "dx"):
            if out.get(k) is not None:
                report[k] = check_tensor(k, out[k], ref[k], dtype, what)
    return report
