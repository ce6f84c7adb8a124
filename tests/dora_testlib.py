"""Helpers shared by the GPU tests: move generated inputs to the device, run the
library's three calls on NaN-filled output buffers, run the oracle on the same
values, compare.

Tolerances (per output tensor), all checked together:

  norm C and g          max_i |gpu - ref| / |ref| <= 1e-4   (fp32 outputs)
  g - 1                 max |gpu - ref| <= 1e-3 * max |ref| (near-unity check)
  y, dm, dA, dB, dx     ||gpu - ref||_F / ||ref||_F <= 2e-2 (bf16) or 1e-4 (fp32) and cosine >= 0.9999
                        every element within its own rounding-error bound (below)
                        every row of y, dA, dB, dx within the Frobenius tolerance
  merged weight         element-wise, in tests/test_merge_gpu.py

Element bounds. Each output is a dot product o = sum_k a_k b_k of stored
operands; the GPU rounds some operands to the storage type before the product
(s*u, dz, du, pre), accumulates in fp32 and rounds the result once. With unit
roundoff u (2^-8 for bf16, 2^-24 for fp32):

  * the final rounding moves o by at most u |o|;
  * operands rounded as a_k (1 + d_k), |d_k| <= u, with the d_k independent
    and of mean zero (round to nearest even on continuous data), move o by
    sum_k d_k a_k b_k, which Hoeffding's inequality bounds by
    lam u sqrt(sum_k a_k^2 b_k^2) except with probability 2 exp(-lam^2 / 2);
  * fp32 accumulation over K terms stays within lam sqrt(K) u_acc sum_k |a_k b_k|
    <= lam sqrt(K) u_acc ||a||_2 ||b||_2 with the same probability (the
    probabilistic rounding-error bound of Higham and Mary, 2019; Cauchy-Schwarz
    for the sum of magnitudes), u_acc = 2^-23 so truncating adds are covered;
  * g, C and g - 1 enter as the GPU's own fp32 values, whose measured errors
    (checked first, against 1e-4) are carried into the bound column by column.

lam = 8: each element's bound fails by chance with probability below 3e-14.
Where a sum of squares would need a full-size product (sum_i dz_ti^2 W0_ik^2),
Hoelder's inequality replaces it by ||dz_t||_4 ||W'_k||_4. The bounds are
derived term by term in the functions below.
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
LAM = 8.0
U_ACC = 2.0 ** -23
UNIT_ROUNDOFF = {"bf16": 2.0 ** -8, "fp32": 2.0 ** -24}


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


def poisoned(shape, dtype, device="cuda"):
    """An output buffer filled with NaN: any element a kernel fails to write stays NaN."""
    import torch
    return torch.full(tuple(shape), float("nan"), dtype=dtype, device=device)


def run_gpu(dev: dict, s: float, need_dx=True):
    """The three calls, every output (and the saved s*u and pre) in a NaN-filled buffer."""
    import torch
    import dora_weight_decomposed_b200 as dw
    W0, A, x = dev["W0"], dev["A"], dev["x"]
    dt, d = W0.dtype, W0.device
    d_out, d_in = W0.shape
    r, T = A.shape[0], x.shape[0]
    f32 = torch.float32
    norm, g, gm1 = dw.dora_norm(W0, A, dev["B"], dev["m"], s, norm_out=poisoned((d_out,), f32, d),
                                g_out=poisoned((d_out,), f32, d), gm1_out=poisoned((d_out,), f32, d))
    y, su, pre = dw.dora_forward(x, W0, A, dev["B"], gm1, s, y=poisoned((T, d_out), dt, d),
                                 su_save=poisoned((T, r), dt, d), pre_save=poisoned((T, d_out), dt, d))
    out = {"C": norm, "g": g, "gm1": gm1, "y": y, "su": su, "pre": pre}
    if "dy" in dev:
        dm, dA, dB, dx = dw.dora_backward(dev["dy"], x, W0, A, dev["B"], norm, g, su, pre, s, need_dx=need_dx,
                                          dm=poisoned((d_out,), f32, d), dA=poisoned((r, d_in), dt, d),
                                          dB=poisoned((d_out, r), dt, d),
                                          dx=poisoned((T, d_in), dt, d) if need_dx else None)
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
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
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
        assert np.all(np.isfinite(a)), f"{what} {k}: non-finite values"
        err = float(np.max(np.abs(a - b) / np.abs(b))) if a.size else 0.0
        assert err <= NORM_RTOL, f"{what} {k}: max rel err {err:.3e} > {NORM_RTOL}"
    a, b = host(out["gm1"]), ref["gm1"]
    assert np.all(np.isfinite(a)), f"{what} gm1: non-finite values"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= GM1_TOL * float(np.max(np.abs(b))), f"{what} gm1: max abs err {err:.3e}"


def check_tensor(name, gpu_t, ref, dtype: str, what=""):
    """Normwise: ||gpu - ref||_F / ||ref||_F and cosine (the stated tolerance)."""
    a = host(gpu_t)
    b = np.asarray(ref, dtype=np.float64)
    assert a.shape == b.shape, f"{what} {name}: shape {a.shape} vs {b.shape}"
    assert np.all(np.isfinite(a)), f"{what} {name}: {int(np.sum(~np.isfinite(a)))} non-finite values"
    rtol = BF16_RTOL if dtype == "bf16" else F32_RTOL
    e = rel_fro(a, b)
    c = cosine(a, b)
    assert e <= rtol and c >= MIN_COSINE, f"{what} {name}: rel err {e:.3e} (tol {rtol}), cosine {c:.6f}"
    return e, c


def check_rows(name, gpu_t, ref, dtype: str, what=""):
    """Every row (first index) within the Frobenius tolerance of its own norm."""
    a = host(gpu_t)
    b = np.asarray(ref, dtype=np.float64)
    if b.size == 0:
        return
    rtol = BF16_RTOL if dtype == "bf16" else F32_RTOL
    den = np.sqrt(np.sum(b * b, axis=1))
    num = np.sqrt(np.sum((a - b) ** 2, axis=1))
    bad = ~(num <= rtol * np.maximum(den, 1e-300))
    # Rows of exact zeros (e.g. dA for an all-zero column of du) compare absolutely.
    bad &= ~((den == 0) & (num == 0))
    assert not bad.any(), (f"{what} {name}: {int(bad.sum())} rows over {rtol} relative, "
                           f"first row {int(np.argmax(bad))}: {num[bad][0]:.3e} vs norm {den[bad][0]:.3e}")


def check_elementwise(name, gpu_t, ref, bound, what=""):
    """|gpu - ref| <= bound element by element (NaN fails)."""
    a = host(gpu_t)
    b = np.asarray(ref, dtype=np.float64)
    assert a.shape == b.shape == bound.shape, f"{what} {name}: shapes {a.shape} {b.shape} {bound.shape}"
    bad = ~(np.abs(a - b) <= bound)
    if bad.any():
        i = tuple(int(v) for v in np.argwhere(bad)[0])
        raise AssertionError(f"{what} {name}: {int(bad.sum())} of {bad.size} elements outside their rounding "
                             f"bound; first at {i}: got {a[i]:.6g}, oracle {b[i]:.6g}, bound {bound[i]:.3g}")


# ---------------------------------------------------------------- element bounds

def _n2(M, axis):
    return np.sqrt(np.sum(M * M, axis=axis))


def _n4(M, axis):
    return np.sqrt(np.sqrt(np.sum((M * M) ** 2, axis=axis)))


def element_bounds(inp: dict, ref: dict, out: dict, dtype: str) -> dict:
    """Per-element error bounds of y, dm, dA, dB, dx and s*u for the GPU's arithmetic.

    The GPU computes, with [.] a rounding to the storage type:
      su = [s x A^T]   pre = [x W0^T + su B^T] (stored)   y = [pre32 + gm1 pre32]
      dz = [g dy]      du = [s dz B]      dB = [dz^T su]   dA = [du^T x]
      dm = sum_t dy pre / C                dx = [dz W0 + du A]
    and the oracle the same quantities exactly in float64. Term names follow
    the rules in the module docstring: rnd (final rounding), op (operand
    roundings, Hoeffding), acc (fp32 accumulation), gerr (the GPU's g, g - 1, C).
    Large terms are accumulated in place to keep the host memory of the
    largest workload bounded.
    """
    u = UNIT_ROUNDOFF[dtype]
    lam = LAM
    f = lambda k: np.asarray(inp[k], dtype=np.float64)
    x, W0, A, B, s = f("x"), f("W0"), f("A"), f("B"), float(inp["s"])
    T, d_in = x.shape
    d_out, r = B.shape
    sa = abs(s)
    g = ref["g"]
    # Measured per-row errors of the GPU's fp32 scale factors (checked against 1e-4 beforehand).
    eg = np.abs(host(out["g"]) - g)
    egm1 = np.abs(host(out["gm1"]) - ref["gm1"])
    eC = np.abs(host(out["C"]) - ref["C"])
    su = s * (x @ A.T)
    n2x, n2A, n2B, n2W0, n2su = _n2(x, 1), _n2(A, 1), _n2(B, 1), _n2(W0, 1), _n2(su, 1)
    absB_n2A = np.abs(B) @ n2A  # sum_j |B_ij| ||A_j||: carries s u's accumulation error into pre
    bd = {}
    # s u: rnd + acc over d_in.
    bd["su"] = u * np.abs(su) + lam * np.sqrt(d_in) * U_ACC * sa * np.outer(n2x, n2A)
    # Worst-case fp32 accumulation error of pre_ti (over d_in + r, plus s u's own through B).
    def pre_acc():
        t = np.outer(n2x, n2W0)
        t += np.outer(n2su, n2B)
        t *= lam * np.sqrt(d_in + r) * U_ACC
        t += (lam * np.sqrt(d_in) * U_ACC * sa) * np.outer(n2x, absB_n2A)
        return t
    # y = (1 + gm1) pre:  rnd u|y|; gerr |d gm1_i| |pre|; op (s u rounded)
    #   lam u sqrt(sum_j su_tj^2 B_ij^2); acc of pre; all but rnd scaled by g_i.
    y = ref["y"]
    pre = y / g[None, :]
    b = np.sqrt((su * su) @ (B * B).T)
    b *= lam * u
    b += pre_acc()
    b *= g[None, :]
    b += (u + 2.0 ** -23) * np.abs(y)
    b += egm1[None, :] * np.abs(pre)
    bd["y"] = b
    if "dm" not in ref:
        return bd
    dy = f("dy")
    C = ref["C"]
    # dm_i = sum_t dy_ti pre_ti / C_i with pre stored (rounded) and C the GPU's:
    #   op: pre's rounding lam u sqrt(sum_t dy^2 pre^2); s u's rounding inside pre,
    #       lam u sqrt(sum_{t,j} dy_ti^2 su_tj^2 B_ij^2); acc of pre (worst case over t); acc of dm.
    M = (dy * dy).T @ (su * su)
    dm = ref["dm"]
    abs_dy = np.abs(dy)
    dm_acc_pre = lam * np.sqrt(d_in + r) * U_ACC * (n2W0 * (abs_dy.T @ n2x) + n2B * (abs_dy.T @ n2su)) \
        + lam * np.sqrt(d_in) * U_ACC * sa * absB_n2A * (abs_dy.T @ n2x)
    bd["dm"] = ((2.0 ** -23 + eC / C) * np.abs(dm)
                + (lam * u * np.sqrt(np.sum((dy * pre) ** 2, axis=0))
                   + lam * u * np.sqrt(np.sum(B * B * M, axis=1))
                   + dm_acc_pre
                   + lam * np.sqrt(max(T, 1)) * U_ACC * _n2(dy, 0) * _n2(pre, 0)) / C)
    del pre, abs_dy
    dz = dy * g[None, :]
    del dy
    du = s * (dz @ B)
    n2dz = _n2(dz, 1)
    n2Bc = _n2(B, 0)
    # dB_ij = sum_t dz_ti su_tj: rnd; gerr (g_i scales row i); op (dz and s u rounded, |d| <= 2u);
    #   acc over T; s u's own acc carried through dz (worst case over t).
    dB = ref["dB"]
    bd["dB"] = ((u + (eg / g)[:, None]) * np.abs(dB) + lam * 2 * u * np.sqrt((dz * dz).T @ (su * su))
                + lam * np.sqrt(max(T, 1)) * U_ACC * np.outer(_n2(dz, 0), _n2(su, 0))
                + lam * np.sqrt(d_in) * U_ACC * sa * np.outer(np.abs(dz).T @ n2x, n2A))
    # du_tj = s sum_i dz_ti B_ij (stored, rounded); dA_jk = sum_t du_tj x_tk:
    #   op: du's rounding lam u sqrt(sum_t du^2 x^2); dz's rounding through du,
    #       lam u |s| sqrt(sum_{t,i} x_tk^2 dz_ti^2 B_ij^2); gerr through du (worst case);
    #   acc of du over d_out (worst case over t) and of dA over T; rnd.
    dA = ref["dA"]
    rel_g = (eg / g)[None, :]
    bd["dA"] = (u * np.abs(dA) + lam * u * np.sqrt((du * du).T @ (x * x))
                + lam * u * sa * np.sqrt(((x * x).T @ ((dz * dz) @ (B * B))).T)
                + sa * (np.abs(x).T @ ((np.abs(dz) * rel_g) @ np.abs(B))).T
                + lam * np.sqrt(d_out) * U_ACC * sa * np.outer(n2Bc, np.abs(x).T @ n2dz)
                + lam * np.sqrt(max(T, 1)) * U_ACC * np.outer(_n2(du, 0), _n2(x, 0)))
    # dx_tk = sum_i dz_ti W0_ik + sum_j du_tj A_jk:
    #   op: dz's rounding reaches dx through W0 and, via du, through s B A, i.e. through W';
    #       lam u ||dz_t||_4 ||W'_:k||_4 (Hoelder); du's rounding lam u sqrt(sum_j du^2 A^2);
    #   gerr (worst case, Cauchy-Schwarz); acc of du carried through A; acc of dx; rnd.
    Vp = oracle.adapted_direction(W0, A, B, s)
    n4Vp, n2Vp = _n4(Vp, 0), _n2(Vp, 0)
    del Vp
    n4dz = _n4(dz, 1)
    dx = ref["dx"]
    b = np.sqrt((du * du) @ (A * A))
    b *= lam * u
    b += (u + 2.0 ** -23) * np.abs(dx)
    b += lam * u * np.outer(n4dz, n4Vp)
    b += float(np.max(eg / g)) * np.outer(n2dz, n2Vp)
    b += lam * np.sqrt(d_out) * U_ACC * sa * np.outer(n2dz, n2Bc @ np.abs(A))
    b += lam * np.sqrt(d_out + r) * U_ACC * (np.outer(n2dz, _n2(W0, 0)) + np.outer(_n2(du, 1), _n2(A, 0)))
    bd["dx"] = b
    return bd


def check_all(out: dict, ref: dict, inp: dict, what="", backward=True):
    """Norms, then y (and the gradients): normwise, per row and element by element."""
    dtype = inp["workload"].dtype
    check_norms(out, ref, what)
    bd = element_bounds(inp, ref, out, dtype)
    report = {}
    names = ["y"] + (["dm", "dA", "dB", "dx"] if backward else [])
    for k in names:
        if out.get(k) is None:
            continue
        report[k] = check_tensor(k, out[k], ref[k], dtype, what)
        if k != "dm":
            check_rows(k, out[k], ref[k], dtype, what)
        check_elementwise(k, out[k], ref[k], bd[k], what)
    return report


def check_near_unity(y_gpu, inp: dict, ref: dict, what=""):
    """Near-unity layers (g = 1 + O(1e-3)): the adapted part must survive in y.

    1. y - x W0^T against the oracle's y - x W0^T, every token row normwise within 2e-2 of its
       norm plus y's own bf16 rounding (u ||y_row||), which at g - 1 ~ 1e-3 is the larger term.
    2. The effective g - 1 carried by y: per output feature i the least-squares scale of the
       deviation, beta_i = <y_:i - pre_:i, pre_:i> / ||pre_:i||^2 (pre = y_ref / g), regressed on the
       oracle's g - 1 over all features. The slope must be 1 within a Hoeffding bound (lam = 8) on
       y's rounding errors (|e_ti| <= u |y_ti|), and that bound must be small enough (< 0.5) that
       a y built from a rounded g (g - 1 quantised to 0, slope 0) fails.
    """
    u = UNIT_ROUNDOFF[inp["workload"].dtype]
    a = host(y_gpu)
    x, W0 = inp["x"].astype(np.float64), inp["W0"].astype(np.float64)
    base = x @ W0.T
    d_got, d_ref = a - base, ref["y"] - base
    num = np.sqrt(np.sum((d_got - d_ref) ** 2, axis=1))
    lim = BF16_RTOL * np.sqrt(np.sum(d_ref ** 2, axis=1)) + u * np.sqrt(np.sum(ref["y"] ** 2, axis=1))
    assert np.all(num <= lim), f"{what}: y - x W0^T off in {int(np.sum(num > lim))} rows"
    pre = ref["y"] / ref["g"][None, :]
    pp = np.sum(pre * pre, axis=0)
    beta = np.sum((a - pre) * pre, axis=0) / pp
    gm1 = ref["gm1"]
    den = float(np.sum(gm1 * gm1))
    slope = float(np.sum(beta * gm1)) / den
    bound = LAM * u * float(np.sqrt(np.sum(gm1 * gm1 * np.sum(ref["y"] ** 2 * pre * pre, axis=0) / pp ** 2))) / den
    assert bound < 0.5, f"{what}: too few tokens to resolve g - 1 (bound {bound:.3f})"
    assert abs(slope - 1.0) <= bound, f"{what}: y carries g - 1 with slope {slope:.4f} (bound {bound:.4f})"
    return slope, bound
