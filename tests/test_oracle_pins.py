"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

Each pin is a function of an oracle-like object so that the same pins can be
run against deliberately broken copies of the oracle (planted on the CPU, at
the end of this file) to show that a plausible mistake fails at least one pin.

What pins what:
  golden      hand-derived examples (tests/golden/dora_hand_examples.json),
              every output including the full gradient and the merge
  factored    the oracle's dense norm equals base + cross + Gram
              (Scaling DoRA abstract) on random inputs
  factored_norm  norm_factored (the factored form without the dense B A) gives
              the dense norm's C, g, g - 1, the golden values, and
              C = |W0_i| at B = 0 (numpy.linalg.norm)
  zero_B      B = 0 gives C = |W0_i| and g = m / |W0_i| (numpy.linalg.norm)
  init        B = 0 and m = |W0_i| gives y = x W0^T (DoRA notes sec. 3.1:
              training starts from the pretrained weight)
  scale       (a W0, a B) leaves y, dm, dx and dA unchanged and divides dB by a
              (eq. (6) is invariant under a common scale of W0 + sBA)
  merge       y equals x W_merged^T and the merged rows have length m
              (Algorithm 1 steps 16-17)
  fd_x_m      central finite differences of L = sum(dy * y) in x and m
  fd_detached finite differences with the norm held fixed give dA, dB
              (detach, DoRA notes sec. 3.4)
  fd_full     finite differences of the true L give the eq. (A.1) gradient
  a2_term     detached minus full dV equals the dropped term (A.2)
  eq8         dm_n = |grad W'_n| cos(grad W'_n, V'_n) (eq. (8), second form)
  near_unity  m = C (1 + delta) gives g - 1 = delta
  vera_fd     DVoRA (DoRA notes sec. 3.5): finite differences of L in the
              trained vectors b and d, with the norm held fixed and free, give
              vera_gradients of the detached and the full dB'
  vera_unit   b = 1 and d = 1 reduce DVoRA to DoRA with B = B_shared, and
              B' scales each row by b and each column by d
"""
import json
import os
import types

import numpy as np
import pytest

import oracle
from dora_inputs import make_inputs, round_to_bf16, workload, near_unity_magnitude

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "dora_hand_examples.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)["examples"]


def _rand_layer(rng, d_out, d_in, r, T, s=0.7):
    return dict(W0=rng.standard_normal((d_out, d_in)), A=rng.standard_normal((r, d_in)) * 0.5,
                B=rng.standard_normal((d_out, r)) * 0.5, m=rng.uniform(0.5, 2.0, d_out),
                x=rng.standard_normal((T, d_in)), dy=rng.standard_normal((T, d_out)), s=s)


def _close(a, b, rtol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= rtol * scale, f"{what}: max abs err {err:.3e} > {rtol:.1e} * {scale:.3e}"


# ----------------------------------------------------------------------------- pins

def pin_golden(orc):
    for ex in _golden():
        e = ex["expected"]
        W0, A, B, m, x, dy, s = (np.array(ex[k], dtype=np.float64) for k in
                                 ("W0", "A", "B", "m", "x", "dy", "s"))
        s = float(s)
        C, g, gm1 = orc.norm(W0, A, B, m, s)
        _close(C, e["C"], 1e-14, "C")
        _close(g, e["g"], 1e-14, "g")
        _close(gm1, e["gm1"], 1e-14, "gm1")
        _close(orc.forward(x, W0, A, B, m, s), e["y"], 1e-14, "y")
        gr = orc.backward(dy, x, W0, A, B, m, s)
        for k in ("dm", "dA", "dB", "dx"):
            _close(gr[k], e[k], 1e-14, k)
        gf = orc.backward(dy, x, W0, A, B, m, s, full=True)
        _close(gf["dA"], e["dA_full"], 1e-14, "dA_full")
        _close(gf["dB"], e["dB_full"], 1e-14, "dB_full")
        _close(gf["dm"], e["dm"], 1e-14, "dm_full")
        _close(gf["dx"], e["dx"], 1e-14, "dx_full")
        if "merged" in e:
            _close(orc.merge(W0, A, B, m, s), e["merged"], 1e-14, "merged")


def pin_factored(orc):
    rng = np.random.default_rng(7)
    for (d_out, d_in, r) in [(5, 7, 3), (16, 40, 8), (33, 64, 1)]:
        L = _rand_layer(rng, d_out, d_in, r, 2, s=1.3)
        W0, A, B, s = L["W0"], L["A"], L["B"], L["s"]
        base = np.einsum("ij,ij->i", W0, W0)
        cross = 2.0 * s * np.einsum("ir,ir->i", B, W0 @ A.T)
        gram = s * s * np.einsum("ir,rq,iq->i", B, A @ A.T, B)
        C, _, _ = orc.norm(W0, A, B, L["m"], s)
        _close(C * C, base + cross + gram, 1e-12, "factored identity")


def pin_factored_norm(orc):
    rng = np.random.default_rng(8)
    for (d_out, d_in, r, s) in [(5, 7, 3, 1.3), (16, 40, 8, -0.6), (9, 4, 12, 2.0)]:
        L = _rand_layer(rng, d_out, d_in, r, 2, s=s)
        got = orc.norm_factored(L["W0"], L["A"], L["B"], L["m"], s)
        want = orc.norm(L["W0"], L["A"], L["B"], L["m"], s)
        for a, b, what in zip(got, want, ("C", "g", "gm1")):
            _close(a, b, 1e-12, f"factored {what}")
    for ex in _golden():
        W0, A, B, m = (np.array(ex[k], dtype=np.float64) for k in ("W0", "A", "B", "m"))
        C, g, gm1 = orc.norm_factored(W0, A, B, m, float(ex["s"]))
        _close(C, ex["expected"]["C"], 1e-14, "factored C (golden)")
        _close(gm1, ex["expected"]["gm1"], 1e-14, "factored gm1 (golden)")
    L = _rand_layer(rng, 6, 9, 3, 2)
    C, _, _ = orc.norm_factored(L["W0"], L["A"], np.zeros_like(L["B"]), L["m"], L["s"])
    _close(C, np.linalg.norm(L["W0"], axis=1), 1e-14, "factored C(B=0)")


def pin_zero_B(orc):
    rng = np.random.default_rng(11)
    L = _rand_layer(rng, 6, 9, 3, 2)
    B0 = np.zeros_like(L["B"])
    C, g, gm1 = orc.norm(L["W0"], L["A"], B0, L["m"], L["s"])
    ref = np.linalg.norm(L["W0"], axis=1)
    _close(C, ref, 1e-14, "C(B=0)")
    _close(g, L["m"] / ref, 1e-14, "g(B=0)")
    _close(gm1, L["m"] / ref - 1.0, 1e-13, "gm1(B=0)")


def pin_init(orc):
    rng = np.random.default_rng(12)
    L = _rand_layer(rng, 6, 9, 3, 4)
    B0 = np.zeros_like(L["B"])
    m0 = np.linalg.norm(L["W0"], axis=1)
    y = orc.forward(L["x"], L["W0"], L["A"], B0, m0, L["s"])
    _close(y, L["x"] @ L["W0"].T, 1e-13, "y at init")


def pin_scale(orc):
    rng = np.random.default_rng(13)
    L = _rand_layer(rng, 5, 8, 2, 3)
    a = 3.0
    args = (L["W0"], L["A"], L["B"], L["m"], L["s"])
    argsa = (a * L["W0"], L["A"], a * L["B"], L["m"], L["s"])
    _close(orc.forward(L["x"], *argsa), orc.forward(L["x"], *args), 1e-13, "y scale invariance")
    g1 = orc.backward(L["dy"], L["x"], *args)
    g2 = orc.backward(L["dy"], L["x"], *argsa)
    for k in ("dm", "dx", "dA"):
        _close(g2[k], g1[k], 1e-12, f"{k} scale invariance")
    _close(a * g2["dB"], g1["dB"], 1e-12, "dB scales by 1/a")


def pin_merge(orc):
    rng = np.random.default_rng(14)
    L = _rand_layer(rng, 7, 6, 2, 3)
    Wm = orc.merge(L["W0"], L["A"], L["B"], L["m"], L["s"])
    _close(np.linalg.norm(Wm, axis=1), L["m"], 1e-13, "merged row lengths")
    y = orc.forward(L["x"], L["W0"], L["A"], L["B"], L["m"], L["s"])
    _close(y, L["x"] @ Wm.T, 1e-13, "y = x W_merged^T")


def _fd(fun, X, h=1e-5):
    G = np.zeros_like(X)
    it = np.nditer(X, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = X[i]
        X[i] = old + h
        fp = fun()
        X[i] = old - h
        fm = fun()
        X[i] = old
        G[i] = (fp - fm) / (2 * h)
    return G


def pin_fd_x_m(orc):
    rng = np.random.default_rng(15)
    L = _rand_layer(rng, 3, 5, 2, 3)
    loss = lambda: float(np.sum(L["dy"] * orc.forward(L["x"], L["W0"], L["A"], L["B"], L["m"], L["s"])))
    gr = orc.backward(L["dy"], L["x"], L["W0"], L["A"], L["B"], L["m"], L["s"])
    _close(gr["dx"], _fd(loss, L["x"]), 1e-7, "dx vs FD")
    _close(gr["dm"], _fd(loss, L["m"]), 1e-7, "dm vs FD")


def pin_fd_detached(orc):
    rng = np.random.default_rng(16)
    L = _rand_layer(rng, 3, 5, 2, 3)
    C0, _, _ = orc.norm(L["W0"], L["A"], L["B"], L["m"], L["s"])
    loss = lambda: float(np.sum(L["dy"] * orc.forward(L["x"], L["W0"], L["A"], L["B"], L["m"], L["s"], C=C0)))
    gr = orc.backward(L["dy"], L["x"], L["W0"], L["A"], L["B"], L["m"], L["s"])
    _close(gr["dA"], _fd(loss, L["A"]), 1e-7, "dA (detached) vs FD")
    _close(gr["dB"], _fd(loss, L["B"]), 1e-7, "dB (detached) vs FD")


def pin_fd_full(orc):
    rng = np.random.default_rng(17)
    L = _rand_layer(rng, 3, 5, 2, 3)
    loss = lambda: float(np.sum(L["dy"] * orc.forward(L["x"], L["W0"], L["A"], L["B"], L["m"], L["s"])))
    gr = orc.backward(L["dy"], L["x"], L["W0"], L["A"], L["B"], L["m"], L["s"], full=True)
    _close(gr["dA"], _fd(loss, L["A"]), 1e-7, "dA (full) vs FD")
    _close(gr["dB"], _fd(loss, L["B"]), 1e-7, "dB (full) vs FD")


def pin_a2_term(orc):
    rng = np.random.default_rng(18)
    L = _rand_layer(rng, 4, 6, 3, 5)
    W0, A, B, m, s, x, dy = (L[k] for k in ("W0", "A", "B", "m", "s", "x", "dy"))
    gd = orc.backward(dy, x, W0, A, B, m, s)
    gf = orc.backward(dy, x, W0, A, B, m, s, full=True)
    V = W0 + s * (B @ A)
    C = np.linalg.norm(V, axis=1)
    GW = dy.T @ x
    dropped = -(m / C**3)[:, None] * np.einsum("ij,ij->i", GW, V)[:, None] * V
    _close(gf["dB"] - gd["dB"], s * dropped @ A.T, 1e-12, "dB full - detached = (A.2) term")
    _close(gf["dA"] - gd["dA"], s * B.T @ dropped, 1e-12, "dA full - detached = (A.2) term")


def pin_eq8(orc):
    rng = np.random.default_rng(19)
    L = _rand_layer(rng, 6, 7, 2, 4)
    W0, A, B, m, s, x, dy = (L[k] for k in ("W0", "A", "B", "m", "s", "x", "dy"))
    V = W0 + s * (B @ A)
    GW = dy.T @ x
    cos = np.array([np.dot(GW[n], V[n]) / (np.linalg.norm(GW[n]) * np.linalg.norm(V[n])) for n in range(6)])
    ref = np.linalg.norm(GW, axis=1) * cos
    _close(orc.backward(dy, x, W0, A, B, m, s)["dm"], ref, 1e-12, "eq. (8)")


def pin_near_unity(orc):
    rng = np.random.default_rng(20)
    L = _rand_layer(rng, 50, 30, 4, 2)
    C = np.linalg.norm(L["W0"] + L["s"] * L["B"] @ L["A"], axis=1)
    delta = rng.uniform(-1e-3, 1e-3, 50)
    m = C * (1.0 + delta)
    _, g, gm1 = orc.norm(L["W0"], L["A"], L["B"], m, L["s"])
    _close(gm1, delta, 1e-15, "g - 1 = delta")
    _close(g, 1.0 + delta, 1e-15, "g = 1 + delta")


def pin_vera_fd(orc):
    rng = np.random.default_rng(21)
    L = _rand_layer(rng, 4, 5, 3, 3)
    Bs = L["B"]
    b, d = rng.uniform(0.5, 1.5, 4), rng.uniform(-1.0, 1.0, 3)
    W0, A, m, s, x, dy = (L[k] for k in ("W0", "A", "m", "s", "x", "dy"))
    C0, _, _ = orc.norm(W0, A, orc.vera_direction(Bs, b, d), m, s)
    for full in (False, True):
        Cf = None if full else C0
        loss = lambda: float(np.sum(dy * orc.forward(x, W0, A, orc.vera_direction(Bs, b, d), m, s, C=Cf)))
        dBp = orc.backward(dy, x, W0, A, orc.vera_direction(Bs, b, d), m, s, full=full)["dB"]
        db, dd = orc.vera_gradients(dBp, Bs, b, d)
        _close(db, _fd(loss, b), 1e-7, f"db vs FD (full={full})")
        _close(dd, _fd(loss, d), 1e-7, f"dd vs FD (full={full})")


def pin_vera_unit(orc):
    rng = np.random.default_rng(22)
    Bs = rng.standard_normal((5, 3))
    _close(orc.vera_direction(Bs, np.ones(5), np.ones(3)), Bs, 0.0, "b = d = 1 gives B_shared")
    b, d = rng.uniform(0.5, 2.0, 5), rng.uniform(0.5, 2.0, 3)
    Bp = orc.vera_direction(Bs, b, d)
    _close(Bp[2] / Bs[2], b[2] * d, 1e-15, "row 2 scaled by b_2 d")
    _close(Bp[:, 1] / Bs[:, 1], b * d[1], 1e-15, "column 1 scaled by b d_1")


PINS = [pin_golden, pin_factored, pin_factored_norm, pin_zero_B, pin_init, pin_scale, pin_merge, pin_fd_x_m,
        pin_fd_detached, pin_fd_full, pin_a2_term, pin_eq8, pin_near_unity, pin_vera_fd, pin_vera_unit]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(oracle)


# --------------------------------------------------- input generator sanity checks

def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -1.0 - 2.0 ** -8, 0.0])])
    # torch converts float32 -> bf16 with one RNE rounding; feed it values exact in fp32.
    v32 = v.astype(np.float32).astype(np.float64)
    ours = round_to_bf16(v32)
    ref = torch.from_numpy(v32.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours, ref)


def test_workload_param_count():
    # DoRA notes appendix A.3: d = k = 4096, r = 16 gives r (d + k) + k = 135,168 trainable values.
    wl = workload("c2")
    assert wl.r * (wl.d_out + wl.d_in) + wl.d_out == 135168


def test_generator_is_deterministic_and_rounded():
    wl = workload("c2", d_out=64, d_in=96, r=16, T=8)
    a = make_inputs(wl)
    b = make_inputs(wl)
    for k in ("W0", "A", "B", "m", "x", "dy"):
        assert np.array_equal(a[k], b[k]), k
    for k in ("W0", "A", "B", "x", "dy"):
        bits = a[k].view(np.uint32)
        assert not np.any(bits & 0xFFFF), f"{k} not bf16-exact"


def test_near_unity_generator():
    wl = workload("c4a", d_out=48, d_in=64, r=16, T=4)
    inp = make_inputs(wl)
    assert inp["m"] is None and np.all(np.abs(inp["delta"]) <= 1e-3)
    C, _, _ = oracle.norm(inp["W0"], inp["A"], inp["B"], np.ones(48), inp["s"])
    m = near_unity_magnitude(C, inp["delta"])
    _, g, _ = oracle.norm(inp["W0"], inp["A"], inp["B"], m, inp["s"])
    assert np.all(np.abs(g - 1.0) <= 1e-3 + 1e-6)


# ------------------------------------------- planted mistakes must fail some pin

def _mutant(**overrides):
    ns = types.SimpleNamespace(adapted_direction=oracle.adapted_direction, norm=oracle.norm,
                               norm_factored=oracle.norm_factored,
                               forward=oracle.forward, backward=oracle.backward, merge=oracle.merge,
                               vera_direction=oracle.vera_direction, vera_gradients=oracle.vera_gradients)
    for k, v in overrides.items():
        setattr(ns, k, v)
    return ns


def _V(W0, A, B, s):
    return np.asarray(W0, float) + s * (np.asarray(B, float) @ np.asarray(A, float))


def _norm_using(Vfun, axis=1):
    def norm(W0, A, B, m, s):
        V = Vfun(W0, A, B, s)
        C = np.sqrt(np.sum(V * V, axis=axis))
        m = np.asarray(m, float)
        return C, m / C, (m - C) / C
    return norm


def _forward_using(Vfun):
    def forward(x, W0, A, B, m, s, C=None):
        V = Vfun(W0, A, B, s)
        if C is None:
            C = np.linalg.norm(V, axis=1)
        return (np.asarray(x, float) @ V.T) * (np.asarray(m, float) / C)[None, :]
    return forward


def _backward_variant(kind):
    def backward(dy, x, W0, A, B, m, s, full=False):
        dy = np.asarray(dy, float); x = np.asarray(x, float)
        A = np.asarray(A, float); B = np.asarray(B, float); m = np.asarray(m, float)
        V = _V(W0, A, B, s)
        C = np.linalg.norm(V, axis=1)
        g = m / C
        GW = dy.T @ x
        dm = np.sum(GW * V, axis=1) / (C * C if kind == "dm_over_C2" else C)
        dV = GW if kind == "no_g_in_dV" else g[:, None] * GW
        if full:
            sign = -1.0 if kind == "proj_sign" else 1.0
            dV = dV - sign * (np.sum(dV * V, axis=1) / (C * C))[:, None] * V
        dB = s * dV @ A.T
        dA = (B.T @ dV) if kind == "dA_no_s" else s * (B.T @ dV)
        dx = dy @ V if kind == "dx_no_g" else dy @ (g[:, None] * V)
        if kind == "dx_W0_only":
            dx = dy @ (g[:, None] * np.asarray(W0, float))
        return {"dm": dm, "dA": dA, "dB": dB, "dx": dx}
    return backward


def _gm1_flipped(W0, A, B, m, s):
    C, g, gm1 = oracle.norm(W0, A, B, m, s)
    return C, g, -gm1


def _forward_ignores_C(x, W0, A, B, m, s, C=None):
    return oracle.forward(x, W0, A, B, m, s)


def _factored_gram_s(W0, A, B, m, s):
    """The Gram term scaled by s instead of s^2."""
    W0, A, B, m = (np.asarray(v, float) for v in (W0, A, B, m))
    sq = np.sum(W0 * W0, axis=1) + 2 * s * np.sum(B * (W0 @ A.T), axis=1) + s * np.sum(B * (B @ (A @ A.T)), axis=1)
    C = np.sqrt(sq)
    return C, m / C, (m - C) / C


_V_no_s = lambda W0, A, B, s: np.asarray(W0, float) + np.asarray(B, float) @ np.asarray(A, float)
_V_neg = lambda W0, A, B, s: np.asarray(W0, float) - s * (np.asarray(B, float) @ np.asarray(A, float))
_V_s2 = lambda W0, A, B, s: np.asarray(W0, float) + s * s * (np.asarray(B, float) @ np.asarray(A, float))

MUTANTS = {
    "dropped_s": _mutant(adapted_direction=_V_no_s, norm=_norm_using(_V_no_s), forward=_forward_using(_V_no_s)),
    "wrong_sign": _mutant(norm=_norm_using(_V_neg), forward=_forward_using(_V_neg)),
    "s_squared": _mutant(norm=_norm_using(_V_s2), forward=_forward_using(_V_s2)),
    "column_norm": _mutant(norm=_norm_using(_V, axis=0)),
    "gm1_flipped": _mutant(norm=_gm1_flipped),
    "factored_gram_times_s": _mutant(norm_factored=_factored_gram_s),
    "forward_ignores_fixed_C": _mutant(forward=_forward_ignores_C),
    "dV_without_g": _mutant(backward=_backward_variant("no_g_in_dV")),
    "dm_over_C2": _mutant(backward=_backward_variant("dm_over_C2")),
    "projection_sign": _mutant(backward=_backward_variant("proj_sign")),
    "dA_without_s": _mutant(backward=_backward_variant("dA_no_s")),
    "dx_without_g": _mutant(backward=_backward_variant("dx_no_g")),
    "dx_from_W0_only": _mutant(backward=_backward_variant("dx_W0_only")),
    "vera_b_d_swapped": _mutant(vera_direction=lambda Bs, b, d: np.asarray(Bs, float) * np.outer(
        np.resize(np.asarray(d, float), len(b)), np.resize(np.asarray(b, float), len(d)))),
    "vera_dd_missing_b": _mutant(vera_gradients=lambda dBp, Bs, b, d: (
        (np.asarray(dBp) * Bs) @ np.asarray(d, float), np.sum(np.asarray(dBp) * Bs, axis=0))),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    failed = []
    for pin in PINS:
        try:
            pin(MUTANTS[name])
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake '{name}' passed every pin"
