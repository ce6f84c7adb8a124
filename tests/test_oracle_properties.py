"""Property checks of the oracle over many small random layers (hypothesis):
the same facts the pins fix on a few fixed layers, here across shapes, scales
and signs of s, so that a mistake that only shows for some shape (a
transposed operand that happens to be square, a sign that cancels at s > 0)
fails too.

  factored  C_i^2 = |W0_i|^2 + 2 s B_i (A W0_i^T) + s^2 B_i (A A^T) B_i^T
  merge     forward(x) = x W_merged^T
  detached  finite differences with the norm held fixed give dA and dB
  full      full minus detached dV is the dropped projection term (A.2)
  vera      b = d = 1 leaves DoRA unchanged; db, dd follow from dB' by the chain rule
"""
import numpy as np
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st

import oracle

SETTINGS = settings(max_examples=25, deadline=None)


@st.composite
def layers(draw):
    d_out = draw(st.integers(1, 6))
    d_in = draw(st.integers(1, 7))
    r = draw(st.integers(1, 3))
    T = draw(st.integers(1, 4))
    s = draw(st.sampled_from([-1.5, -0.5, 0.25, 1.0, 2.0]))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    W0 = rng.standard_normal((d_out, d_in)) + 0.5  # keep rows away from zero norm
    return dict(W0=W0, A=rng.standard_normal((r, d_in)) * 0.5, B=rng.standard_normal((d_out, r)) * 0.5,
                m=rng.uniform(0.5, 2.0, d_out), x=rng.standard_normal((T, d_in)),
                dy=rng.standard_normal((T, d_out)), s=s)


@given(layers())
@SETTINGS
def test_factored_norm_identity(L):
    W0, A, B, s = L["W0"], L["A"], L["B"], L["s"]
    C, _, _ = oracle.norm(W0, A, B, L["m"], s)
    base = np.sum(W0 * W0, axis=1)
    cross = np.sum(B * (W0 @ A.T), axis=1)
    gram = np.sum((B @ (A @ A.T)) * B, axis=1)
    np.testing.assert_allclose(C * C, base + 2 * s * cross + s * s * gram, rtol=1e-10, atol=1e-10)


@given(layers())
@SETTINGS
def test_forward_is_the_merged_product(L):
    y = oracle.forward(L["x"], L["W0"], L["A"], L["B"], L["m"], L["s"])
    Wm = oracle.merge(L["W0"], L["A"], L["B"], L["m"], L["s"])
    np.testing.assert_allclose(y, L["x"] @ Wm.T, rtol=1e-10, atol=1e-10)


def _fd_entry(f, X, idx, h=1e-6):
    old = X[idx]
    X[idx] = old + h
    fp = f()
    X[idx] = old - h
    fm = f()
    X[idx] = old
    return (fp - fm) / (2 * h)


@given(layers(), st.integers(0, 10**6))
@SETTINGS
def test_detached_gradient_matches_fd_with_fixed_norm(L, pick):
    W0, A, B, m, s, x, dy = (L[k] for k in ("W0", "A", "B", "m", "s", "x", "dy"))
    C0, _, _ = oracle.norm(W0, A, B, m, s)
    loss = lambda: float(np.sum(dy * oracle.forward(x, W0, A, B, m, s, C=C0)))
    g = oracle.backward(dy, x, W0, A, B, m, s)
    ia = np.unravel_index(pick % A.size, A.shape)
    ib = np.unravel_index(pick % B.size, B.shape)
    np.testing.assert_allclose(g["dA"][ia], _fd_entry(loss, A, ia), rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(g["dB"][ib], _fd_entry(loss, B, ib), rtol=1e-5, atol=1e-6)


@given(layers())
@SETTINGS
def test_full_minus_detached_is_the_dropped_term(L):
    W0, A, B, m, s, x, dy = (L[k] for k in ("W0", "A", "B", "m", "s", "x", "dy"))
    gd = oracle.backward(dy, x, W0, A, B, m, s)
    gf = oracle.backward(dy, x, W0, A, B, m, s, full=True)
    V = W0 + s * (B @ A)
    C = np.linalg.norm(V, axis=1)
    kappa = (m / C) * gd["dm"] / C  # g_n dm_n / C_n
    np.testing.assert_allclose(gf["dB"] - gd["dB"], -s * (kappa[:, None] * V) @ A.T, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(gf["dA"] - gd["dA"], -s * B.T @ (kappa[:, None] * V), rtol=1e-9, atol=1e-9)


@given(layers())
@SETTINGS
def test_vera_reduces_to_dora_and_chain_rule(L):
    W0, A, B, m, s, x, dy = (L[k] for k in ("W0", "A", "B", "m", "s", "x", "dy"))
    d_out, r = B.shape
    Bp = oracle.vera_direction(B, np.ones(d_out), np.ones(r))
    np.testing.assert_array_equal(Bp, B)
    rng = np.random.default_rng(d_out * 7 + r)
    b, d = rng.uniform(0.5, 1.5, d_out), rng.uniform(-1.0, 1.0, r)
    dBp = oracle.backward(dy, x, W0, A, oracle.vera_direction(B, b, d), m, s)["dB"]
    db, dd = oracle.vera_gradients(dBp, B, b, d)
    np.testing.assert_allclose(db, np.einsum("nc,nc,c->n", dBp, B, d), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dd, np.einsum("nc,nc,n->c", dBp, B, b), rtol=1e-12, atol=1e-12)
