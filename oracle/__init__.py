"""Plain CPU float64 oracle for the DoRA adapter layer -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the benchmark's CPU-baseline/reference leg
may import this package. The CUDA library never calls it and shares no code
with it: this file forms the dense adapted weight W0 + s*B*A and applies the
definitions directly, so that every shortcut the GPU path takes (the factored
norm, the fused near-unity compose, the u/du gradient route) is checked
against the definition it has to reproduce.

Sources (cited by page and equation):
  [DoRA notes]    "DoRA 阅读笔记" (zhongzhuzhou.org reading notes on DoRA,
                  arXiv 2402.09353): LoRA eq. (1); DoRA eq. (6); Algorithm 1
                  steps 7-14 and 16-17; gradients eq. (7) and eq. (8); the
                  detach trick of section 3.4; the full gradient eq. (A.1)
                  and the dropped term (A.2) of appendix A.
                  Section 3.5: DVoRA, the direction update taken from VeRA,
                  diag(b) B_shared diag(d) A_shared with the shared pair frozen.
  [Scaling DoRA]  "Scaling DoRA" (gptget.net/papers/2603.22276), English
                  abstract: the row-wise norm of W + sBA with W of shape
                  [d_out, d_in], and the g - 1 near-unity rescaling regime.

Readings where the pages are silent or disagree (each also listed in the
design notes):
  * One norm per output feature, i.e. per row of W0 [d_out x d_in]. The notes
    write W in R^{d x k} with column norms and m in R^{1 x k}; the abstract
    says row-wise for [d_out, d_in]. Both name the norm of one output unit's
    weight vector.
  * The LoRA scale s multiplies B*A inside the norm and the output (abstract:
    "W + sBA"); eq. (6) is the s = 1 case.
  * No epsilon is added to the norm; a zero norm gives inf/NaN.
  * The backward treats the norm as a constant (section 3.4, Algorithm 1 step 9)
    unless full=True, which follows eq. (A.1).
  * There is no bias and no dropout.

Every function computes in float64 from the given (already rounded) inputs.
Parity pins for every function live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np

__all__ = ["adapted_direction", "norm", "norm_factored", "forward", "backward", "merge", "vera_direction",
           "vera_gradients"]


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def adapted_direction(W0, A, B, s: float) -> np.ndarray:
    """V' = W0 + s * B @ A, dense [d_out x d_in].

    [DoRA notes] LoRA eq. (1) (W0 + BA with B [d x r], A [r x k]) and
    Algorithm 1 steps 7-8; the scale s as in [Scaling DoRA] ("W + sBA").
    """
    return _f64(W0) + float(s) * (_f64(B) @ _f64(A))


def _row_norms(V: np.ndarray) -> np.ndarray:
    return np.sqrt(np.sum(V * V, axis=1))


def norm(W0, A, B, m, s: float):
    """Per-output-row norm C = ||V'_i||, scale g = m / C and g - 1 = (m - C) / C.

    [DoRA notes] eq. (6) and Algorithm 1 step 9 (norm of each output unit's
    weight vector of W0 + BA); [Scaling DoRA] abstract (row-wise norm of W + sBA).
    Returns (C, g, gm1) as float64 [d_out] arrays.
    """
    C = _row_norms(adapted_direction(W0, A, B, s))
    m = _f64(m)
    return C, m / C, (m - C) / C


def norm_factored(W0, A, B, m, s: float):
    """The same (C, g, g - 1) as norm(), from the factored row norm without the dense B A.

    [Scaling DoRA] abstract: ||W + sBA||_row^2 splits into a base term ||W0_i||^2,
    a cross term 2 s B_i . (W0 A^T)_i and a Gram term s^2 B_i (A A^T) B_i^T, so
    only [d_out x r] and [r x r] intermediates are formed. Used as the CPU
    float64 timing baseline of the factored form (the benchmark times it beside
    the dense definition); the pins check it against norm().
    """
    W0, A, B, m = _f64(W0), _f64(A), _f64(B), _f64(m)
    s = float(s)
    base = np.einsum("ij,ij->i", W0, W0)
    cross = 2.0 * s * np.einsum("ir,ir->i", B, W0 @ A.T)
    gram = s * s * np.einsum("ir,ir->i", B @ (A @ A.T), B)
    C = np.sqrt(np.maximum(base + cross + gram, 0.0))
    return C, m / C, (m - C) / C


def forward(x, W0, A, B, m, s: float, C=None) -> np.ndarray:
    """y = x @ W'^T with W' = m * V' / C, i.e. y[t, i] = (m_i / C_i) * (x_t . V'_i).

    [DoRA notes] eq. (6) and Algorithm 1 steps 10-11. If C is given it is used
    instead of the current norm (the detached norm held fixed; used by the
    finite-difference pins of the detached gradient).
    """
    V = adapted_direction(W0, A, B, s)
    if C is None:
        C = _row_norms(V)
    g = _f64(m) / _f64(C)
    return (_f64(x) @ V.T) * g[None, :]


def backward(dy, x, W0, A, B, m, s: float, full: bool = False) -> dict:
    """Gradients of L = sum(dy * y) for y = forward(x, W0, A, B, m, s).

    [DoRA notes] Algorithm 1 steps 12-14 with the norm detached (section 3.4):
      grad wrt the composed weight W':  G_W = dy^T @ x            [d_out x d_in]
      eq. (8):  dm_n = G_W[n] . V'_n / ||V'_n||
      eq. (7):  dV = (m / C) * G_W   (row n scaled by m_n / C_n)
      eq. (1) through V' = W0 + s*B*A:  dB = s * dV @ A^T,  dA = s * B^T @ dV
      dx = dy @ W'   with W' = (m / C) * V'
    full=True uses eq. (A.1) instead of eq. (7): dV_n is projected onto the
    complement of V'_n, dV_n -= (dV_n . V'_n / C_n^2) V'_n. W0 is frozen and
    gets no gradient.
    Returns float64 arrays dm [d_out], dA [r x d_in], dB [d_out x r], dx [T x d_in].
    """
    dy = _f64(dy)
    x = _f64(x)
    V = adapted_direction(W0, A, B, s)
    C = _row_norms(V)
    g = _f64(m) / C
    G_W = dy.T @ x
    dm = np.sum(G_W * V, axis=1) / C
    dV = g[:, None] * G_W
    if full:
        dV = dV - (np.sum(dV * V, axis=1) / (C * C))[:, None] * V
    dB = float(s) * (dV @ _f64(A).T)
    dA = float(s) * (_f64(B).T @ dV)
    dx = dy @ (g[:, None] * V)
    return {"dm": dm, "dA": dA, "dB": dB, "dx": dx}


def merge(W0, A, B, m, s: float) -> np.ndarray:
    """Merged dense weight W' = m * (W0 + s*B*A) / C, [d_out x d_in].

    [DoRA notes] Algorithm 1 steps 16-17 (deployment merge).
    """
    V = adapted_direction(W0, A, B, s)
    return (_f64(m) / _row_norms(V))[:, None] * V


def vera_direction(B_shared, b, d) -> np.ndarray:
    """B' = diag(b) @ B_shared @ diag(d), [d_out x r].

    [DoRA notes] section 3.5 (DVoRA): the per-layer update is
    diag(b) B_shared diag(d) A_shared, so DVoRA is DoRA with B = B' and
    A = A_shared; norm, forward, backward and merge apply unchanged.
    """
    return _f64(b)[:, None] * _f64(B_shared) * _f64(d)[None, :]


def vera_gradients(dBp, B_shared, b, d):
    """Gradients of the two trained vectors from dB' = dL/dB' (chain rule through B').

    [DoRA notes] section 3.5: only b, d (and the magnitude m) are trained;
    A_shared and B_shared are frozen. With B'[n, c] = b[n] B_shared[n, c] d[c]:
      db[n] = sum_c dB'[n, c] B_shared[n, c] d[c]
      dd[c] = sum_n dB'[n, c] b[n] B_shared[n, c]
    """
    P = _f64(dBp) * _f64(B_shared)
    return P @ _f64(d), _f64(b) @ P
