"""Seeded synthetic inputs for the DoRA adapter layer.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It draws random tensors with the shapes and value
distributions of the layer workloads and rounds them once to the storage
precision. It holds none of the DoRA arithmetic (no norm of W0 + s*B*A, no
composition, no gradient).

Workloads (one PCG64 stream per workload, seed = 1000 + index):

  c1  tiny fp32        d_out=64    d_in=128  r=8    s=2.0  T=16
      W0, x ~ N(0, 1/sqrt(d_in)); m = |W0_i| * U(0.9, 1.1)
  c2  attention proj   d_out=4096  d_in=4096 r=16   s=2.0  T=2048
  c3  high-rank        d_out=8192  d_in=8192 r=384  s=0.5  T=4096
  c4a launch-bound     d_out=2048  d_in=6144 r=64   s=2.0  T=512
  c4b launch-bound     d_out=6144  d_in=2048 r=64   s=2.0  T=512
  c5  32B-VLM MLP up   d_out=27648 d_in=5120 r=384  s=0.5  T=8192

  bf16 workloads: W0 ~ N(0, 0.02), x ~ N(0, 1), B ~ N(0, 0.01),
  m = |W0_i| * U(0.95, 1.05); c4 draws a relative offset delta ~ U(-1e-3, 1e-3)
  instead, and the caller sets m = C * (1 + delta) from a norm it trusts
  (the near-unity regime the Scaling DoRA abstract names).
  Every workload: A ~ U(-1/sqrt(d_in), 1/sqrt(d_in)) (the "Kaiming uniform"
  LoRA-A initialisation of the DoRA reading notes, Algorithm 1 step 3, read
  with a = sqrt(5)); dy ~ N(0, 1). N(0, sigma) means standard deviation sigma.

Values are drawn in float64 and rounded once to bf16 (round to nearest even)
or to fp32; they are returned as float32 arrays holding those exact values.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = ["Workload", "WORKLOADS", "workload", "make_inputs", "round_to_bf16",
           "near_unity_magnitude", "bf16_bits"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    d_out: int
    d_in: int
    r: int
    s: float
    T: int
    dtype: str            # "bf16" or "fp32"
    w0_std: float | None  # None: 1/sqrt(d_in)
    x_std: float | None   # None: 1/sqrt(d_in)
    b_std: float
    m_lo: float | None    # m = |W0_i| * U(m_lo, m_hi); None: near-unity delta
    m_hi: float | None
    delta: float          # half-width of the near-unity offset (used when m_lo is None)
    seed: int

    def shapes(self) -> dict:
        return dict(W0=(self.d_out, self.d_in), A=(self.r, self.d_in), B=(self.d_out, self.r),
                    m=(self.d_out,), x=(self.T, self.d_in), dy=(self.T, self.d_out))


def _wl(name, d_out, d_in, r, s, T, dtype, seed, w0_std=0.02, x_std=1.0, b_std=0.01,
        m_lo=0.95, m_hi=1.05, delta=0.0):
    return Workload(name, d_out, d_in, r, s, T, dtype, w0_std, x_std, b_std, m_lo, m_hi, delta, seed)


WORKLOADS = {
    "c1": _wl("c1_tiny_fp32", 64, 128, 8, 2.0, 16, "fp32", 1001, w0_std=None, x_std=None,
              b_std=0.02, m_lo=0.9, m_hi=1.1),
    "c2": _wl("c2_attn_4096x4096_r16", 4096, 4096, 16, 2.0, 2048, "bf16", 1002),
    "c3": _wl("c3_8192x8192_r384", 8192, 8192, 384, 0.5, 4096, "bf16", 1003),
    "c4a": _wl("c4a_2048x6144_r64", 2048, 6144, 64, 2.0, 512, "bf16", 1004,
               m_lo=None, m_hi=None, delta=1e-3),
    "c4b": _wl("c4b_6144x2048_r64", 6144, 2048, 64, 2.0, 512, "bf16", 1005,
               m_lo=None, m_hi=None, delta=1e-3),
    "c5": _wl("c5_27648x5120_r384", 27648, 5120, 384, 0.5, 8192, "bf16", 1006),
}


def workload(key: str, **overrides) -> Workload:
    """A named workload, optionally with some fields replaced (e.g. smaller T)."""
    return dataclasses.replace(WORKLOADS[key], **overrides)


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values once to bf16 (8 significant bits, ties to even).

    Exact for normal values: frexp splits v = f * 2**e with 0.5 <= |f| < 1, so
    f * 256 carries the 8 kept bits in its integer part and np.rint rounds the
    rest to nearest even. Returned as float32, which holds every bf16 value.
    """
    v = np.asarray(v, dtype=np.float64)
    f, e = np.frexp(v)
    return np.ldexp(np.rint(np.ldexp(f, 8)), e - 8).astype(np.float32)


def bf16_bits(v32: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are exact bf16 values."""
    v32 = np.ascontiguousarray(v32, dtype=np.float32)
    bits = v32.view(np.uint32)
    if np.any(bits & 0xFFFF):
        raise ValueError("values are not exact bf16")
    return (bits >> 16).astype(np.uint16)


def _store(v64: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bf16(v64)
    if dtype == "fp32":
        return np.asarray(v64, dtype=np.float64).astype(np.float32)
    raise ValueError(dtype)


def make_inputs(wl: Workload, with_backward: bool = True, token_seed: int | None = None) -> dict:
    """Draw one workload's tensors. Order of draws: W0, A, B, m factor, x, dy.

    Returns float32 numpy arrays (exact storage-precision values) plus 's' and,
    for near-unity workloads, 'delta' with m = None. With token_seed, x and dy
    come from their own stream (data-parallel ranks share the weights but not
    the tokens).
    """
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    w0_std = wl.w0_std if wl.w0_std is not None else 1.0 / math.sqrt(wl.d_in)
    x_std = wl.x_std if wl.x_std is not None else 1.0 / math.sqrt(wl.d_in)
    bound = 1.0 / math.sqrt(wl.d_in)

    out = {"s": float(wl.s), "workload": wl}
    out["W0"] = _store(rng.standard_normal((wl.d_out, wl.d_in)) * w0_std, wl.dtype)
    out["A"] = _store(rng.uniform(-bound, bound, (wl.r, wl.d_in)), wl.dtype)
    out["B"] = _store(rng.standard_normal((wl.d_out, wl.r)) * wl.b_std, wl.dtype)
    if wl.m_lo is not None:
        factor = rng.uniform(wl.m_lo, wl.m_hi, wl.d_out)
        # Magnitude initialised from the frozen weight's row lengths, then jittered.
        w0_len = np.sqrt(np.sum(np.square(out["W0"], dtype=np.float64), axis=1))
        out["m"] = (w0_len * factor).astype(np.float32)
        out["delta"] = None
    else:
        out["delta"] = rng.uniform(-wl.delta, wl.delta, wl.d_out)
        out["m"] = None
    if token_seed is not None:
        rng = np.random.Generator(np.random.PCG64([wl.seed, token_seed]))
    out["x"] = _store(rng.standard_normal((wl.T, wl.d_in)) * x_std, wl.dtype)
    if with_backward:
        out["dy"] = _store(rng.standard_normal((wl.T, wl.d_out)), wl.dtype)
    return out


def near_unity_magnitude(C: np.ndarray, delta: np.ndarray) -> np.ndarray:
    """m = C * (1 + delta) in float32, for a norm C supplied by the caller."""
    return (np.asarray(C, dtype=np.float64) * (1.0 + np.asarray(delta, dtype=np.float64))).astype(np.float32)
