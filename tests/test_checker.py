"""The GPU parity checker, pinned on the CPU.

The element-wise bounds of tests/dora_testlib.py are derived from the
rounding steps of the GPU's arithmetic. Here that arithmetic is replayed in
NumPy (every stored intermediate rounded to bf16 or fp32 exactly where the
kernels round it, accumulation in float64 then rounded to fp32), and the
replay must pass every check against the oracle: the bounds are not tighter
than the arithmetic allows. Then mistakes are planted in copies of the replayed
outputs -- a zeroed tile, a tile copied from its neighbour, an unwritten
(NaN) element, swapped rows, a scaled row, a flipped dm entry, a y composed
without g - 1 -- and each must fail: the bounds are tight enough to see them.
No GPU is involved.
"""
import numpy as np
import pytest

import dora_testlib as tl
from dora_inputs import round_to_bf16, workload


def _f32(v):
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)


def _replay(inp, ref):
    """The kernels' rounding sequence on the CPU (see element_bounds for the formulas)."""
    wl = inp["workload"]
    rnd = (lambda v: round_to_bf16(v).astype(np.float64)) if wl.dtype == "bf16" else _f32
    f = lambda k: np.asarray(inp[k], dtype=np.float64)
    x, W0, A, B, m, s, dy = f("x"), f("W0"), f("A"), f("B"), f("m"), inp["s"], f("dy")
    C = _f32(ref["C"])
    g = _f32(m / C)
    gm1 = _f32((m - C) / C)
    su = rnd(_f32(s * (x @ A.T)))
    pre32 = _f32(x @ W0.T + su @ B.T)
    y = rnd(_f32(pre32 + gm1[None, :] * pre32))
    pre = rnd(pre32)
    dz = rnd(_f32(g[None, :] * dy))
    du = rnd(_f32(s * (dz @ B)))
    return {"C": C, "g": g, "gm1": gm1, "y": y, "su": su, "pre": pre,
            "dm": _f32(_f32(np.sum(dy * pre, axis=0)) / C), "dB": rnd(_f32(dz.T @ su)),
            "dA": rnd(_f32(du.T @ x)), "dx": rnd(_f32(dz @ W0 + du @ A))}


CASES = {
    "bf16_ragged": ("c3", dict(d_out=96, d_in=160, r=24, T=40)),
    "bf16_wide_r": ("c3", dict(d_out=136, d_in=128, r=136, T=33)),
    "bf16_one_token": ("c2", dict(d_out=16, d_in=24, r=8, T=1)),
    "fp32_c1": ("c1", {}),
    "near_unity": ("c4a", dict(d_out=512, d_in=512, T=192)),
}


def _case(name):
    key, ov = CASES[name]
    wl = workload(key, **ov)
    inp = tl.prepare(wl)
    ref = tl.run_oracle(inp)
    return inp, ref, _replay(inp, ref)


@pytest.mark.parametrize("name", sorted(CASES))
def test_replayed_arithmetic_passes(name):
    inp, ref, out = _case(name)
    tl.check_all(out, ref, inp, what=name)
    tl.check_elementwise("su", out["su"], inp["s"] * (inp["x"].astype(np.float64) @ inp["A"].astype(np.float64).T),
                         tl.element_bounds(inp, ref, out, inp["workload"].dtype)["su"], name)


def test_near_unity_slope_of_replay_is_one():
    inp, ref, out = _case("near_unity")
    slope, bound = tl.check_near_unity(out["y"], inp, ref, "replay")
    assert bound < 0.5


def _fails(inp, ref, out):
    with pytest.raises(AssertionError):
        tl.check_all(out, ref, inp, what="planted")


@pytest.mark.parametrize("name", ["bf16_ragged", "fp32_c1"])
def test_zeroed_tile_fails(name):
    inp, ref, out = _case(name)
    out["y"] = out["y"].copy()
    out["y"][0:8, 16:32] = 0.0
    _fails(inp, ref, out)


def test_neighbour_tile_fails():
    inp, ref, out = _case("bf16_ragged")
    out["dx"] = out["dx"].copy()
    out["dx"][8:16, 0:16] = out["dx"][8:16, 16:32]
    _fails(inp, ref, out)


def test_unwritten_element_fails():
    inp, ref, out = _case("bf16_ragged")
    out["dx"] = out["dx"].copy()
    out["dx"][-1, -1] = np.nan
    _fails(inp, ref, out)


def test_swapped_rows_fail():
    inp, ref, out = _case("bf16_wide_r")
    out["dA"] = out["dA"].copy()
    out["dA"][[3, 4]] = out["dA"][[4, 3]]
    _fails(inp, ref, out)


def test_scaled_row_fails():
    inp, ref, out = _case("bf16_ragged")
    out["dB"] = out["dB"].copy()
    out["dB"][5] *= 1.05
    _fails(inp, ref, out)


def test_flipped_dm_fails():
    inp, ref, out = _case("bf16_ragged")
    out["dm"] = out["dm"].copy()
    i = int(np.argmax(np.abs(ref["dm"])))
    out["dm"][i] = -out["dm"][i]
    _fails(inp, ref, out)


def test_y_without_g_minus_one_fails_near_unity():
    """A y composed with a g rounded to bf16 (g - 1 lost at g ~ 1 +- 1e-3) passes the normwise
    check but not the near-unity slope."""
    inp, ref, out = _case("near_unity")
    pre32 = _f32(inp["x"].astype(np.float64) @ inp["W0"].astype(np.float64).T
                 + out["su"] @ inp["B"].astype(np.float64).T)
    g_bf16 = round_to_bf16(out["g"]).astype(np.float64)
    y_bad = round_to_bf16(pre32 * g_bf16[None, :]).astype(np.float64)
    tl.check_tensor("y", y_bad, ref["y"], "bf16")  # the normwise tolerance cannot see it
    with pytest.raises(AssertionError):
        tl.check_near_unity(y_bad, inp, ref, "planted")
