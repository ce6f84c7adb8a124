"""GPU parity on seeded random layer shapes: every dimension a multiple of 8
(the bf16 layout rule) but otherwise arbitrary, so tile tails, single partial
tiles, split-K choices and rank padding all get exercised together. Each
shape runs the layer step, the merge and the full gradient against the
oracle.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import dora_testlib as tl
import dora_weight_decomposed_b200 as dw
import oracle
from dora_inputs import workload

pytestmark = pytest.mark.gpu


def _shapes(n=10, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        d_out = 8 * int(rng.integers(1, 150))
        d_in = 8 * int(rng.integers(1, 150))
        r = 8 * int(rng.integers(1, 65))
        T = int(rng.integers(1, 700))
        out.append((d_out, d_in, r, T))
    return out


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dora_weight_decomposed_b200 import build
    build.build()
    yield
    assert dw.dora_device_status() == 0, "a kernel's bounded wait ran out"


@pytest.mark.parametrize("shape", _shapes(), ids=lambda s: "x".join(map(str, s)))
def test_random_shape_parity(shape):
    d_out, d_in, r, T = shape
    wl = workload("c3", d_out=d_out, d_in=d_in, r=r, T=T, s=0.5 if r > 64 else 2.0)
    inp = tl.prepare(wl)
    dev = tl.to_device(inp)
    out = tl.run_gpu(dev, wl.s)
    ref = tl.run_oracle(inp)
    tl.check_all(out, ref, inp, what=f"{shape}")
    W0, A, B, m, x, dy = (inp[k] for k in ("W0", "A", "B", "m", "x", "dy"))
    Wm = dw.dora_merge(dev["W0"], dev["A"], dev["B"], out["g"], wl.s)
    tl.check_tensor("W_merged", Wm, oracle.merge(W0, A, B, m, wl.s), "bf16", what=f"{shape}")
    full = dw.dora_backward_full(dev["dy"], dev["x"], dev["W0"], dev["A"], dev["B"], out["C"], out["g"], out["su"],
                                 out["pre"], wl.s)
    ref_full = oracle.backward(dy, x, W0, A, B, m, wl.s, full=True)
    tl.check_tensor("dA_full", full[1], ref_full["dA"], "bf16", what=f"{shape}")
    tl.check_tensor("dB_full", full[2], ref_full["dB"], "bf16", what=f"{shape}")
