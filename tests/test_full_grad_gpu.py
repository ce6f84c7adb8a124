"""GPU parity of dora_backward_full (the gradient through the norm, appendix
A eq. A.1) against the oracle's full=True backward.

With random dy the term the detach drops is about cos(dV_n, V'_n) ~ 1/sqrt(d_in)
of the gradient, well under the bf16 tolerance, so a wrong correction could
pass unnoticed. The cases therefore also use a dy correlated with the layer's
own output (dy = a * pre / std(pre) + noise), which makes the dropped term a
large part of dA and dB; the full and the detached results must then differ
as the oracle says. dm and dx do not pass through the norm: they must equal
the detached call's bit for bit.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import dora_testlib as tl
import dora_weight_decomposed_b200 as dw
import oracle
from dora_inputs import round_to_bf16, workload
from test_parity_gpu import SMALL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dora_weight_decomposed_b200 import build
    build.build()
    yield
    assert dw.dora_device_status() == 0, "a kernel's bounded wait ran out"


def _correlated_dy(inp, a=1.5, seed=5):
    """dy = a pre / std(pre) + N(0, 1), pre = x (W0 + s B A)^T, rounded like the other inputs."""
    V = oracle.adapted_direction(inp["W0"], inp["A"], inp["B"], inp["s"])
    pre = inp["x"].astype(np.float64) @ V.T
    dy = a * pre / pre.std() + np.random.default_rng(seed).standard_normal(pre.shape)
    return dy.astype(np.float32) if inp["workload"].dtype == "fp32" else round_to_bf16(dy).astype(np.float32)


def _run(wl, correlated):
    inp = tl.prepare(wl)
    if correlated:
        inp["dy"] = _correlated_dy(inp)
    dev = tl.to_device(inp)
    norm, g, gm1 = dw.dora_norm(dev["W0"], dev["A"], dev["B"], dev["m"], wl.s)
    y, su, pre = dw.dora_forward(dev["x"], dev["W0"], dev["A"], dev["B"], gm1, wl.s)
    det = dw.dora_backward(dev["dy"], dev["x"], dev["W0"], dev["A"], dev["B"], norm, g, su, pre, wl.s)
    # NaN-filled outputs: an element the full-gradient kernels leave unwritten stays NaN.
    dt, T, r = dev["W0"].dtype, dev["x"].shape[0], wl.r
    full = dw.dora_backward_full(dev["dy"], dev["x"], dev["W0"], dev["A"], dev["B"], norm, g, su, pre, wl.s,
                                 dm=tl.poisoned((wl.d_out,), torch.float32), dA=tl.poisoned((r, wl.d_in), dt),
                                 dB=tl.poisoned((wl.d_out, r), dt), dx=tl.poisoned((T, wl.d_in), dt))
    W0, A, B, m, x = (inp[k] for k in ("W0", "A", "B", "m", "x"))
    ref_full = oracle.backward(inp["dy"], x, W0, A, B, m, wl.s, full=True)
    ref_det = oracle.backward(inp["dy"], x, W0, A, B, m, wl.s)
    return det, full, ref_det, ref_full


def _check_full(wl, correlated):
    det, full, ref_det, ref_full = _run(wl, correlated)
    assert torch.equal(full[0], det[0]), "dm must not change"
    assert torch.equal(full[3], det[3]), "dx must not change"
    for i, k in ((1, "dA"), (2, "dB")):
        tl.check_tensor(k, full[i], ref_full[k], wl.dtype, what=f"{wl.name} full")
        if not correlated:  # with dy correlated to pre, rows of the full gradient can nearly cancel
            tl.check_rows(k, full[i], ref_full[k], wl.dtype, what=f"{wl.name} full")
        if correlated:
            # The dropped term is large here: full - detached must follow the oracle.
            got = tl.host(full[i]) - tl.host(det[i])
            want = ref_full[k] - ref_det[k]
            assert np.linalg.norm(want) > 0.2 * np.linalg.norm(ref_det[k]), "dy not correlated enough"
            assert tl.rel_fro(got, want) <= 5e-2 and tl.cosine(got, want) >= 0.998, \
                (k, tl.rel_fro(got, want), tl.cosine(got, want))


@pytest.mark.parametrize("name", sorted(SMALL))
def test_full_gradient_small(name):
    key, ov = SMALL[name]
    _check_full(workload(key, **ov), correlated=True)


@pytest.mark.parametrize("key", ["c2", "c3"])
def test_full_gradient_large(key):
    wl = workload(key, T=512)
    _check_full(wl, correlated=False)


def test_full_gradient_c3_correlated():
    _check_full(workload("c3", d_out=1024, d_in=2048, T=384), correlated=True)


def test_full_gradient_empty_batch():
    wl = workload("c2", d_out=64, d_in=128, T=0)
    inp = tl.prepare(wl)
    dev = tl.to_device(inp)
    norm, g, gm1 = dw.dora_norm(dev["W0"], dev["A"], dev["B"], dev["m"], wl.s)
    y, su, pre = dw.dora_forward(dev["x"], dev["W0"], dev["A"], dev["B"], gm1, wl.s)
    dm, dA, dB, dx = dw.dora_backward_full(dev["dy"], dev["x"], dev["W0"], dev["A"], dev["B"], norm, g, su, pre,
                                           wl.s)
    assert torch.count_nonzero(dm) == 0 and torch.count_nonzero(dA) == 0 and torch.count_nonzero(dB) == 0
