"""GPU parity of dora_merge (the deployment merge W' = diag(g) (W0 + s B A))
against the oracle's merge, element by element.

Bound per element: the bf16 output is rounded once from an fp32 value whose
own error is dominated by g (fp32, within the norm tolerance), so
|gpu - ref| <= 2^-8 |ref| + 1e-4 max|ref|; fp32 outputs get 2e-4 |ref| +
1e-6 max|ref|. The merge is separable by rows, so the largest workload is
checked on a seeded sample of rows that the oracle computes on its own.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import dora_testlib as tl
import dora_weight_decomposed_b200 as dw
import oracle
from dora_inputs import workload
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


def _check(name, got, ref, dtype):
    a = tl.host(got)
    assert a.shape == ref.shape and np.all(np.isfinite(a)), name
    rtol, atol = (2.0 ** -8, 1e-4) if dtype == "bf16" else (2e-4, 1e-6)
    bound = rtol * np.abs(ref) + atol * float(np.max(np.abs(ref)))
    bad = np.abs(a - ref) > bound
    assert not bad.any(), f"{name}: {int(bad.sum())} elements out of bound, first at {np.argwhere(bad)[0]}"


def _merge_case(wl, rows=None):
    inp = tl.prepare(wl, with_backward=False)
    dev = tl.to_device(inp)
    _, g, _ = dw.dora_norm(dev["W0"], dev["A"], dev["B"], dev["m"], wl.s)
    Wm = dw.dora_merge(dev["W0"], dev["A"], dev["B"], g, wl.s, out=tl.poisoned(dev["W0"].shape, dev["W0"].dtype))
    W0, A, B, m = inp["W0"], inp["A"], inp["B"], inp["m"]
    if rows is None:
        ref = oracle.merge(W0, A, B, m, wl.s)
        got = Wm
    else:
        ref = oracle.merge(W0[rows], A, B[rows], np.asarray(m)[rows], wl.s)
        got = Wm[torch.from_numpy(rows).to(Wm.device)]
    _check(wl.name, got, ref, wl.dtype)
    return dev, g, Wm


@pytest.mark.parametrize("name", sorted(SMALL))
def test_merge_small(name):
    key, ov = SMALL[name]
    _merge_case(workload(key, **ov))


@pytest.mark.parametrize("key", ["c2", "c3", "c4a"])
def test_merge_full(key):
    _merge_case(workload(key))


def test_merge_largest_sampled_rows():
    wl = workload("c5")
    rows = np.sort(np.random.default_rng(7).choice(wl.d_out, 512, replace=False))
    rows[0], rows[-1] = 0, wl.d_out - 1
    _merge_case(wl, rows=np.unique(rows))


def test_merge_in_place_matches_out_of_place():
    wl = workload("c3", d_out=520, d_in=776, r=136)
    dev, g, Wm = _merge_case(wl)
    W = dev["W0"].clone()
    out = dw.dora_merge(W, dev["A"], dev["B"], g, wl.s, out=W)
    torch.cuda.synchronize()
    assert out.data_ptr() == W.data_ptr()
    assert torch.equal(W, Wm)


def test_merged_weight_reproduces_forward():
    """x W'^T equals the DoRA forward y = (g - 1) pre + pre up to bf16 rounding."""
    wl = workload("c2", d_out=384, d_in=512, T=96)
    inp = tl.prepare(wl, with_backward=False)
    dev = tl.to_device(inp)
    _, g, gm1 = dw.dora_norm(dev["W0"], dev["A"], dev["B"], dev["m"], wl.s)
    y, _, _ = dw.dora_forward(dev["x"], dev["W0"], dev["A"], dev["B"], gm1, wl.s)
    Wm = dw.dora_merge(dev["W0"], dev["A"], dev["B"], g, wl.s)
    y_merged = tl.host(dev["x"]) @ tl.host(Wm).T
    tl.check_tensor("x W'^T", y, y_merged, "bf16")
