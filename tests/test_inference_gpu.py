"""Cached-norm inference on the GPU: the norm is computed once (A, B and m
fixed), then dora_forward runs on several token batches with nothing saved
for a backward (su and pre stay in the workspace / are not written), and
each y must match the oracle's forward for that batch. The merged weight of
dora_merge gives the same outputs as a plain product x W'^T.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import dora_testlib as tl
import dora_weight_decomposed_b200 as dw
import oracle
from dora_inputs import make_inputs, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dora_weight_decomposed_b200 import build
    build.build()
    yield
    assert dw.dora_device_status() == 0, "a kernel's bounded wait ran out"


@pytest.mark.parametrize("key,ov", [("c2", dict(d_out=512, d_in=768, T=0)),
                                    ("c3", dict(d_out=640, d_in=1024, r=136, T=0)),
                                    ("c4a", dict(d_out=384, d_in=1024, T=0))])
def test_cached_norm_forward_over_batches(key, ov):
    wl = workload(key, **ov)
    inp = tl.prepare(wl, with_backward=False)
    dev = tl.to_device(inp)
    C, g, gm1 = dw.dora_norm(dev["W0"], dev["A"], dev["B"], dev["m"], wl.s)
    norm_gpu = {"C": C, "g": g, "gm1": gm1}
    Cr, gr, gm1r = oracle.norm(inp["W0"], inp["A"], inp["B"], inp["m"], wl.s)
    ws = torch.empty(dw.dora_workspace_size(wl.d_out, wl.d_in, wl.r, torch.bfloat16, wl.s, 300,
                                            dw.DORA_OP_FORWARD), dtype=torch.uint8, device="cuda")
    for seed, T in ((11, 300), (12, 1), (13, 129)):
        x_np = make_inputs(workload(key, **dict(ov, T=T)), with_backward=False, token_seed=seed)["x"]
        x = torch.from_numpy(x_np).cuda().to(torch.bfloat16).contiguous()
        y, su, pre = dw.dora_forward(x, dev["W0"], dev["A"], dev["B"], gm1, wl.s, save_for_backward=False, ws=ws,
                                     y=tl.poisoned((T, wl.d_out), torch.bfloat16))
        assert su is None and pre is None
        ref = {"C": Cr, "g": gr, "gm1": gm1r, "y": oracle.forward(x_np, inp["W0"], inp["A"], inp["B"], inp["m"], wl.s)}
        batch = dict(inp, x=x_np)
        what = f"{key} T={T}"
        tl.check_tensor("y", y, ref["y"], "bf16", what=what)
        tl.check_rows("y", y, ref["y"], "bf16", what=what)
        tl.check_elementwise("y", y, ref["y"], tl.element_bounds(batch, ref, norm_gpu, "bf16")["y"], what=what)
        if wl.m_lo is None:  # near-unity layer: the adapted part y - x W0^T must survive too
            base = x_np.astype(np.float64) @ inp["W0"].astype(np.float64).T
            a, b = tl.host(y) - base, ref["y"] - base
            assert tl.rel_fro(a, b) <= tl.BF16_RTOL and tl.cosine(a, b) >= 0.999, (key, T)
            if T >= 100:
                tl.check_near_unity(y, batch, ref, what=what)


def test_forward_without_saves_matches_forward_with_saves():
    wl = workload("c3", d_out=384, d_in=512, r=64, T=200)
    inp = tl.prepare(wl, with_backward=False)
    dev = tl.to_device(inp)
    _, _, gm1 = dw.dora_norm(dev["W0"], dev["A"], dev["B"], dev["m"], wl.s)
    y1, su, pre = dw.dora_forward(dev["x"], dev["W0"], dev["A"], dev["B"], gm1, wl.s)
    y2, _, _ = dw.dora_forward(dev["x"], dev["W0"], dev["A"], dev["B"], gm1, wl.s, save_for_backward=False)
    assert torch.equal(y1, y2)
