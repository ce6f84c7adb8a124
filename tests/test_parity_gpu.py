"""GPU parity: the library's CUDA path against the CPU oracle, element by
element on the same seeded inputs.

Small cases span several tiles and ragged tails in every dimension; the full
workloads run at their stated sizes in the same launch configuration the
benchmark uses. Tolerances are in tests/dora_testlib.py.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import dora_testlib as tl
import dora_weight_decomposed_b200 as dw
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


SMALL = {
    "c1_fp32_full": ("c1", {}),
    "fp32_ragged": ("c1", dict(d_out=72, d_in=100, r=5, T=33)),
    "ragged_r24": ("c2", dict(d_out=200, d_in=264, r=24, T=77)),
    "ragged_r136": ("c3", dict(d_out=320, d_in=392, r=136, T=300)),
    "r384_tiles": ("c3", dict(d_out=256, d_in=640, r=384, T=257)),
    "r512": ("c3", dict(d_out=136, d_in=128, r=512, T=64)),
    "r8_one_token": ("c2", dict(d_out=8, d_in=8, r=8, T=1)),
    "r16_wide": ("c2", dict(d_out=640, d_in=384, r=16, T=200)),
    "r64_near_unity": ("c4a", dict(d_out=384, d_in=1024, T=130)),
    # few dB/dA tiles over a long K = T: two cluster split-K launches instead of the grouped one
    "long_T_few_tiles": ("c4a", dict(d_out=256, d_in=512, T=16384)),
    # 74 + 2 grouped dB/dA tiles of 256 x 128: more tiles than SM pairs, so pairs run two tiles
    # through the grouped kernel's two TMEM accumulators
    "grouped_two_waves": ("c4a", dict(d_out=18944, d_in=512, T=64)),
}


def test_gram_beside_norm_parity():
    """28 row tiles x 2 K splits leave 36 SMs beside the norm GEMM: the Gram takes 4 CTAs per
    tile and runs while the norm GEMM streams W0; the forward GEMM splits K over clusters of 2
    pairs and dx over 4."""
    wl = workload("c3", d_out=7168, d_in=2048, T=64)
    inp = tl.prepare(wl)
    out = tl.run_gpu(tl.to_device(inp), wl.s)
    tl.check_all(out, tl.run_oracle(inp), inp, what="gram beside norm")


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_parity(name):
    key, ov = SMALL[name]
    wl = workload(key, **ov)
    inp = tl.prepare(wl)
    dev = tl.to_device(inp)
    out = tl.run_gpu(dev, wl.s)
    ref = tl.run_oracle(inp)
    tl.check_all(out, ref, inp, what=name)
    # Intermediate saved for the backward: su = s x A^T, element by element.
    su_ref = wl.s * (inp["x"].astype(np.float64) @ inp["A"].astype(np.float64).T)
    tl.check_tensor("su", out["su"], su_ref, wl.dtype, what=name)
    tl.check_elementwise("su", out["su"], su_ref, tl.element_bounds(inp, ref, out, wl.dtype)["su"], what=name)
    if wl.m_lo is None:
        tl.check_near_unity(out["y"], inp, ref, what=name)


FULL = ["c2", "c3", "c4a", "c4b", "c5"]


@pytest.mark.parametrize("key", FULL)
def test_full_workload_parity(key):
    wl = workload(key)
    inp = tl.prepare(wl)
    dev = tl.to_device(inp)
    out = tl.run_gpu(dev, wl.s)
    del dev
    ref = tl.run_oracle(inp)
    tl.check_all(out, ref, inp, what=wl.name)
    if wl.m_lo is None:  # c4a, c4b: g = 1 +- 1e-3, the adapted part of y must survive the rounding
        tl.check_near_unity(out["y"], inp, ref, what=wl.name)


def test_near_unity_gm1_resolution():
    """g - 1 ~ 1e-3: taking it from a rounded g would lose it; (m - C) / C keeps it."""
    wl = workload("c4b", T=16)
    inp = tl.prepare(wl, with_backward=False)
    dev = tl.to_device(inp)
    _, _, gm1 = dw.dora_norm(dev["W0"], dev["A"], dev["B"], dev["m"], wl.s)
    ref = tl.run_oracle(inp, with_backward=False)["gm1"]
    a = tl.host(gm1)
    assert np.max(np.abs(ref)) < 2e-3
    assert np.max(np.abs(a - ref)) <= 1e-3 * np.max(np.abs(ref))
    assert tl.cosine(a, ref) >= 0.9999


def test_init_invariant_gives_base_projection():
    """B = 0 and m = |W0_i| reproduce the frozen layer: g = 1 and y = x W0^T."""
    wl = workload("c2", d_out=256, d_in=512, T=64)
    inp = make_inputs(wl)
    W0 = inp["W0"].astype(np.float64)
    inp["B"] = np.zeros_like(inp["B"])
    inp["m"] = np.sqrt(np.sum(W0 * W0, axis=1)).astype(np.float32)
    dev = tl.to_device(inp)
    out = tl.run_gpu(dev, wl.s)
    assert np.max(np.abs(tl.host(out["gm1"]))) <= 1e-5
    assert np.max(np.abs(tl.host(out["g"]) - 1.0)) <= 1e-5
    tl.check_tensor("y", out["y"], inp["x"].astype(np.float64) @ W0.T, "bf16", what="init")


def test_empty_batch():
    wl = workload("c2", d_out=64, d_in=128, T=0)
    inp = make_inputs(wl)
    dev = tl.to_device(inp)
    out = tl.run_gpu(dev, wl.s)
    assert out["y"].shape == (0, 64)
    assert torch.count_nonzero(out["dm"]) == 0
    assert torch.count_nonzero(out["dA"]) == 0 and torch.count_nonzero(out["dB"]) == 0


def test_bitwise_deterministic():
    wl = workload("c3", d_out=384, d_in=768, r=64, T=320)
    inp = tl.prepare(wl)
    dev = tl.to_device(inp)
    a = tl.run_gpu(dev, wl.s)
    b = tl.run_gpu(dev, wl.s)
    for k in ("C", "g", "gm1", "y", "su", "pre", "dm", "dA", "dB", "dx"):
        assert torch.equal(a[k], b[k]), k


def test_side_stream_and_no_dx():
    wl = workload("c2", d_out=256, d_in=256, T=96)
    inp = tl.prepare(wl)
    dev = tl.to_device(inp)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        norm, g, gm1 = dw.dora_norm(dev["W0"], dev["A"], dev["B"], dev["m"], wl.s, stream=s)
        y, su, pre = dw.dora_forward(dev["x"], dev["W0"], dev["A"], dev["B"], gm1, wl.s, stream=s)
        dm, dA, dB, dx = dw.dora_backward(dev["dy"], dev["x"], dev["W0"], dev["A"], dev["B"], norm, g, su, pre,
                                          wl.s, need_dx=False, stream=s)
    s.synchronize()
    assert dx is None
    ref = tl.run_oracle(inp)
    tl.check_tensor("y", y, ref["y"], "bf16")
    tl.check_tensor("dA", dA, ref["dA"], "bf16")
    tl.check_tensor("dm", dm, ref["dm"], "bf16")


def test_zero_norm_row_propagates():
    """A row with W0_i = 0 and B_i = 0 has C_i = 0 (no epsilon, read 5 of the design notes): g_i and
    g_i - 1 are +inf for m_i > 0 and the row's outputs are NaN (inf * 0), as in the oracle; the other
    rows are unaffected."""
    wl = workload("c2", d_out=128, d_in=256, T=40)
    inp = make_inputs(wl)
    inp["W0"][5] = 0.0
    inp["B"][5] = 0.0
    dev = tl.to_device(inp)
    out = tl.run_gpu(dev, wl.s)
    C, g, gm1, y = (tl.host(out[k]) for k in ("C", "g", "gm1", "y"))
    assert C[5] == 0.0 and np.isposinf(g[5]) and np.isposinf(gm1[5])
    assert np.all(np.isnan(y[:, 5]))
    ref = tl.run_oracle(inp)
    keep = np.arange(wl.d_out) != 5
    assert np.max(np.abs(C[keep] - ref["C"][keep]) / ref["C"][keep]) <= tl.NORM_RTOL
    tl.check_tensor("y (other rows)", out["y"][:, torch.from_numpy(keep).cuda()], ref["y"][:, keep], "bf16")


@pytest.mark.parametrize("key,ov", [("c4a", {}), ("c2", dict(d_out=1024, d_in=4096, T=1024)),
                                    ("c4b", {})])
def test_backward_fork_matches_serial(key, ov):
    """At these sizes dx leaves SM pairs idle and runs on the library's second stream beside the
    grouped dB/dA launch. Its results must be the serial backward's bits (the kernel profiler keeps
    the backward serial), eagerly and replayed from a CUDA graph holding the two branches."""
    wl = workload(key, **ov)
    inp = tl.prepare(wl)
    dev = tl.to_device(inp)
    a = tl.run_gpu(dev, wl.s)
    dw.dora_profile_start(64)
    try:
        b = tl.run_gpu(dev, wl.s)
    finally:
        dw.dora_profile_stop()
    for k in ("dm", "dA", "dB", "dx"):
        assert torch.equal(a[k], b[k]), k
    W0 = dev["W0"]
    d_out, d_in = W0.shape
    r, T = dev["A"].shape[0], dev["x"].shape[0]
    ws = torch.empty(max(dw.dora_workspace_size(d_out, d_in, r, W0.dtype, wl.s, T, dw.DORA_OP_BACKWARD), 256),
                     dtype=torch.uint8, device=W0.device)
    outs = dict(dm=tl.poisoned((d_out,), torch.float32), dA=tl.poisoned((r, d_in), W0.dtype),
                dB=tl.poisoned((d_out, r), W0.dtype), dx=tl.poisoned((T, d_in), W0.dtype))
    torch.cuda.synchronize()
    gph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gph):
        dw.dora_backward(dev["dy"], dev["x"], W0, dev["A"], dev["B"], a["C"], a["g"], a["su"], a["pre"], wl.s,
                         ws=ws, **outs)
    gph.replay()
    torch.cuda.synchronize()
    for k in ("dm", "dA", "dB", "dx"):
        assert torch.equal(outs[k], a[k]), f"{k} (graph)"
    del gph
