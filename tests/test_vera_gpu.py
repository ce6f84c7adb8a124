"""GPU parity of the DVoRA calls (DoRA notes section 3.5): B' is formed by
dora_vera_compose, the DoRA calls run on it unchanged, and dora_vera_grad
turns dB' into the gradients of the trained vectors b and d; every output is
compared with the oracle's vera_direction / backward / vera_gradients.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import dora_testlib as tl
import dora_weight_decomposed_b200 as dw
import oracle
from dora_inputs import make_inputs, round_to_bf16, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dora_weight_decomposed_b200 import build
    build.build()
    yield
    assert dw.dora_device_status() == 0, "a kernel's bounded wait ran out"


def _vectors(d_out, r, seed=3):
    rng = np.random.default_rng(seed)
    return rng.uniform(0.5, 1.5, d_out).astype(np.float32), rng.uniform(-1.0, 1.0, r).astype(np.float32)


CASES = [("c2", dict(d_out=264, d_in=200, r=24, T=77)), ("c3", dict(d_out=320, d_in=392, r=136, T=150)),
         ("c1", dict(d_out=72, d_in=100, r=12, T=33))]


@pytest.mark.parametrize("key,ov", CASES, ids=[c[0] for c in CASES])
def test_dvora_layer_step(key, ov):
    wl = workload(key, **ov)
    inp = make_inputs(wl)
    b, d = _vectors(wl.d_out, wl.r)
    Bs = inp["B"] * 10.0  # the frozen shared matrix, larger than a trained LoRA B
    Bs = Bs.astype(np.float32) if wl.dtype == "fp32" else round_to_bf16(Bs).astype(np.float32)
    dt = torch.float32 if wl.dtype == "fp32" else torch.bfloat16
    dev = lambda a, t=dt: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(t).contiguous()
    W0, A, x, dy, Bs_d = dev(inp["W0"]), dev(inp["A"]), dev(inp["x"]), dev(inp["dy"]), dev(Bs)
    m = dev(inp["m"], torch.float32)
    b_d, d_d = dev(b, torch.float32), dev(d, torch.float32)
    Bp = dw.dora_vera_compose(Bs_d, b_d, d_d, out=tl.poisoned((wl.d_out, wl.r), dt))
    out = tl.run_gpu({"W0": W0, "A": A, "B": Bp, "m": m, "x": x, "dy": dy}, wl.s)
    dBp = out["dB"]
    db, dd = dw.dora_vera_grad(Bs_d, b_d, d_d, dBp, db=tl.poisoned((wl.d_out,), torch.float32),
                               dd=tl.poisoned((wl.r,), torch.float32))

    Bp_ref = oracle.vera_direction(Bs, b, d)
    # B' is rounded once from an fp32 product: within one rounding of the exact value.
    rel = np.abs(tl.host(Bp) - Bp_ref) / np.maximum(np.abs(Bp_ref), 1e-30)
    assert np.max(rel) <= (2.0 ** -8 if wl.dtype == "bf16" else 1e-6)
    # The rest against the oracle on the device's B' (the rounded values the layer really used).
    inp_used = dict(inp, B=tl.host(Bp))
    ref = tl.run_oracle(inp_used)
    tl.check_all(out, ref, inp_used, what="dvora")
    rdb, rdd = oracle.vera_gradients(ref["dB"], Bs, b, d)
    tl.check_tensor("db", db, rdb, wl.dtype, what="dvora")
    tl.check_tensor("dd", dd, rdd, wl.dtype, what="dvora")


@pytest.mark.parametrize("dtype,r", [("bf16", 136), ("fp32", 136), ("fp32", 324), ("bf16", 512), ("bf16", 8)])
def test_vera_grad_reductions(dtype, r):
    """db, dd from a given dB' (fp32 sums of exact input values): tight tolerance. fp32 rows wider
    than a block (r > 256) take the reduction's per-column branch."""
    rng = np.random.default_rng(9)
    d_out = 1000
    Bs = rng.standard_normal((d_out, r))
    dB = rng.standard_normal((d_out, r))
    if dtype == "bf16":
        Bs, dB = round_to_bf16(Bs), round_to_bf16(dB)
    b, d = _vectors(d_out, r, seed=4)
    t = torch.bfloat16 if dtype == "bf16" else torch.float32
    dev = lambda a, tt=t: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(tt).contiguous()
    db, dd = dw.dora_vera_grad(dev(Bs), dev(b, torch.float32), dev(d, torch.float32), dev(dB))
    rdb, rdd = oracle.vera_gradients(dB, Bs, b, d)
    for got, want in ((db, rdb), (dd, rdd)):
        err = np.max(np.abs(tl.host(got) - want)) / np.max(np.abs(want))
        assert err <= 1e-5, err
