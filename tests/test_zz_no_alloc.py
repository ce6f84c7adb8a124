"""dora_norm_noalloc (the norm call that uses the library's built-in scratch
array instead of a caller workspace) against dora_norm, through the C ABI.

Callers that cannot allocate device memory or pass a workspace use this call;
its results must equal the workspace call's. The file name makes pytest
collect it last, so a run that stops at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import dora_weight_decomposed_b200 as dw
from dora_inputs import make_inputs, workload

pytestmark = pytest.mark.gpu

NORM_RTOL = 1e-4  # the norm tolerance of the parity tests


def _lib():
    from dora_weight_decomposed_b200 import build
    build.build()
    lib = dw.load_library()
    P = ctypes.c_void_p
    lib.dora_norm_noalloc.argtypes = [ctypes.POINTER(dw.DoraDesc), P, P, P, P, P, P, P, P]
    lib.dora_norm_noalloc.restype = ctypes.c_int
    return lib


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return _lib()


CASES = {"c3_full": ("c3", {}), "ragged_r24": ("c2", dict(d_out=200, d_in=264, r=24)),
         "c1_fp32": ("c1", {})}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_workspace_call_twice(lib, name):
    key, ov = CASES[name]
    wl = workload(key, T=1, **ov)
    inp = make_inputs(wl, with_backward=False)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    W0, A, B = (torch.from_numpy(inp[k]).cuda().to(dt).contiguous() for k in ("W0", "A", "B"))
    m = torch.from_numpy(inp["m"]).cuda()
    ref = [t.double().cpu().numpy() for t in dw.dora_norm(W0, A, B, m, wl.s)]
    desc = dw.DoraDesc(wl.d_out, wl.d_in, wl.r, 0 if dt == torch.bfloat16 else 1, wl.s)
    stream = torch.cuda.current_stream().cuda_stream or None
    for call in range(2):
        outs = [torch.full((wl.d_out,), float("nan"), device="cuda") for _ in range(3)]
        st = lib.dora_norm_noalloc(ctypes.byref(desc), W0.data_ptr(), A.data_ptr(), B.data_ptr(), m.data_ptr(),
                                   outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(), stream)
        assert st == 0, dw.dora_last_error()
        torch.cuda.synchronize()
        C, g, gm1 = (t.double().cpu().numpy() for t in outs)
        assert np.max(np.abs(C - ref[0]) / ref[0]) <= NORM_RTOL, f"call {call}: C"
        assert np.max(np.abs(g - ref[1]) / np.abs(ref[1])) <= NORM_RTOL, f"call {call}: g"
        assert np.max(np.abs(gm1 - ref[2])) <= 1e-3 * np.max(np.abs(ref[2])), f"call {call}: gm1"
    assert dw.dora_device_status() == 0


def test_noalloc_rejects_layers_beyond_its_scratch(lib):
    # fp32 27648 x 5120, r = 384 needs about 82 MiB of norm scratch. NULL
    # tensors: the size check rejects the call before any pointer is used.
    desc = dw.DoraDesc(27648, 5120, 384, 1, 0.5)
    assert lib.dora_workspace_size(ctypes.byref(desc), 0, 0) > (16 << 20)
    st = lib.dora_norm_noalloc(ctypes.byref(desc), None, None, None, None, None, None, None, None)
    assert st == 2
    assert "16 MiB" in dw.dora_last_error()
