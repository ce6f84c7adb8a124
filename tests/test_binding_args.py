"""The Python binding checks every tensor's shape, dtype and device before it
calls the library (the C ABI cannot see them, and a wrong shape would send a
kernel past a buffer). On CPU: valid arguments get as far as the device check
(CUDA tensors required), invalid ones are refused with a message naming the
tensor. No kernel is launched."""
import pytest

torch = pytest.importorskip("torch")

import dora_weight_decomposed_b200 as dw

CUDA_ONLY = "tensors must be on a CUDA device"
bf, f32 = torch.bfloat16, torch.float32
d_out, d_in, r, T = 64, 96, 16, 24


def _layer():
    return dict(W0=torch.zeros(d_out, d_in, dtype=bf), A=torch.zeros(r, d_in, dtype=bf),
                B=torch.zeros(d_out, r, dtype=bf), m=torch.ones(d_out, dtype=f32), x=torch.zeros(T, d_in, dtype=bf),
                dy=torch.zeros(T, d_out, dtype=bf), g=torch.ones(d_out, dtype=f32), gm1=torch.zeros(d_out, dtype=f32),
                C=torch.ones(d_out, dtype=f32), su=torch.zeros(T, r, dtype=bf), pre=torch.zeros(T, d_out, dtype=bf))


def _expect_device_error(fn, *a, **k):
    with pytest.raises(ValueError, match=CUDA_ONLY):
        fn(*a, **k)


def test_valid_arguments_reach_the_device_check():
    L = _layer()
    _expect_device_error(dw.dora_norm, L["W0"], L["A"], L["B"], L["m"], 2.0)
    _expect_device_error(dw.dora_forward, L["x"], L["W0"], L["A"], L["B"], L["gm1"], 2.0)
    _expect_device_error(dw.dora_forward, L["x"], L["W0"], L["A"], L["B"], L["gm1"], 2.0, save_for_backward=False)
    _expect_device_error(dw.dora_backward, L["dy"], L["x"], L["W0"], L["A"], L["B"], L["C"], L["g"], L["su"],
                         L["pre"], 2.0)
    _expect_device_error(dw.dora_backward_full, L["dy"], L["x"], L["W0"], L["A"], L["B"], L["C"], L["g"],
                         L["su"], L["pre"], 2.0, need_dx=False)
    _expect_device_error(dw.dora_merge, L["W0"], L["A"], L["B"], L["g"], 2.0)
    _expect_device_error(dw.dora_vera_compose, L["B"], L["g"], torch.ones(r, dtype=f32))
    _expect_device_error(dw.dora_vera_grad, L["B"], L["g"], torch.ones(r, dtype=f32), L["B"])


@pytest.mark.parametrize("case", ["short_y", "wrong_dtype_x", "fp64_gm1", "short_dA", "bad_W0", "short_out",
                                  "f32_norm_out_bf16", "missing_su"])
def test_invalid_arguments_are_refused(case):
    L = _layer()
    if case == "short_y":
        with pytest.raises(ValueError, match="y has shape"):
            dw.dora_forward(L["x"], L["W0"], L["A"], L["B"], L["gm1"], 2.0, y=torch.zeros(T - 1, d_out, dtype=bf))
    elif case == "wrong_dtype_x":
        with pytest.raises(TypeError, match="x is"):
            dw.dora_forward(L["x"].float(), L["W0"], L["A"], L["B"], L["gm1"], 2.0)
    elif case == "fp64_gm1":
        with pytest.raises(TypeError, match="gm1 is"):
            dw.dora_forward(L["x"], L["W0"], L["A"], L["B"], L["gm1"].double(), 2.0)
    elif case == "short_dA":
        with pytest.raises(ValueError, match="dA has shape"):
            dw.dora_backward(L["dy"], L["x"], L["W0"], L["A"], L["B"], L["C"], L["g"], L["su"], L["pre"], 2.0,
                             dA=torch.zeros(r, d_in - 8, dtype=bf))
    elif case == "bad_W0":
        with pytest.raises(ValueError, match="W0 has shape"):
            dw.dora_backward(L["dy"], L["x"], L["W0"][:, :-8].contiguous(), L["A"], L["B"], L["C"], L["g"],
                             L["su"], L["pre"], 2.0)
    elif case == "short_out":
        with pytest.raises(ValueError, match="out has shape"):
            dw.dora_merge(L["W0"], L["A"], L["B"], L["g"], 2.0, out=torch.zeros(d_out - 8, d_in, dtype=bf))
    elif case == "f32_norm_out_bf16":
        with pytest.raises(TypeError, match="norm_out is"):
            dw.dora_norm(L["W0"], L["A"], L["B"], L["m"], 2.0, norm_out=torch.zeros(d_out, dtype=bf))
    elif case == "missing_su":
        with pytest.raises(ValueError, match="required"):
            dw.dora_backward(L["dy"], L["x"], L["W0"], L["A"], L["B"], L["C"], L["g"], None, L["pre"], 2.0)
