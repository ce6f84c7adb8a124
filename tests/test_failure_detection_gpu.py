"""Failure detection without a GPU fault: a kernel's bounded wait on an
mbarrier that nothing completes runs out after a short limit, the kernel
returns, the host reads the timeout from dora_device_status (bit 0,
DORA_ETIMEOUT), the word is cleared by the read, and the context keeps
computing correct results afterwards. Host-side faults (NULL and misaligned
pointers, short workspaces, bad descriptors) are covered in test_abi.py.
"""
import pytest

torch = pytest.importorskip("torch")

import dora_testlib as tl
import dora_weight_decomposed_b200 as dw
from dora_inputs import workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dora_weight_decomposed_b200 import build
    build.build()


def test_bounded_wait_times_out_and_context_survives():
    assert dw.dora_device_status() == 0
    assert dw.dora_selftest_timeout(20000) == 1          # the wait ran out after ~20 ms
    assert dw.dora_device_status() == 1                  # reported once ...
    assert dw.dora_device_status() == 0                  # ... and cleared by the read
    wl = workload("c2", d_out=256, d_in=384, T=64)
    inp = tl.prepare(wl)
    out = tl.run_gpu(tl.to_device(inp), wl.s)
    tl.check_all(out, tl.run_oracle(inp), inp, what="after a timeout")
    assert dw.dora_device_status() == 0

