"""The launch planner (make_plan) on the CPU: which kernels, cluster sizes and overlaps a
call gets for each workload, checked without a GPU.

tests/planner_probe.cpp is compiled together with the planner's translation unit by g++,
with the kernels' entry points stubbed out and B200 cluster-occupancy figures; it prints one
call's plan as JSON. The decisions pinned here are the ones the GPU launch lists show (the
kernel instantiations and grids in profiles/launches_*_layer_step.md), and the invariants are
the SM budgets the overlapping launches rely on.
"""
import json
import math
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
OP_NORM, OP_FORWARD, OP_BACKWARD = 0, 1, 2
SMS, PAIRS = 148, 74


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None or not os.path.exists(os.path.join(CUDA, "include", "cuda_runtime.h")):
        pytest.skip("g++ or the CUDA runtime headers are missing")
    exe = str(tmp_path_factory.mktemp("planner") / "planner_probe")
    csrc = os.path.join(ROOT, "dora_weight_decomposed_b200", "csrc")
    cmd = [gxx, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"), "-I", csrc, "-I",
           os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "planner_probe.cpp"), "-x", "c++",
           os.path.join(csrc, "dora_api.cu"), "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    env = dict(os.environ, LD_LIBRARY_PATH=os.path.join(CUDA, "lib64") + ":" + os.environ.get("LD_LIBRARY_PATH", ""))

    def plan(d_out, d_in, r, T, op):
        out = subprocess.run([exe, str(d_out), str(d_in), str(r), str(T), str(op)], check=True,
                             capture_output=True, text=True, env=env).stdout
        p = json.loads(out)
        assert p["sms"] == SMS
        return p
    return plan


C2, C3, C4A, C4B, C5 = (4096, 4096, 16, 2048), (8192, 8192, 384, 4096), (2048, 6144, 64, 512), \
    (6144, 2048, 64, 512), (27648, 5120, 384, 8192)


def test_large_layers_take_no_overlap(probe):
    """c3 and c5: the base GEMMs fill every pair for several waves, so nothing runs beside them."""
    for shape in (C3, C5):
        f = probe(*shape, OP_FORWARD)
        assert f["fwd_cs"] == 0 and f["fwd_defer"] == 0 and f["fwd_pairs"] == PAIRS
        b = probe(*shape, OP_BACKWARD)
        assert b["dx_cs"] == 0 and b["bwd_fork"] == 0 and b["dx_defer"] == 0
        assert b["dBA_grouped"] == 1
    b = probe(*C3, OP_BACKWARD)
    assert (b["du_bn"], b["du_cs"], b["dB_bn"]) == (256, 2, 384)


def test_c4a_plan(probe):
    f = probe(*C4A, OP_FORWARD)
    assert (f["u_bn"], f["u_cs"], f["fwd_cs"], f["fwd_defer"]) == (64, 8, 3, 1)
    b = probe(*C4A, OP_BACKWARD)
    # 48 dx tiles fill one wave, one per pair: the cluster kernel with one pair per cluster; the
    # 26 pairs left take dB/dA (32 tiles, two per pair at most) and dx starts beside du
    assert (b["dx_cs"], b["bwd_fork"], b["dx_pairs"], b["dBA_pairs"], b["dx_defer"]) == (1, 1, 48, 26, 1)
    assert (b["du_bn"], b["du_cs"]) == (128, 4)


def test_c4b_plan(probe):
    f = probe(*C4B, OP_FORWARD)
    assert (f["u_cs"], f["fwd_cs"], f["fwd_defer"]) == (8, 1, 1)
    b = probe(*C4B, OP_BACKWARD)
    assert b["bwd_fork"] == 1 and b["dx_defer"] == 1 and b["dx_cs"] >= 2


def test_c2_plan(probe):
    f = probe(*C2, OP_FORWARD)
    # 128 forward tiles in two waves run on 64 pairs, so u (8 tiles, one pair each) fits beside
    assert (f["fwd_cs"], f["fwd_pairs"], f["u_cs"], f["fwd_defer"]) == (0, 64, 1, 1)
    b = probe(*C2, OP_BACKWARD)
    # dx on 64 pairs, dB/dA on the other 10; du and dx together would not fit
    assert (b["bwd_fork"], b["dx_pairs"], b["dBA_pairs"], b["dx_defer"]) == (1, 64, 10, 0)


SWEEP = [(d_out, d_in, r, T) for (d_out, d_in) in ((2048, 6144), (6144, 2048), (4096, 4096), (8192, 8192),
                                                   (1024, 4096), (18944, 512))
         for r in (16, 64, 384) for T in (64, 256, 512, 1024, 2048, 4096)]


@pytest.mark.parametrize("shape", SWEEP[::3] + SWEEP[1::7])
def test_overlap_budgets(probe, shape):
    """Whatever the shape, the launches that run at once fit on the SMs."""
    d_out, d_in, r, T = shape
    f = probe(d_out, d_in, r, T, OP_FORWARD)
    assert 1 <= f["fwd_pairs"] <= PAIRS
    if f["fwd_defer"] and f["fwd_cs"] == 0:
        tiles_u = math.ceil(T / 256) * math.ceil(r / f["u_bn"])
        assert 2 * f["fwd_pairs"] + 2 * f["u_cs"] * tiles_u <= SMS
    b = probe(d_out, d_in, r, T, OP_BACKWARD)
    if b["bwd_fork"]:
        assert b["dBA_grouped"] == 1
        assert b["dx_pairs"] + b["dBA_pairs"] <= PAIRS and b["dBA_pairs"] >= 1
    else:
        assert b["dx_defer"] == 0
    if b["dx_defer"]:
        tiles_du = math.ceil(T / 256) * math.ceil(r / b["du_bn"])
        assert 2 * b["du_cs"] * tiles_du + 2 * b["dx_pairs"] <= SMS


def test_backward_workspace_grows_with_tokens(probe):
    """The backward keeps a second copy of du whether or not it forks, so a workspace sized for T
    tokens serves every smaller batch."""
    for d_out, d_in, r in ((2048, 6144, 64), (4096, 4096, 16), (8192, 8192, 384)):
        sizes = [probe(d_out, d_in, r, T, OP_BACKWARD)["total"] for T in (1, 64, 256, 512, 1024, 2048, 4096)]
        assert sizes == sorted(sizes)
