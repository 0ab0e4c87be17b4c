"""The allocation-free backward (ssm_selective_scan_bwd_noalloc).

It serves callers that cannot give the backward any device scratch: ones with
no device allocator at hand, or that must not call one (cudaMalloc/cudaFree
can synchronise the whole device; some runtimes forbid allocation after
start-up).  Its checkpoint scratch is a static array inside the library that
every call shares, so these tests call it twice in a row and compare each
result with the regular entry point's.  This file sorts last so that a run
stopping at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

import oracle
from selective_state_space_50_b200 import ssm_scan
from selective_state_space_50_b200.workloads import Workload, generate, to_torch

from helpers import assert_close_grad, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm_scan.load_library()


GRADS = ("du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias")


_OUT = {}


def _noalloc_into(dv, w):
    """Calls the entry point on gradient buffers kept from the previous call,
    so that the call itself is the only thing that could allocate."""
    g = _OUT["g"]
    shape = ssm_scan.make_shape(w.batch, w.dim, w.seqlen, w.dstate, dv["u"].dtype)
    ssm_scan.bwd_noalloc_raw(shape, dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"],
                             dv["z"], dv["delta_bias"], w.softplus, dv["dout"], g["du"],
                             g["ddelta"], g["dA"], g["dB"], g["dC"], g["dD"], g["dz"],
                             g["ddelta_bias"])


def _noalloc(dv, w, fill):
    shape = ssm_scan.make_shape(w.batch, w.dim, w.seqlen, w.dstate, dv["u"].dtype)
    f32 = dict(device="cuda", dtype=torch.float32)
    u = dv["u"]
    g = {"du": torch.full(u.shape, fill, **f32), "ddelta": torch.full(u.shape, fill, **f32),
         "dA": torch.full(dv["A"].shape, fill, **f32), "dB": torch.full(dv["B"].shape, fill, **f32),
         "dC": torch.full(dv["C"].shape, fill, **f32), "dD": torch.full(dv["D"].shape, fill, **f32),
         "dz": torch.full(u.shape, fill, **f32),
         "ddelta_bias": torch.full(dv["delta_bias"].shape, fill, **f32)}
    ssm_scan.bwd_noalloc_raw(shape, dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"],
                             dv["z"], dv["delta_bias"], w.softplus, dv["dout"], g["du"],
                             g["ddelta"], g["dA"], g["dB"], g["dC"], g["dD"], g["dz"],
                             g["ddelta_bias"])
    torch.cuda.synchronize()
    _OUT["g"] = g
    return g


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_noalloc_matches_regular_backward_on_two_calls(io):
    w = Workload("noalloc", 2, 300, 96, 16, io, seed=31, A_dist="neg_lognormal",
                 D_dist="u0.5_1.5")
    inp = generate(w, with_dout=True)
    dv = to_torch(inp, w, "cuda")
    ref = ssm_scan.selective_scan_bwd(dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"],
                                      dv["z"], dv["delta_bias"], w.softplus, dv["dout"])
    torch.cuda.synchronize()
    exact = oracle.bwd_workload(inp, w)
    # second call starts from the first call's scratch contents; outputs are
    # pre-filled with different junk each time
    for call, fill in enumerate((float("nan"), 1.0e30)):
        got = _noalloc(dv, w, fill)
        for k in GRADS:
            assert_close_grad(to_f64(got[k]), to_f64(ref[k]), f"call {call}: {k}")
            assert_close_grad(to_f64(got[k]), exact[k], f"call {call}: {k} vs the fp64 oracle")


def test_noalloc_allocates_no_device_memory():
    """After a first call (which may load the library's module on the device),
    further calls leave the device's free memory unchanged: the entry point
    allocates nothing."""
    w = Workload("noalloc", 2, 256, 160, 16, "bf16", seed=32, A_dist="neg_lognormal",
                 D_dist="u0.5_1.5")
    dv = to_torch(generate(w, with_dout=True), w, "cuda")
    _noalloc(dv, w, 0.0)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        _noalloc_into(dv, w)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)


def test_noalloc_rejects_shapes_beyond_its_buffer():
    lib = ssm_scan.load_library()
    # 8 x 1536 channels x 8192 steps needs 8*1536*1024*16*4 B = 768 MiB of checkpoints
    shape = ssm_scan.make_shape(8, 1536, 8192, 16, torch.bfloat16)
    assert ssm_scan.bwd_scratch_bytes(shape, False) > ssm_scan.NOALLOC_SCRATCH_BYTES
    st = lib.ssm_selective_scan_bwd_noalloc(ctypes.byref(shape), *([None] * 8), 1,
                                            *([None] * 10))
    assert st == ssm_scan.SSM_ERR_UNSUPPORTED
    msg = ssm_scan.last_error()
    assert "static buffer" in msg and str(ssm_scan.NOALLOC_SCRATCH_BYTES) in msg
