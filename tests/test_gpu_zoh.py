"""GPU parity of the zero-order-hold discretisation (B̄ = (exp(ΔA) - 1)/A · B,
the _ex entry points) against the fp64 oracle: forward, backward with and
without checkpoints, and the single step."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_50_b200 import ssm_scan
from selective_state_space_50_b200.workloads import generate

from helpers import assert_close_grad, assert_close_io, to_device, to_f64
from test_gpu_parity import small_workload
from test_gpu_step import make_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm_scan.load_library()


def _inputs(case, a_scale=1.0):
    w = small_workload(*case)
    inp = generate(w, with_dout=True)
    if a_scale != 1.0:   # |ΔA| small enough for the series branches, and exact zeros
        A = (inp["A"] * np.float32(a_scale)).astype(np.float32)
        A[:, 0] = 0.0
        inp["A"], inp["A_f64"] = A, A.astype(np.float64)
    return w, inp


def _oracle_fwd(inp, w):
    return oracle.fwd(inp["u_f64"], inp["delta_f64"], inp["A_f64"], inp["B_f64"], inp["C_f64"],
                      inp["D_f64"] if w.has_D else None, inp["z_f64"] if w.has_z else None,
                      inp["delta_bias_f64"] if w.has_bias else None, w.softplus, zoh=True)


CASES = [
    # batch, dim, L, N, io, z, D, bias, softplus, A_dist
    (2, 5, 70, 16, "f32", True, True, True, True, "neg_lognormal"),
    (1, 9, 129, 8, "f32", False, False, False, False, "neg_lognormal"),
    (2, 37, 200, 16, "bf16", True, True, True, True, "neg_n1"),
    (2, 17, 64, 32, "f32", True, True, True, True, "neg_lognormal"),
    (1, 70, 100, 2, "bf16", True, True, True, True, "neg_lognormal"),
    (2, 1200, 64, 16, "bf16", True, True, True, True, "neg_lognormal"),   # shape of the TMA kernels
    (2, 2400, 72, 16, "f32", True, True, True, True, "neg_lognormal"),    # TMA forward, ragged tile
    (1, 4800, 264, 16, "bf16", False, True, True, True, "neg_n1"),        # TMA forward, no gate
    (8, 1536, 64, 16, "bf16", True, True, True, True, "neg_lognormal"),   # TMA forward, 4 lanes per channel
]


@pytest.mark.parametrize("a_scale", [1.0, 1e-3])
@pytest.mark.parametrize("case", CASES)
def test_zoh_forward(case, a_scale):
    w, inp = _inputs(case, a_scale)
    dv = to_device(inp, w)
    out, last, _ = ssm_scan.selective_scan_fwd(dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"],
                                               dv["D"], dv["z"], dv["delta_bias"], w.softplus,
                                               return_last_state=True, zoh=True)
    torch.cuda.synchronize()
    ref, rlast = _oracle_fwd(inp, w)
    assert_close_io(to_f64(out), ref, w.io_dtype)
    assert_close_io(to_f64(last), rlast, "f32" if w.io_dtype == "f32" else "bf16", "last_state")


@pytest.mark.parametrize("use_ckpt", [True, False])
@pytest.mark.parametrize("a_scale", [1.0, 1e-3])
@pytest.mark.parametrize("case", CASES[:2] + CASES[3:-1])
def test_zoh_backward(case, a_scale, use_ckpt):
    w, inp = _inputs(case, a_scale)
    dv = to_device(inp, w)
    ck = None
    if use_ckpt:
        _, _, ck = ssm_scan.selective_scan_fwd(dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"],
                                               dv["D"], dv["z"], dv["delta_bias"], w.softplus,
                                               return_ckpt=True, zoh=True)
    g = ssm_scan.selective_scan_bwd(dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"],
                                    dv["z"], dv["delta_bias"], w.softplus, dv["dout"], ckpt=ck,
                                    zoh=True)
    torch.cuda.synchronize()
    # dstate 16 with at least one channel row per SM takes the TMA backward
    tma = w.dstate == 16 and w.batch * w.dim >= 148 and (w.seqlen * (2 if w.io_dtype == "bf16" else 4)) % 16 == 0
    assert ssm_scan.last_kernel_path() == ("bwd:tma" if tma else "bwd:general")
    ref = oracle.bwd(inp["u_f64"], inp["delta_f64"], inp["A_f64"], inp["B_f64"], inp["C_f64"],
                     inp["D_f64"] if w.has_D else None, inp["z_f64"] if w.has_z else None,
                     inp["delta_bias_f64"] if w.has_bias else None, w.softplus,
                     inp["dout_f64"], zoh=True)
    assert set(g) == set(ref)
    for k in ref:
        assert_close_grad(to_f64(g[k]), ref[k], k)


@pytest.mark.parametrize("N,io,dim", [(16, "bf16", 300), (4, "f32", 300), (32, "f32", 300),
                                      (16, "bf16", 384), (16, "f32", 256)])
def test_zoh_step(N, io, dim):
    c = make_case(41 + N, 3, dim, N, io)
    out = ssm_scan.selective_state_update(c["state"], c["u"], c["delta"], c["A"], c["B"], c["C"],
                                          c["D"], c["z"], c["bias"], True, zoh=True)
    torch.cuda.synchronize()
    ref_out, ref_state = oracle.step(c["state64"], c["u64"], c["delta64"], c["A64"], c["B64"],
                                     c["C64"], c["D64"], c["z64"], c["bias64"], True, zoh=True)
    assert_close_io(out.double().cpu().numpy(), ref_out, io, "out")
    assert_close_io(c["state"].double().cpu().numpy(), ref_state, "f32", "state")


@pytest.mark.parametrize("case", [
    (2, 5, 70, 16, "f32", True, True, True, False, "neg_lognormal"),      # general forward
    (2, 2400, 72, 16, "f32", True, True, True, False, "neg_lognormal"),   # TMA forward
])
def test_zoh_forward_at_series_switch(case):
    """Δ·A straddles ±0.1, where the zero-order-hold factor switches from its
    Taylor series to (Ā - 1)/(ΔA) (booiljung.github.io, "3.2 선택적 스캔
    (Selective Scan) 알고리즘" §2.1: B̄ = (ΔA)⁻¹(exp(ΔA) - I)ΔB): A = -1 and
    Δ in [0.05, 0.2] (softplus off, no bias), fp32 bound 1e-4 (1 + |y|)."""
    w = small_workload(*case)
    inp = generate(w, with_dout=True)
    rng = np.random.default_rng(7)
    A = np.full(inp["A"].shape, -1.0, dtype=np.float32)
    dl = rng.uniform(0.05, 0.2, size=inp["delta"].shape).astype(np.float32)
    bias = np.zeros(inp["delta_bias"].shape, dtype=np.float32)
    for k, v in (("A", A), ("delta", dl), ("delta_bias", bias)):
        inp[k], inp[k + "_f64"] = v, v.astype(np.float64)
    x = dl.astype(np.float64) * -1.0
    assert (x > -0.1).any() and (x < -0.1).any()
    dv = to_device(inp, w)
    out, last, _ = ssm_scan.selective_scan_fwd(dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"],
                                               dv["D"], dv["z"], dv["delta_bias"], False,
                                               return_last_state=True, zoh=True)
    torch.cuda.synchronize()
    ref, rlast = oracle.fwd(inp["u_f64"], inp["delta_f64"], inp["A_f64"], inp["B_f64"],
                            inp["C_f64"], inp["D_f64"], inp["z_f64"], inp["delta_bias_f64"],
                            False, zoh=True)
    assert_close_io(to_f64(out), ref, "f32")
    assert_close_io(to_f64(last), rlast, "f32", "last_state")
