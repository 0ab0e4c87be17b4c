"""GPU parity of the single-step recurrent update (ssm_selective_state_update)
against the fp64 oracle's step, and against the CUDA scan run one step at a
time.  Tolerances are those of the forward (helpers.py)."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_50_b200 import ssm_scan

from helpers import assert_close_io

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm_scan.load_library()


def make_case(seed, batch, dim, N, io, z=True, D=True, bias=True, softplus=True):
    r = np.random.default_rng(seed)
    tdt = torch.bfloat16 if io == "bf16" else torch.float32

    def io_t(x):   # io-dtype device tensor and the exact values it holds (fp64)
        t = torch.from_numpy(x.astype(np.float32)).to(tdt)
        return t.cuda(), t.double().numpy()

    c = {}
    c["u"], c["u64"] = io_t(r.standard_normal((batch, dim)))
    # without softplus the caller supplies the step size itself: keep it >= 0
    # (a negative step makes exp(ΔA) > 1)
    delta = r.standard_normal((batch, dim)) if softplus else np.abs(r.standard_normal((batch, dim))) * 0.1
    c["delta"], c["delta64"] = io_t(delta)
    c["B"], c["B64"] = io_t(r.standard_normal((batch, N)))
    c["C"], c["C64"] = io_t(r.standard_normal((batch, N)))
    if z:
        c["z"], c["z64"] = io_t(r.standard_normal((batch, dim)))
    else:
        c["z"], c["z64"] = None, None
    A = (-np.exp(r.standard_normal((dim, N)))).astype(np.float32)
    c["A"], c["A64"] = torch.from_numpy(A).cuda(), A.astype(np.float64)
    Dv = r.uniform(0.5, 1.5, dim).astype(np.float32) if D else None
    c["D"], c["D64"] = (torch.from_numpy(Dv).cuda(), Dv.astype(np.float64)) if D else (None, None)
    b0 = r.uniform(1e-3, 0.1, dim)
    bv = (np.log(np.expm1(b0)) if softplus else b0).astype(np.float32) if bias else None
    c["bias"], c["bias64"] = (torch.from_numpy(bv).cuda(), bv.astype(np.float64)) if bias else (None, None)
    st = r.standard_normal((batch, dim, N)).astype(np.float32)
    c["state"], c["state64"] = torch.from_numpy(st).cuda(), st.astype(np.float64)
    c["softplus"] = softplus
    return c


def run_and_check(c, io, state=None):
    state = c["state"] if state is None else state
    out = ssm_scan.selective_state_update(state, c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"],
                                          c["z"], c["bias"], c["softplus"])
    torch.cuda.synchronize()
    ref_out, ref_state = oracle.step(c["state64"], c["u64"], c["delta64"], c["A64"], c["B64"],
                                     c["C64"], c["D64"], c["z64"], c["bias64"], c["softplus"])
    assert_close_io(out.double().cpu().numpy(), ref_out, io, "out")
    # the state is fp32 in any io dtype
    assert_close_io(state.double().cpu().numpy(), ref_state, "f32", "state")


CASES = [
    # batch, dim, N, io, z, D, bias, softplus
    (1, 1, 1, "f32", True, True, True, True),
    (2, 37, 2, "f32", False, True, False, True),
    (3, 100, 4, "bf16", True, False, True, True),
    (4, 513, 8, "f32", True, True, True, False),
    (8, 1536, 16, "bf16", True, True, True, True),
    (2, 2049, 16, "f32", False, False, False, True),
    (5, 300, 32, "bf16", True, True, True, True),
    (64, 5120, 16, "bf16", True, True, True, True),
    (3, 256, 16, "f32", False, False, False, False),
    (300, 1024, 16, "bf16", True, True, True, True),
    (1, 128, 16, "bf16", True, False, True, True),
]


@pytest.mark.parametrize("case", CASES)
def test_step_matches_oracle(case):
    batch, dim, N, io, z, D, bias, sp = case
    c = make_case(11 + dim, batch, dim, N, io, z, D, bias, sp)
    run_and_check(c, io)


def test_repeated_steps_in_place():
    """Several steps in a row update the state in place consistently: each
    step's output and state match the oracle stepped from the previous
    oracle state."""
    c = make_case(21, 4, 512, 16, "bf16")
    st64 = c["state64"]
    for _ in range(3):
        out = ssm_scan.selective_state_update(c["state"], c["u"], c["delta"], c["A"], c["B"], c["C"],
                                              c["D"], c["z"], c["bias"], True)
        torch.cuda.synchronize()
        ref_out, st64 = oracle.step(st64, c["u64"], c["delta64"], c["A64"], c["B64"], c["C64"],
                                    c["D64"], c["z64"], c["bias64"], True)
        assert_close_io(out.double().cpu().numpy(), ref_out, "bf16", "out")
        assert_close_io(c["state"].double().cpu().numpy(), st64, "f32", "state")


def test_step_unaligned_state_uses_scalar_path():
    c = make_case(5, 3, 200, 16, "f32")
    buf = torch.empty(c["state"].numel() + 1, device="cuda", dtype=torch.float32)
    st = buf[1:].view(c["state"].shape)            # 4-byte but not 16-byte aligned
    st.copy_(c["state"])
    run_and_check(c, "f32", state=st)


def test_steps_reproduce_the_cuda_scan():
    """L steps from a zero state agree with the CUDA forward scan and its final
    state (both fp32 arithmetic)."""
    batch, dim, L, N = 2, 300, 24, 16
    r = np.random.default_rng(3)
    u = torch.from_numpy(r.standard_normal((batch, dim, L)).astype(np.float32)).cuda()
    delta = torch.from_numpy(r.standard_normal((batch, dim, L)).astype(np.float32)).cuda()
    z = torch.from_numpy(r.standard_normal((batch, dim, L)).astype(np.float32)).cuda()
    B = torch.from_numpy(r.standard_normal((batch, N, L)).astype(np.float32)).cuda()
    C = torch.from_numpy(r.standard_normal((batch, N, L)).astype(np.float32)).cuda()
    A = torch.from_numpy((-np.exp(r.standard_normal((dim, N)))).astype(np.float32)).cuda()
    D = torch.from_numpy(r.uniform(0.5, 1.5, dim).astype(np.float32)).cuda()
    bias = torch.from_numpy(np.log(np.expm1(r.uniform(1e-3, 0.1, dim))).astype(np.float32)).cuda()
    out, last, _ = ssm_scan.selective_scan_fwd(u, delta, A, B, C, D, z, bias, True, return_last_state=True)
    st = torch.zeros(batch, dim, N, device="cuda", dtype=torch.float32)
    for t in range(L):
        y = ssm_scan.selective_state_update(st, u[..., t].contiguous(), delta[..., t].contiguous(), A,
                                            B[..., t].contiguous(), C[..., t].contiguous(), D,
                                            z[..., t].contiguous(), bias, True)
        torch.cuda.synchronize()
        np.testing.assert_allclose(y.cpu().numpy(), out[..., t].cpu().numpy(), rtol=1e-4, atol=1e-4)
    np.testing.assert_allclose(st.cpu().numpy(), last.cpu().numpy(), rtol=1e-4, atol=1e-4)


def test_step_rejects_out_aliasing_state():
    c = make_case(7, 2, 16, 4, "f32")
    with pytest.raises(ssm_scan.SSMError):
        ssm_scan.state_update_raw(ssm_scan.make_shape(2, 16, 1, 4, ssm_scan.SSM_F32), c["state"],
                                  c["u"], c["delta"], c["A"], c["B"], c["C"], None, None, None,
                                  True, c["state"])
