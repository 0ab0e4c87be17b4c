"""GPU parity: the CUDA library (called through its C ABI) against the fp64
oracle on the same seeded inputs.  Tolerances are documented in helpers.py."""
import math

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_50_b200 import ssm_scan
from selective_state_space_50_b200.workloads import WORKLOADS, Workload, generate

from helpers import (assert_close_grad, assert_close_io, subset_channels, to_device, to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm_scan.load_library()


def run_fwd(dv, w, **kw):
    out, last, ck = ssm_scan.selective_scan_fwd(dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"],
                                                dv["D"], dv["z"], dv["delta_bias"], w.softplus,
                                                return_last_state=True, **kw)
    torch.cuda.synchronize()
    return out, last, ck


def check_fwd(w: Workload, channels=None, path=None):
    inp = generate(w)
    dv = to_device(inp, w)
    out, last, _ = run_fwd(dv, w)
    if path is not None:   # the kernel the library chose for this shape
        assert ssm_scan.last_kernel_path() == path
    if channels is not None:
        sub = subset_channels(inp, channels)
        ref, rlast = oracle.fwd_workload(sub, w)
        got = to_f64(out)[:, channels]
        glast = to_f64(last)[:, channels]
    else:
        ref, rlast = oracle.fwd_workload(inp, w)
        got, glast = to_f64(out), to_f64(last)
    e = assert_close_io(got, ref, w.io_dtype)
    # the final state is fp32 in any io dtype
    assert_close_io(glast, rlast, "f32" if w.io_dtype == "f32" else "bf16", "last_state")
    return e


def test_fwd_tiny_f32():
    check_fwd(WORKLOADS["tiny_f32"])


@pytest.mark.parametrize("name", ["mamba130m_layer", "mamba2p8b_layer"])
def test_fwd_layer_shapes_full(name):
    check_fwd(WORKLOADS[name], path="fwd:tma")


def test_fwd_long_context_sampled_channels():
    """Through the public forward, which gives the library its workspace: at
    1 x 2048 channels over 131072 steps it takes the two-level scan."""
    w = WORKLOADS["long_context"]
    check_fwd(w, channels=slice(0, w.dim, 97), path="fwd:chunked")


SMALL = [
    # batch, dim, L, N, io, z, D, bias, softplus, A_dist
    (1, 1, 1, 16, "f32", True, True, True, True, "neg_lognormal"),
    (2, 5, 7, 16, "f32", True, True, True, True, "neg_lognormal"),
    (1, 37, 33, 16, "bf16", True, True, True, True, "neg_lognormal"),
    (3, 19, 100, 8, "f32", False, True, True, True, "neg_lognormal"),
    (2, 9, 1023, 32, "f32", True, False, False, False, "neg_lognormal"),
    (1, 130, 64, 4, "bf16", True, True, True, True, "neg_n1"),
    (2, 7, 129, 2, "f32", True, True, True, True, "neg_lognormal"),
    (2, 7, 129, 1, "bf16", False, False, True, True, "neg_lognormal"),
    (1, 2048, 300, 16, "bf16", True, True, True, True, "neg_lognormal"),   # few (b,d): per-state lanes
    (1, 1000, 77, 32, "f32", True, True, True, True, "neg_lognormal"),
    (1, 1000, 77, 8, "f32", True, True, True, True, "neg_lognormal"),
    (1, 1000, 77, 4, "f32", True, True, True, True, "neg_lognormal"),
]


def small_workload(batch, dim, L, N, io, z, D, bias, sp, A_dist, seed=77):
    # without softplus the caller supplies the step size itself: draw it >= 0
    # (a negative step makes Ā > 1 and the state grows without bound)
    return Workload("small", batch, L, dim, N, io, seed=seed, has_z=z, has_D=D, has_bias=bias,
                    softplus=sp, A_dist=A_dist, D_dist="u0.5_1.5",
                    delta_abs=not sp, delta_std=1.0 if sp else 0.1,
                    bias_dist="expm1_u" if sp else "step_u")


@pytest.mark.parametrize("case", SMALL)
def test_fwd_small_and_ragged(case):
    check_fwd(small_workload(*case))


def test_fwd_ckpt_holds_chunk_end_states():
    w = small_workload(2, 6, 200, 16, "f32", True, True, True, True, "neg_lognormal")
    inp = generate(w)
    dv = to_device(inp, w)
    out, last, ck = run_fwd(dv, w, return_ckpt=True)
    ck = to_f64(ck).reshape(2, 6, -1, 16)
    assert ck.shape[2] == math.ceil(200 / ssm_scan.CKPT_CHUNK)
    for k in range(ck.shape[2]):
        tend = min(200, (k + 1) * ssm_scan.CKPT_CHUNK)
        _, st = oracle.fwd(inp["u_f64"][..., :tend], inp["delta_f64"][..., :tend], inp["A_f64"],
                           inp["B_f64"][..., :tend], inp["C_f64"][..., :tend], inp["D_f64"],
                           inp["z_f64"][..., :tend], inp["delta_bias_f64"], True)
        assert_close_io(ck[:, :, k], st, "f32", f"ckpt[{k}]")


def test_fwd_unaligned_rows_use_elementwise_path():
    """Rows that are not 16-byte aligned (odd L, offset base) still match."""
    w = small_workload(2, 5, 61, 16, "bf16", True, True, True, True, "neg_lognormal")
    inp = generate(w)
    dv = to_device(inp, w)
    shifted = {}
    for k in ("u", "delta", "z", "B", "C"):
        t = dv[k]
        buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
        v = buf[1:].view(t.shape)
        v.copy_(t)
        shifted[k] = v
    dv.update(shifted)
    out, last, _ = run_fwd(dv, w)
    ref, rlast = oracle.fwd_workload(inp, w)
    assert_close_io(to_f64(out), ref, "bf16")


def test_fwd_on_side_stream():
    w = small_workload(2, 33, 150, 16, "f32", True, True, True, True, "neg_lognormal")
    inp = generate(w)
    dv = to_device(inp, w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out, last, _ = ssm_scan.selective_scan_fwd(dv["u"], dv["delta"], dv["A"], dv["B"],
                                                   dv["C"], dv["D"], dv["z"], dv["delta_bias"],
                                                   True, return_last_state=True)
    s.synchronize()
    ref, _ = oracle.fwd_workload(inp, w)
    assert_close_io(to_f64(out), ref, "f32")


def test_fwd_repeatable_bitwise():
    w = small_workload(2, 40, 300, 16, "bf16", True, True, True, True, "neg_lognormal")
    dv = to_device(generate(w), w)
    o1, _, _ = run_fwd(dv, w)
    o2, _, _ = run_fwd(dv, w)
    assert torch.equal(o1, o2)


# ------------------------------------------------------------------ backward

def check_bwd(w: Workload, use_ckpt: bool, path=None):
    inp = generate(w, with_dout=True)
    dv = to_device(inp, w)
    ck = None
    if use_ckpt:
        _, _, ck = run_fwd(dv, w, return_ckpt=True)
    g = ssm_scan.selective_scan_bwd(dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"],
                                    dv["z"], dv["delta_bias"], w.softplus, dv["dout"], ckpt=ck)
    torch.cuda.synchronize()
    if path is not None:   # the kernel the library chose for this shape
        assert ssm_scan.last_kernel_path() == path
    ref = oracle.bwd_workload(inp, w)
    assert set(g) == set(ref)
    errs = {}
    for k in ref:
        errs[k] = assert_close_grad(to_f64(g[k]), ref[k], k)
    return errs


BWD_SMALL = [
    (1, 3, 12, 4, "f32", True, True, True, True, "neg_lognormal"),
    (2, 5, 70, 16, "f32", True, True, True, True, "neg_lognormal"),
    (2, 37, 200, 16, "bf16", True, True, True, True, "neg_lognormal"),
    (1, 9, 129, 8, "f32", False, False, False, False, "neg_lognormal"),
    (2, 17, 64, 32, "f32", True, True, True, True, "neg_lognormal"),
    (1, 70, 100, 2, "bf16", True, True, True, True, "neg_lognormal"),
    (1, 70, 100, 1, "f32", True, False, True, True, "neg_lognormal"),
]


@pytest.mark.parametrize("case", BWD_SMALL)
@pytest.mark.parametrize("use_ckpt", [True, False])
def test_bwd_small(case, use_ckpt):
    check_bwd(small_workload(*case), use_ckpt)


def test_bwd_layer_shape_full():
    check_bwd(WORKLOADS["mamba130m_layer_fwdbwd"], use_ckpt=True, path="bwd:tma")


# Shapes with dstate 16, 16-byte aligned rows and at least one channel row per
# SM take the TMA-fed persistent backward; these cover its ragged last tile and
# window, fp32 io, several passes per CTA, CTAs whose rows span two batch rows,
# CTAs with mostly idle warps, and the optional inputs switched off.
BWD_TMA_CASES = [
    # batch, dim, L, N, io, z, D, bias, softplus, A_dist
    (2, 2400, 72, 16, "bf16", True, True, True, True, "neg_lognormal"),
    (3, 2000, 40, 16, "f32", True, False, True, True, "neg_lognormal"),
    (2, 15000, 16, 16, "bf16", True, True, True, True, "neg_lognormal"),
    (1, 4800, 1000, 16, "bf16", True, True, True, True, "neg_n1"),
    (2, 3000, 200, 16, "f32", False, False, False, True, "neg_lognormal"),
    (2, 2400, 64, 16, "bf16", True, True, True, False, "neg_lognormal"),
    (1, 200, 64, 16, "bf16", True, True, True, True, "neg_lognormal"),
    (1, 1500, 132, 16, "f32", True, True, True, True, "neg_lognormal"),
    (4, 700, 256, 16, "bf16", False, True, True, True, "neg_lognormal"),
]


@pytest.mark.parametrize("case", BWD_TMA_CASES)
@pytest.mark.parametrize("use_ckpt", [True, False])
def test_bwd_tma_path(case, use_ckpt):
    check_bwd(small_workload(*case), use_ckpt)


def test_bwd_tma_gradients_8_byte_aligned():
    """du, dΔ and dz that are 8- but not 16-byte aligned still take the TMA
    backward; its epilogue then stores element by element.  The gradients
    equal those of 16-byte aligned buffers bit for bit, and the kernel is the
    TMA one."""
    w = small_workload(2, 2400, 72, 16, "bf16", True, True, True, True, "neg_lognormal")
    inp = generate(w, with_dout=True)
    dv = to_device(inp, w)
    _, _, ck = run_fwd(dv, w, return_ckpt=True)
    shape = ssm_scan.make_shape(w.batch, w.dim, w.seqlen, w.dstate, dv["u"].dtype)
    n = w.batch * w.dim * w.seqlen
    f32 = dict(device="cuda", dtype=torch.float32)

    def grads(offset):
        g = {k: torch.zeros(n + 4, **f32)[offset:offset + n].view(w.batch, w.dim, w.seqlen)
             for k in ("du", "ddelta", "dz")}
        g["dA"] = torch.zeros(w.dim, w.dstate, **f32)
        g["dB"] = torch.zeros(w.batch, w.dstate, w.seqlen, **f32)
        g["dC"] = torch.zeros(w.batch, w.dstate, w.seqlen, **f32)
        g["dD"] = torch.zeros(w.dim, **f32)
        g["ddelta_bias"] = torch.zeros(w.dim, **f32)
        ssm_scan.bwd_raw(shape, dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"],
                         dv["delta_bias"], w.softplus, dv["dout"], ck, g["du"], g["ddelta"], g["dA"],
                         g["dB"], g["dC"], g["dD"], g["dz"], g["ddelta_bias"], None)
        torch.cuda.synchronize()
        assert ssm_scan.last_kernel_path() == "bwd:tma"
        return g

    g16, g8 = grads(0), grads(2)
    assert g8["du"].data_ptr() % 16 == 8
    for k in ("du", "ddelta", "dz"):
        assert torch.equal(g8[k], g16[k]), k
    # the parameter and dB/dC sums take float atomics in a run-dependent order
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        torch.testing.assert_close(g8[k], g16[k], rtol=1e-5, atol=1e-5)


# ------------------------------------------------------------------ TMA forward path
# Shapes with >= 32 channels per SM and L a multiple of 8 take the TMA-fed
# persistent kernel; these cover its ragged last tile, fp32 io, N = 8 / 32,
# several passes per CTA and CTAs whose rows span two batch rows.
TMA_CASES = [
    # batch, dim, L, N, io, z, D, bias, softplus, A_dist
    (2, 2400, 72, 16, "bf16", True, True, True, True, "neg_lognormal"),
    (3, 2000, 40, 16, "f32", True, False, True, True, "neg_lognormal"),
    (2, 2400, 64, 8, "bf16", False, True, False, True, "neg_lognormal"),
    (2, 2400, 48, 32, "bf16", True, True, True, False, "neg_lognormal"),
    (2, 15000, 16, 16, "bf16", True, True, True, True, "neg_lognormal"),
    (4, 5120, 24, 16, "bf16", True, True, True, True, "neg_lognormal"),
    (1, 4800, 1000, 16, "bf16", True, True, True, True, "neg_n1"),
    (2, 3000, 200, 16, "f32", False, False, False, True, "neg_lognormal"),
    # fewer rows per SM: 8 and 16 lanes per channel
    (2, 2960, 64, 16, "bf16", True, True, True, True, "neg_lognormal"),
    (1, 2000, 264, 16, "bf16", True, True, True, True, "neg_lognormal"),
    (1, 1500, 128, 16, "f32", True, True, True, True, "neg_lognormal"),
    (1, 3000, 64, 32, "bf16", True, True, True, True, "neg_lognormal"),
    (2, 2400, 64, 8, "f32", True, True, True, True, "neg_lognormal"),
    (1, 200, 64, 16, "bf16", True, True, True, True, "neg_lognormal"),
]


@pytest.mark.parametrize("case", TMA_CASES)
def test_fwd_tma_path(case):
    check_fwd(small_workload(*case))


def test_fwd_tma_ckpt_and_state():
    w = small_workload(2, 2400, 136, 16, "bf16", True, True, True, True, "neg_lognormal")
    inp = generate(w)
    dv = to_device(inp, w)
    out, last, ck = run_fwd(dv, w, return_ckpt=True)
    ck = to_f64(ck).reshape(2, 2400, -1, 16)
    chans = slice(0, 2400, 37)
    sub = subset_channels(inp, chans)
    for k in range(ck.shape[2]):
        tend = min(136, (k + 1) * ssm_scan.CKPT_CHUNK)
        _, st = oracle.fwd(sub["u_f64"][..., :tend], sub["delta_f64"][..., :tend], sub["A_f64"],
                           sub["B_f64"][..., :tend], sub["C_f64"][..., :tend], sub["D_f64"],
                           sub["z_f64"][..., :tend], sub["delta_bias_f64"], True)
        assert_close_io(ck[:, chans, k], st, "bf16", f"ckpt[{k}]")


def _run_forced(kernel, shape_args):
    """Runs one forward in a fresh process with SSM_FWD_KERNEL set; returns its
    stdout (the kernel choice is read once per process)."""
    import os
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, %r); sys.path.insert(0, %r)\n"
        "import torch, numpy as np, oracle\n"
        "from selective_state_space_50_b200 import ssm_scan\n"
        "from selective_state_space_50_b200.workloads import Workload, generate, to_torch\n"
        "w = Workload('f', *%r, seed=5, A_dist='neg_lognormal', D_dist='u0.5_1.5')\n"
        "inp = generate(w); dv = to_torch(inp, w, 'cuda')\n"
        "try:\n"
        "    out, _, _ = ssm_scan.selective_scan_fwd(dv['u'], dv['delta'], dv['A'], dv['B'], dv['C'],"
        " dv['D'], dv['z'], dv['delta_bias'], True)\n"
        "    torch.cuda.synchronize()\n"
        "except ssm_scan.SSMError as e:\n"
        "    print('SSMError', e.status); raise SystemExit(0)\n"
        "ref, _ = oracle.fwd_workload(inp, w)\n"
        "err = np.abs(out.float().cpu().double().numpy() - ref) / (1 + np.abs(ref))\n"
        "print('maxerr', err.max())\n"
    ) % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
         os.path.dirname(os.path.abspath(__file__)), shape_args)
    env = dict(os.environ, SSM_FWD_KERNEL=kernel)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stdout


def test_forced_general_backward():
    """SSM_BWD_KERNEL=general keeps a shape the TMA backward covers on the
    general kernel; both agree with the oracle."""
    import os
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, %r); sys.path.insert(0, %r)\n"
        "import torch, numpy as np, oracle\n"
        "from selective_state_space_50_b200 import ssm_scan\n"
        "from selective_state_space_50_b200.workloads import Workload, generate, to_torch\n"
        "w = Workload('f', 2, 64, 1200, 16, 'bf16', seed=6, A_dist='neg_lognormal', D_dist='u0.5_1.5')\n"
        "inp = generate(w, with_dout=True); dv = to_torch(inp, w, 'cuda')\n"
        "g = ssm_scan.selective_scan_bwd(dv['u'], dv['delta'], dv['A'], dv['B'], dv['C'], dv['D'],"
        " dv['z'], dv['delta_bias'], True, dv['dout'])\n"
        "torch.cuda.synchronize()\n"
        "ref = oracle.bwd_workload(inp, w)\n"
        "print('maxrel', max(float(np.linalg.norm(g[k].double().cpu().numpy() - ref[k]) /"
        " np.linalg.norm(ref[k])) for k in ref))\n"
    ) % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
         os.path.dirname(os.path.abspath(__file__)))
    for kern in ("general", "auto"):
        env = dict(os.environ, SSM_BWD_KERNEL=kern)
        r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                           timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        assert float(r.stdout.split()[-1]) <= 1e-3, r.stdout


def test_forced_kernel_selection():
    # batch, seqlen, dim, dstate, io
    big = (2, 64, 2400, 16, "bf16")
    small = (1, 64, 40, 16, "bf16")
    for kern in ("tma", "general"):
        outp = _run_forced(kern, big)
        assert "maxerr" in outp and float(outp.split()[-1]) <= 2e-2, outp
    # the TMA kernel refuses shapes it does not cover, as unsupported
    assert "SSMError %d" % ssm_scan.SSM_ERR_UNSUPPORTED in _run_forced("tma", small)
    outp = _run_forced("general", small)
    assert float(outp.split()[-1]) <= 2e-2
