"""GPU parity of the two-level scan along the sequence (ssm_selective_scan_fwd_ws):
chunk summaries, the carry combine, and every chunk rerun from its carry-in
(booiljung.github.io, "3.2 선택적 스캔(Selective Scan) 알고리즘" §2.2), against
the fp64 oracle and against the one-pass forward on the same inputs.

The library takes the two-level scan where its cost model expects it to win
(long sequences over few channel rows); the first cases are such shapes and
check that a workspace is asked for.  Other splits (4 lanes per channel with
the fp32 B/C copy, fp32 io, several passes) are forced with SSM_FWD_CHUNKS in
a child process, since the library reads that setting once per process."""
import os
import subprocess
import sys

import pytest
import torch

import oracle
from selective_state_space_50_b200 import ssm_scan
from selective_state_space_50_b200.workloads import Workload, generate

from helpers import assert_close_io, subset_channels, to_device, to_f64

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm_scan.load_library()


def _workload(case, seed=123):
    batch, dim, L, N, io, z, D, bias, sp, A_dist = case
    return Workload("chunked", batch, L, dim, N, io, seed=seed, has_z=z, has_D=D, has_bias=bias,
                    softplus=sp, A_dist=A_dist, D_dist="u0.5_1.5", delta_abs=not sp,
                    delta_std=1.0 if sp else 0.1, bias_dist="expm1_u" if sp else "step_u")


def _run(dv, w, chunked, ckpt=False):
    shape = ssm_scan.make_shape(w.batch, w.dim, w.seqlen, w.dstate, dv["u"].dtype)
    out = torch.empty_like(dv["u"])
    last = torch.empty(w.batch, w.dim, w.dstate, device="cuda", dtype=torch.float32)
    ck = (torch.empty(ssm_scan.ckpt_numel(shape), device="cuda", dtype=torch.float32)
          if ckpt else None)
    nws = ssm_scan.fwd_workspace_bytes(shape, w.softplus)
    ws = torch.empty(nws // 4, device="cuda", dtype=torch.float32) if (chunked and nws) else None
    ssm_scan.fwd_raw(shape, dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"],
                     dv["delta_bias"], w.softplus, out, last, ck, workspace=ws)
    torch.cuda.synchronize()
    return out, last, ck, nws


def check_case(case, require_chunked=True):
    w = _workload(case)
    inp = generate(w)
    dv = to_device(inp, w)
    out, last, _, nws = _run(dv, w, chunked=True)
    if require_chunked:
        assert nws > 0, "the shape should take the two-level scan"
        assert ssm_scan.last_kernel_path() == "fwd:chunked"
    chans = slice(0, w.dim, max(1, w.dim // 64))
    sub = subset_channels(inp, chans)
    ref, rlast = oracle.fwd_workload(sub, w.replace(dim=len(range(w.dim)[chans])))
    e = assert_close_io(to_f64(out)[:, chans], ref, w.io_dtype)
    assert_close_io(to_f64(last)[:, chans], rlast, "f32" if w.io_dtype == "f32" else "bf16",
                    "last_state")
    # the one-pass forward on the same inputs agrees as closely
    out1, _, _, _ = _run(dv, w, chunked=False)
    assert_close_io(to_f64(out), to_f64(out1), w.io_dtype, "out vs one pass")
    return nws, e


# shapes the cost model itself sends to the two-level scan
CASES = [
    # batch, dim, L, N, io, z, D, bias, softplus, A_dist
    (1, 256, 4096, 16, "bf16", True, True, True, True, "neg_lognormal"),
    (1, 128, 8192, 16, "bf16", True, True, True, True, "neg_n1"),
    (2, 50, 3000, 16, "bf16", True, True, True, True, "neg_lognormal"),    # ragged last chunk
    (1, 512, 2048, 8, "bf16", False, True, True, True, "neg_lognormal"),
    (1, 150, 8192, 16, "bf16", True, True, True, False, "neg_lognormal"),  # Δ given directly
    (3, 32, 6000, 16, "bf16", True, False, False, True, "neg_lognormal"),  # chunks span batch rows
]


@pytest.mark.parametrize("case", CASES)
def test_chunked_forward_matches_oracle_and_one_pass(case):
    check_case(case)


def test_chunked_checkpoints_match_one_pass():
    """Every chunk writes the checkpoints of its own steps: the buffer equals
    the one-pass forward's to fp32 rounding of the joined states."""
    w = _workload((1, 256, 4096, 16, "bf16", True, True, True, True, "neg_lognormal"))
    dv = to_device(generate(w), w)
    _, _, ck2, nws = _run(dv, w, chunked=True, ckpt=True)
    _, _, ck1, _ = _run(dv, w, chunked=False, ckpt=True)
    assert nws > 0
    assert_close_io(to_f64(ck2), to_f64(ck1), "f32", "ckpt vs one pass")


# splits forced with SSM_FWD_CHUNKS (child process): case, K
FORCED = [
    ((1, 2048, 8192, 16, "bf16", True, True, True, True, "neg_lognormal"), 6),   # 4 lanes, fp32 B/C
    ((1, 2048, 8192, 16, "bf16", True, True, True, True, "neg_n1"), 9),          # two passes per CTA
    ((2, 300, 2048, 16, "f32", True, True, True, True, "neg_lognormal"), 4),      # fp32 io
    ((1, 400, 2048, 32, "bf16", True, False, False, True, "neg_lognormal"), 3),
    ((1, 600, 2048, 16, "bf16", True, True, True, False, "neg_lognormal"), 2),
]


@pytest.mark.parametrize("case,K", FORCED)
def test_forced_chunk_counts(case, K):
    code = ("import sys; sys.path.insert(0, %r); sys.path.insert(0, %r)\n"
            "import test_gpu_chunked as t\n"
            "nws, e = t.check_case(%r)\n"
            "print('ok', nws, e)\n") % (ROOT, HERE, case)
    env = dict(os.environ, SSM_FWD_CHUNKS=str(K))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "ok" in r.stdout


def test_workspace_too_small_is_rejected():
    w = _workload(CASES[0])
    dv = to_device(generate(w), w)
    shape = ssm_scan.make_shape(w.batch, w.dim, w.seqlen, w.dstate, dv["u"].dtype)
    nws = ssm_scan.fwd_workspace_bytes(shape)
    assert nws > 0
    small = torch.empty(max(1, nws // 8), device="cuda", dtype=torch.float32)
    out = torch.empty_like(dv["u"])
    with pytest.raises(ssm_scan.SSMError) as e:
        ssm_scan.fwd_raw(shape, dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"],
                         dv["delta_bias"], True, out, None, None, workspace=small)
    assert e.value.status == ssm_scan.SSM_ERR_INVALID_ARG


def test_shapes_with_many_rows_need_no_workspace():
    for args in ((8, 1536, 2048, 16), (4, 5120, 2048, 16), (2, 64, 100, 16)):
        shape = ssm_scan.make_shape(*args, torch.bfloat16)
        assert ssm_scan.fwd_workspace_bytes(shape) == 0, args
