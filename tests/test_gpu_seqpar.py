"""GPU parity of the sequence-segment entry points and of the sequence-sharded
forward run with all segments on one GPU (the protocol's ranks never wait on
each other, so one GPU runs them in turn):

  * ssm_selective_scan_fwd_segment from a given state h0, against the oracle's
    forward from the same h0 (TMA and general kernels, ZOH);
  * its delta sums and ssm_scan_combine_carries against the oracle's;
  * seqpar.cuda_forward_segments (pass 1, combine, pass 2) against the
    oracle's forward over the whole sequence.
Tolerances are the forward's (helpers.py)."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_50_b200 import seqpar, ssm_scan
from selective_state_space_50_b200.workloads import WORKLOADS, Workload, generate, to_torch

from helpers import assert_close_io, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm_scan.load_library()


def case(batch, dim, L, N, io, seed, **kw):
    w = Workload("seg", batch, L, dim, N, io, seed=seed, A_dist="neg_lognormal",
                 D_dist="u0.5_1.5", **kw)
    inp = generate(w)
    return w, inp, to_torch(inp, w, "cuda")


SEG_CASES = [
    # batch, dim, L, N, io, zoh
    (2, 2400, 72, 16, "bf16", False),     # TMA kernel
    (1, 4800, 256, 16, "bf16", False),    # TMA kernel, one batch row
    (2, 64, 100, 16, "f32", False),       # general kernel
    (2, 40, 64, 8, "f32", True),          # general kernel, zero-order hold
    (2, 2400, 72, 16, "bf16", True),      # TMA kernel, zero-order hold
]


@pytest.mark.parametrize("c", SEG_CASES)
def test_segment_from_initial_state(c):
    batch, dim, L, N, io, zoh = c
    w, inp, dv = case(batch, dim, L, N, io, seed=300 + dim)
    r = np.random.default_rng(dim)
    h0 = r.standard_normal((batch, dim, N)).astype(np.float32)
    out, last, dsum = ssm_scan.selective_scan_fwd_segment(
        dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"], dv["delta_bias"], True,
        h0=torch.from_numpy(h0).cuda(), zoh=zoh)
    torch.cuda.synchronize()
    ref, rlast = oracle.fwd(inp["u_f64"], inp["delta_f64"], inp["A_f64"], inp["B_f64"],
                            inp["C_f64"], inp["D_f64"], inp["z_f64"], inp["delta_bias_f64"], True,
                            zoh=zoh, h0=h0.astype(np.float64))
    assert_close_io(to_f64(out), ref, io, "out")
    assert_close_io(to_f64(last), rlast, "f32", "last_state")
    rds = oracle.delta_sums(inp["delta_f64"], inp["delta_bias_f64"], True)
    np.testing.assert_allclose(to_f64(dsum), rds, rtol=1e-4, atol=1e-4 * np.sqrt(L))


def test_combine_carries_matches_oracle():
    r = np.random.default_rng(1)
    S, batch, dim, N = 5, 3, 70, 16
    A = (-np.exp(r.standard_normal((dim, N)))).astype(np.float32)
    ds = r.uniform(0, 3, (S, batch, dim)).astype(np.float32)
    ends = r.standard_normal((S, batch, dim, N)).astype(np.float32)
    h0 = r.standard_normal((batch, dim, N)).astype(np.float32)
    t = lambda x: torch.from_numpy(x).cuda()
    for hh in (None, h0):
        got = ssm_scan.combine_carries(t(A), t(ds), t(ends), None if hh is None else t(hh))
        torch.cuda.synchronize()
        want = oracle.combine_carries(A, ds, ends, hh)
        np.testing.assert_allclose(to_f64(got), want, rtol=1e-5, atol=1e-5)


SHARD_CASES = [
    # batch, dim, L, N, io, nseg
    (2, 2400, 256, 16, "bf16", 2),
    (1, 4800, 1024, 16, "bf16", 8),
    (2, 64, 96, 16, "f32", 3),
    (8, 1536, 256, 16, "bf16", 2),        # 4 lanes per channel (the layer shape's split)
]


@pytest.mark.parametrize("c", SHARD_CASES)
def test_sharded_forward_equals_whole_sequence(c):
    batch, dim, L, N, io, nseg = c
    w, inp, dv = case(batch, dim, L, N, io, seed=400 + L)
    out, last = seqpar.cuda_forward_segments(dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"],
                                             dv["D"], dv["z"], dv["delta_bias"], True, nseg=nseg)
    torch.cuda.synchronize()
    ref, rlast = oracle.fwd_workload(inp, w)
    assert_close_io(to_f64(out), ref, io, "out")
    assert_close_io(to_f64(last), rlast, "f32", "last_state")


def test_sharded_long_context_sampled_channels():
    """The long-context workload (L = 131072, D = 2048) cut into 8 segments of
    16384 steps: out and final state of 16 sampled channels against the
    oracle over the whole sequence."""
    w = WORKLOADS["long_context"]
    inp = generate(w)
    dv = to_torch(inp, w, "cuda")
    out, last = seqpar.cuda_forward_segments(dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"],
                                             dv["D"], dv["z"], dv["delta_bias"], True, nseg=8)
    torch.cuda.synchronize()
    ch = np.arange(0, w.dim, w.dim // 16)
    sub = {k: (v[:, ch] if k.split("_f64")[0] in ("u", "delta", "z") else
               v[ch] if k.split("_f64")[0] in ("A", "D", "delta_bias") else v)
           for k, v in inp.items() if k.endswith("_f64")}
    ref, rlast = oracle.fwd(sub["u_f64"], sub["delta_f64"], sub["A_f64"], sub["B_f64"],
                            sub["C_f64"], sub["D_f64"], sub["z_f64"], sub["delta_bias_f64"], True)
    assert_close_io(to_f64(out[:, ch]), ref, "bf16", "out")
    assert_close_io(to_f64(last[:, ch]), rlast, "f32", "last_state")
