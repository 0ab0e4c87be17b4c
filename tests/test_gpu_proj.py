"""GPU parity of the selection projections (ssm_selection_projections, the
tcgen05 tensor-core kernels) against the fp64 oracle, and of projections
followed by the scan against the oracle's projections followed by its scan.

Tolerance.  Each output is an fp32 sum of bf16 products rounded once to
bf16: against the fp64 value the rounding alone is at most 2^-9 |ref| and
the fp32 accumulation adds about K 2^-24 Σ|a b|.  dt_low, B and C are
checked against |gpu - ref| <= 2^-8 |ref| + 4e-3 rms(ref).  delta is a sum
over the STORED dt_low, and a stored dt_low value may be the neighbouring
bf16 number of the oracle's one (the fp32 and fp64 sums fall on either side
of a rounding boundary): one step is at most 2^-7 |dt_low|.  So delta gets
the propagated bound 2^-8 |ref| + 2^-7 Σ_r |W_dt[d, r]| |dt_low[r]| +
4e-3 rms(ref)."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_50_b200 import ssm_scan
from selective_state_space_50_b200 import workloads as W

from helpers import to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm_scan.load_library()


def dev_bf16(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def assert_bf16_close(got, ref, name, extra=None):
    g = to_f64(got)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    err = np.abs(g - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 4e-3 * rms
    if extra is not None:
        bound = bound + extra
    bad = err > bound
    assert not bad.any(), (f"{name}: {int(bad.sum())} of {ref.size} outside, max err "
                           f"{err.max():.3e}, max ratio {(err / np.maximum(bound, 1e-30)).max():.2f}")


CASES = [
    # batch, dim, seqlen, dstate, dt_rank
    (2, 64, 64, 16, 8),          # one tile everywhere, K shorter than a slice
    (3, 200, 136, 16, 16),       # ragged M, K and L tails (L = 128 + 8)
    (1, 64, 8, 1, 8),            # shortest sequence, one state
    (2, 1536, 256, 16, 48),      # the 130M layer's channels and rank
    (1, 520, 2048, 32, 40),      # 32 states: 104 projected rows
    (2, 5120, 128, 16, 160),     # two M tiles for x_proj; 80 K slices
]


@pytest.mark.parametrize("case", CASES)
def test_projections_match_oracle(case):
    batch, dim, L, N, R = case
    inp = W.generate_projection(batch, dim, L, N, R, seed=77 + dim)
    x, Wx, Wdt = (dev_bf16(inp[k]) for k in ("x", "W_x", "W_dt"))
    delta, B, C, dt_low = ssm_scan.selection_projections(x, Wx, Wdt, N)
    torch.cuda.synchronize()
    ssm_scan.device_error_status()
    r_low, r_delta, r_B, r_C = oracle.projections(inp["x_f64"], inp["W_x_f64"], inp["W_dt_f64"], R, N)
    assert_bf16_close(dt_low, r_low, "dt_low")
    assert_bf16_close(B, r_B, "B")
    assert_bf16_close(C, r_C, "C")
    assert_bf16_close(delta, r_delta, "delta", delta_flip_bound(inp, r_low))


def delta_flip_bound(inp, r_low):
    """2^-7 Σ_r |W_dt[d, r]| |dt_low[b, r, t]|: the most delta can move when
    every stored dt_low value is the neighbouring bf16 number."""
    return 2.0 ** -7 * np.matmul(np.abs(inp["W_dt_f64"])[None], np.abs(oracle.bf16_round(r_low)))


def test_projections_full_layer_shape():
    """The Mamba-130M layer shape (batch 8, D 1536, L 2048, N 16, rank 48), all
    outputs compared element by element."""
    batch, dim, L, N, R = 8, 1536, 2048, 16, 48
    inp = W.generate_projection(batch, dim, L, N, R, seed=1005)
    x, Wx, Wdt = (dev_bf16(inp[k]) for k in ("x", "W_x", "W_dt"))
    delta, B, C, dt_low = ssm_scan.selection_projections(x, Wx, Wdt, N)
    torch.cuda.synchronize()
    ssm_scan.device_error_status()
    r_low, r_delta, r_B, r_C = oracle.projections(inp["x_f64"], inp["W_x_f64"], inp["W_dt_f64"], R, N)
    for got, ref, name in ((dt_low, r_low, "dt_low"), (B, r_B, "B"), (C, r_C, "C")):
        assert_bf16_close(got, ref, name)
    assert_bf16_close(delta, r_delta, "delta", delta_flip_bound(inp, r_low))


def test_pages_rank_one_broadcast_form():
    """Linear_1 broadcast over channels: rank 8 with only column 0 of W_dt set
    to ones and only row 0 of the rank block of W_x nonzero.  Every channel
    gets the same delta, equal to the stored dt_low row 0."""
    batch, dim, L, N, R = 2, 128, 64, 16, 8
    inp = W.generate_projection(batch, dim, L, N, R, seed=9)
    wx = inp["W_x"].copy()
    wx[1:R] = 0
    wdt = np.zeros((dim, R), dtype=np.uint16)
    wdt[:, 0] = 0x3F80                      # bf16 1.0
    x, Wx, Wdt = dev_bf16(inp["x"]), dev_bf16(wx), dev_bf16(wdt)
    delta, B, C, dt_low = ssm_scan.selection_projections(x, Wx, Wdt, N)
    torch.cuda.synchronize()
    d = to_f64(delta)
    low = to_f64(dt_low)
    for c in range(dim):
        np.testing.assert_array_equal(d[:, c], low[:, 0])
    assert np.all(low[:, 1:] == 0)


def test_projections_feed_the_scan():
    """Projections then the forward scan on the GPU, against the oracle's
    projections (outputs stored as bf16, as the path stores them) and the
    oracle's scan; bf16 scan tolerance 2e-2 (1 + |y|)."""
    batch, dim, L, N, R = 2, 256, 512, 16, 16
    inp = W.generate_projection(batch, dim, L, N, R, seed=21)
    x, Wx, Wdt = (dev_bf16(inp[k]) for k in ("x", "W_x", "W_dt"))
    r = np.random.default_rng(5)
    A = (-np.exp(r.standard_normal((dim, N)))).astype(np.float32)
    Dv = r.uniform(0.5, 1.5, dim).astype(np.float32)
    bias = np.log(np.expm1(r.uniform(1e-3, 0.1, dim))).astype(np.float32)
    zb = W.round_to_bf16_bits(r.standard_normal((batch, dim, L)))
    delta, B, C, _ = ssm_scan.selection_projections(x, Wx, Wdt, N)
    out, _, _ = ssm_scan.selective_scan_fwd(x, delta, torch.from_numpy(A).cuda(), B, C,
                                            torch.from_numpy(Dv).cuda(), dev_bf16(zb),
                                            torch.from_numpy(bias).cuda(), True)
    torch.cuda.synchronize()
    _, r_delta, r_B, r_C = oracle.projections(inp["x_f64"], inp["W_x_f64"], inp["W_dt_f64"], R, N)
    ref, _ = oracle.fwd(inp["x_f64"], oracle.bf16_round(r_delta), A.astype(np.float64),
                        oracle.bf16_round(r_B), oracle.bf16_round(r_C), Dv.astype(np.float64),
                        W.bf16_bits_to_f64(zb), bias.astype(np.float64), True)
    got = to_f64(out)
    err = np.abs(got - ref)
    assert (err <= 2e-2 * (1 + np.abs(ref))).all(), err.max()
