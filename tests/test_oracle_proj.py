"""Pins of the oracle's selection projections (oracle.projections) and of its
bf16 rounding, against facts that do not come from the oracle itself:
one-hot weights that must copy input channels, the pages' rank-1 broadcast
form of the step-size projection, linearity, and torch's own bf16 cast."""
import numpy as np
import pytest
import torch

import oracle


def test_bf16_round_worked_values():
    # bf16 keeps 8 significant bits: the spacing just above 1 is 2^-7
    v = np.array([1.0, 1 + 2**-8, 1 + 3 * 2**-8, 1 + 2**-7 + 2**-9, -2.5, 0.0, -0.0,
                  2.0**-130, 65504.0])
    want = np.array([1.0, 1.0,        # tie -> even (1.0)
                     1 + 2**-6,       # tie -> even (mantissa ...10)
                     1 + 2**-7, -2.5, 0.0, -0.0,
                     2.0**-130,       # exactly representable subnormal
                     65536.0])        # 65504 = 1.9990234 * 2^15 rounds up
    np.testing.assert_array_equal(oracle.bf16_round(v), want)


def test_bf16_round_matches_torch_cast():
    r = np.random.default_rng(0)
    v = (r.standard_normal(100000) * np.exp(r.uniform(-20, 20, 100000))).astype(np.float32)
    t = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.bf16_round(v.astype(np.float64)), t)


def one_hot_case(R, N, dim):
    """W_x picks channel 3j+1 (mod dim) for output row j; W_dt[d] picks rank d mod R."""
    M = R + 2 * N
    W_x = np.zeros((M, dim))
    for j in range(M):
        W_x[j, (3 * j + 1) % dim] = 1.0
    W_dt = np.zeros((dim, R))
    for d in range(dim):
        W_dt[d, d % R] = 1.0
    return W_x, W_dt


@pytest.mark.parametrize("R,N", [(8, 16), (16, 4), (1, 2)])
def test_one_hot_weights_route_channels(R, N):
    dim, L, b = 64, 24, 2
    r = np.random.default_rng(R + N)
    x = oracle.bf16_round(r.standard_normal((b, dim, L)))
    W_x, W_dt = one_hot_case(R, N, dim)
    dt_low, delta, B, C = oracle.projections(x, W_x, W_dt, R, N)
    for j in range(R):
        np.testing.assert_array_equal(dt_low[:, j], x[:, (3 * j + 1) % dim])
    for n in range(N):
        np.testing.assert_array_equal(B[:, n], x[:, (3 * (R + n) + 1) % dim])
        np.testing.assert_array_equal(C[:, n], x[:, (3 * (R + N + n) + 1) % dim])
    for d in range(dim):
        # x is bf16-exact, so the stored intermediate equals the copied channel
        np.testing.assert_array_equal(delta[:, d], dt_low[:, d % R])


def test_rank_one_broadcast_is_the_pages_linear_1():
    """R = 1 with an all-ones up-projection gives the same step-size input to
    every channel: Broadcast_D(Linear_1(x)), and it is w . x_t."""
    dim, L, b, N = 48, 16, 3, 4
    r = np.random.default_rng(7)
    x = r.standard_normal((b, dim, L))
    W_x = r.standard_normal((1 + 2 * N, dim))
    W_dt = np.ones((dim, 1))
    dt_low, delta, _, _ = oracle.projections(x, W_x, W_dt, 1, N, store_low_bf16=False)
    for d in range(dim):
        np.testing.assert_array_equal(delta[:, d], delta[:, 0])
    # w . x_t, summed exactly (math.fsum) for a few (b, t)
    import math
    for bb, t in [(0, 0), (1, 7), (2, 15)]:
        ref = math.fsum(W_x[0, k] * x[bb, k, t] for k in range(dim))
        assert abs(dt_low[bb, 0, t] - ref) <= 1e-12 * (1 + abs(ref))


def test_projections_are_linear_and_rows_are_independent():
    dim, L, b, R, N = 40, 12, 2, 8, 4
    r = np.random.default_rng(3)
    x1, x2 = r.standard_normal((2, b, dim, L))
    W_x = r.standard_normal((R + 2 * N, dim))
    W_dt = r.standard_normal((dim, R))
    p1 = oracle.projections(x1, W_x, W_dt, R, N, store_low_bf16=False)
    p2 = oracle.projections(x2, W_x, W_dt, R, N, store_low_bf16=False)
    p12 = oracle.projections(2.0 * x1 - 0.5 * x2, W_x, W_dt, R, N, store_low_bf16=False)
    for a, b_, c in zip(p1, p2, p12):
        np.testing.assert_allclose(c, 2.0 * a - 0.5 * b_, rtol=1e-12, atol=1e-12)
    # zeroing row R (the first row of B) changes B[:, 0] only
    W_x0 = W_x.copy()
    W_x0[R] = 0.0
    q = oracle.projections(x1, W_x0, W_dt, R, N, store_low_bf16=False)
    np.testing.assert_array_equal(q[0], p1[0])
    np.testing.assert_array_equal(q[1], p1[1])
    np.testing.assert_array_equal(q[3], p1[3])
    assert np.all(q[2][:, 0] == 0.0)
    np.testing.assert_array_equal(q[2][:, 1:], p1[2][:, 1:])


def test_second_product_uses_the_stored_intermediate():
    dim, L, b, R, N = 32, 8, 1, 8, 2
    r = np.random.default_rng(11)
    x = r.standard_normal((b, dim, L))
    W_x = r.standard_normal((R + 2 * N, dim))
    W_dt = r.standard_normal((dim, R))
    dt_low, delta, _, _ = oracle.projections(x, W_x, W_dt, R, N, store_low_bf16=True)
    low = oracle.bf16_round(dt_low)
    assert not np.array_equal(low, dt_low)
    # delta depends on dt_low only through its rounded values
    for d in (0, 5, 31):
        for t in (0, 7):
            ref = sum(W_dt[d, k] * low[0, k, t] for k in range(R))
            assert abs(delta[0, d, t] - ref) <= 1e-12 * (1 + abs(ref))
