"""The oracle's pins catch plausible mistakes: each test below swaps in a
mutant of one oracle function (a swapped operand, a dropped step, a wrong sign
or index) and checks that at least one of the pins for that function fails.
The mutants live only here; the oracle itself is untouched."""
import numpy as np
import pytest

import oracle
import test_oracle as T
import test_oracle_proj as P

_orig_proj = oracle.projections
_orig_combine = oracle.combine_carries
_orig_dsum = oracle.delta_sums


def _proj_swap_bc(x, W_x, W_dt, R, N, store_low_bf16=True):
    low, delta, B, C = _orig_proj(x, W_x, W_dt, R, N, store_low_bf16)
    return low, delta, C, B


def _proj_no_storage_rounding(x, W_x, W_dt, R, N, store_low_bf16=True):
    return _orig_proj(x, W_x, W_dt, R, N, store_low_bf16=False)


def _proj_reversed_rank(x, W_x, W_dt, R, N, store_low_bf16=True):
    return _orig_proj(x, W_x, np.ascontiguousarray(np.asarray(W_dt)[:, ::-1]), R, N, store_low_bf16)


def _proj_rows_off_by_one(x, W_x, W_dt, R, N, store_low_bf16=True):
    W = np.roll(np.asarray(W_x, dtype=np.float64), 1, axis=0)
    return _orig_proj(x, W, W_dt, R, N, store_low_bf16)


PROJ_PINS = [
    lambda: P.test_one_hot_weights_route_channels(8, 16),
    lambda: P.test_one_hot_weights_route_channels(16, 4),
    P.test_rank_one_broadcast_is_the_pages_linear_1,
    P.test_projections_are_linear_and_rows_are_independent,
    P.test_second_product_uses_the_stored_intermediate,
]


def _fails(pins):
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    return failed


@pytest.mark.parametrize("mutant", [_proj_swap_bc, _proj_no_storage_rounding, _proj_reversed_rank,
                                    _proj_rows_off_by_one])
def test_projection_mutants_are_caught(monkeypatch, mutant):
    monkeypatch.setattr(oracle, "projections", mutant)
    assert _fails(PROJ_PINS) >= 1


def test_projection_pins_pass_on_the_oracle():
    assert _fails(PROJ_PINS) == 0


def _combine_inclusive(A, dsums, h_ends, h0=None):
    out = _orig_combine(A, dsums, h_ends, h0)
    decay = np.exp(np.asarray(dsums)[:, :, :, None] * np.asarray(A)[None, None])
    return decay * out + np.asarray(h_ends)      # the state after each segment, not before


def _combine_wrong_sign(A, dsums, h_ends, h0=None):
    with np.errstate(over="ignore", invalid="ignore"):     # exp(+|A| ΣΔ) overflows on purpose
        return _orig_combine(-np.asarray(A), dsums, h_ends, h0)


def _combine_drops_h0(A, dsums, h_ends, h0=None):
    return _orig_combine(A, dsums, h_ends, None)


def _dsum_no_softplus(delta, delta_bias=None, delta_softplus=True):
    return _orig_dsum(delta, delta_bias, False)


def _dsum_no_bias(delta, delta_bias=None, delta_softplus=True):
    return _orig_dsum(delta, None, delta_softplus)


SEG_PINS = [
    lambda: T.test_segments_reassembled_by_carries_equal_the_whole_scan((0, 64, 200)),
    lambda: T.test_segments_reassembled_by_carries_equal_the_whole_scan((0, 1, 97, 150, 200)),
    T.test_delta_sums_softplus_and_raw,
]


@pytest.mark.parametrize("name,mutant", [
    ("combine_carries", _combine_inclusive), ("combine_carries", _combine_wrong_sign),
    ("combine_carries", _combine_drops_h0), ("delta_sums", _dsum_no_softplus),
    ("delta_sums", _dsum_no_bias)])
def test_segment_mutants_are_caught(monkeypatch, name, mutant):
    monkeypatch.setattr(oracle, name, mutant)
    assert _fails(SEG_PINS) >= 1


def test_segment_pins_pass_on_the_oracle():
    assert _fails(SEG_PINS) == 0
