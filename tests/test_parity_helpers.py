"""The comparison helpers of the GPU parity tests, checked on the CPU: a
wrong row that hides under the normwise bound fails the per-row bound, a
dropped row must be exactly zero, and the last-tile token selection covers
each expert's ragged tail."""
import numpy as np

from tests import parity


def test_per_row_bound_catches_a_small_wrong_row():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal((64, 32))
    ref[5] *= 1e-3                      # one row far smaller than the rest
    Y = ref.copy()
    Y[5] = -ref[5]                      # that row has the wrong sign
    assert parity.rel_err(Y, ref) < 2e-2          # normwise: hidden
    assert parity.row_rel_err(Y, ref) > 1.0       # per row: caught
    try:
        parity.assert_rows_close(Y, ref, 2e-2)
    except AssertionError as e:
        assert "per-row" in str(e)
    else:
        raise AssertionError("the wrong row was not caught")


def test_zero_reference_rows_must_be_exactly_zero():
    ref = np.ones((3, 4))
    ref[1] = 0.0
    Y = ref.copy()
    assert parity.row_rel_err(Y, ref) == 0.0
    Y[1, 2] = 1e-30
    assert parity.row_rel_err(Y, ref) == float("inf")


def test_last_tile_tokens_cover_each_tail():
    # expert 0: 300 rows (tail 256..299), expert 1: empty, expert 2: 256 rows (full last block),
    # expert 3: 5 rows
    counts = [300, 0, 256, 5]
    offs = np.concatenate([[0], np.cumsum(counts)])
    st = np.arange(offs[-1]) % 1000 + 10_000     # distinct token ids per row
    got = parity.last_tile_tokens({"offsets": offs, "slot_token": st})
    want = np.unique(np.concatenate([st[256:300], st[300:556], st[556:561]]))
    np.testing.assert_array_equal(got, want)
    got128 = parity.last_tile_tokens({"offsets": offs, "slot_token": st}, tile=128)
    want128 = np.unique(np.concatenate([st[256:300], st[300 + 128:556], st[556:561]]))
    np.testing.assert_array_equal(got128, want128)
