"""The seeded input generators (workloads/): every range of rows is the same whatever
range it is drawn with (rows are keyed by 256-row blocks), values are stored in the
workload's I/O type, and the upstream gradients of the calibration backward are
standard normal and independent of the rows themselves."""
import numpy as np
import pytest

import workloads as W


@pytest.mark.parametrize("name", ["d64", "d4096", "d5120"])
def test_row_ranges_agree(name):
    w = W.get(name)
    whole = W.draw_encoded(w, 0, 700)
    assert np.array_equal(W.draw_encoded(w, 250, 300), whole[250:550])
    up = W.draw_upstream(w, 0, 700)
    assert np.array_equal(W.draw_upstream(w, 511, 100), up[511:611])
    assert up.dtype == whole.dtype == (np.uint16 if w.dtype == "bf16" else np.float32)


def test_upstream_gradients_are_standard_normal_and_not_the_rows():
    w = W.get("d4096")
    g = W.decode_bf16(W.draw_upstream(w, 0, 64))
    x = W.decode_bf16(W.draw_encoded(w, 0, 64))
    assert abs(g.mean()) < 0.01 and abs(g.std() - 1.0) < 0.01
    c = np.corrcoef(g.ravel(), x.ravel())[0, 1]
    assert abs(c) < 0.01


def test_empty_draws():
    w = W.get("d64")
    assert W.draw_upstream(w, 5, 0).shape == (0, 64)


def test_two_sided_cases_of_the_bench():
    """The bench's smaller two-sided cases (--two-sided-cols): V's schedule multiplies out to
    the column count, the full size keeps the workload's own schedule, others are refused."""
    import bench
    w4 = W.get("two_sided")
    assert bench.two_sided_v_schedule(0, w4) == tuple(w4.schedule)
    assert bench.two_sided_v_schedule(w4.n_in, w4) == tuple(w4.schedule)
    for n, want in ((1024, (8, 8, 8, 2)), (2048, (8, 8, 8, 4)), (512, (8, 8, 8)), (64, (8, 8))):
        assert bench.two_sided_v_schedule(n, w4) == want
        assert int(np.prod(want)) == n
    for bad in (3000, 24, 12, 4):
        with pytest.raises(SystemExit):
            bench.two_sided_v_schedule(bad, w4)
