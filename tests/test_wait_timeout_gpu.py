"""A bounded device wait that runs out, on the GPU, without a fault (the kernels' waits poll a
limited number of times, then set the plan's status word and return or repair).

The general tiled kernel stages the next tile's rows by bulk copies completed on an mbarrier.
The test hook harp_test_inject_wait_timeout makes each staging barrier expect a few bytes more
than are copied and polls it only a few times, so every first wait runs out although every
issued copy lands.  The kernel must then report the timeout through the plan's status word
(harp_plan_device_status -> HARP_ERR_TIMEOUT), retire the extra bytes itself, wait (bounded)
for the copies it issued and finish with the right output; with the hook cleared the next
call is clean.  Nothing is left in flight and no wait is unbounded.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from structured_rotations_b200 import harp as HB
from tests._parity import check_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("name,rows,direction", [("d4096", 148 * 8 * 2 + 13, "inverse"),
                                                 ("d5120", 600, "forward")])
def test_staging_wait_runs_out_is_reported_and_repaired(monkeypatch, name, rows, direction):
    monkeypatch.setenv("HARP_KERNEL", "tiled")
    w = W.get(name)
    theta = W.draw_theta(O.theta_count(w.schedule), w.theta_sigma, w.theta_seed)
    gp = H.Plan(w.d, w.schedule, theta=theta, sign_seed=w.sign_seed).materialize()
    tr = O.Transform(O.make_plan(w.d, w.schedule, theta, sign_seed=w.sign_seed))
    enc = W.draw_encoded(w, 0, rows)
    x = torch.from_numpy(enc.view(np.int16)).view(torch.bfloat16).to(DEV)
    gp.device_status()                                  # clean before
    H.inject_wait_timeout(64, 16)
    try:
        y = gp.apply(x, direction=direction)
        assert H.last_kernel() == "harp_tiled_kernel"
    finally:
        H.inject_wait_timeout(0, 0)
    with pytest.raises(HB.HarpError) as e:
        gp.device_status()                              # synchronizes, reads and clears the word
    assert e.value.status == HB.HARP_ERR_TIMEOUT
    gp.device_status()                                  # cleared by the read
    sel = W.sample_rows(rows, 64)
    xf = W.decode_bf16(enc[sel])
    check_bf16(_bits(y)[sel], tr.apply(xf, direction), np.linalg.norm(xf, axis=1), O.round_bf16,
               f"{name} after a repaired timeout")
    y2 = gp.apply(x, direction=direction)               # hook cleared: no timeout, same bits
    gp.device_status()
    assert np.array_equal(_bits(y2), _bits(y))

