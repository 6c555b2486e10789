"""GPU parity of the cluster row kernel (harp_cluster_kernel): the rows' coordinates split over
the CTAs of a thread-block cluster at a stage t*, each CTA staging its share of the blocks in
shared memory once, one exchange between the two phases (HARP technical summary §2.1 Core
Architecture: stages of blocks on stride-separated groups).

Against the float64 oracle (fp32: 2e-6 ||x||; bf16: one ordinal step) and bit for bit against the
tiled kernel, whose stage arithmetic it shares, for the workload schedules and small ones, both
directions, bf16 / fp32 / bf16 -> fp32, batches of 1 row to several tiles with a ragged tail.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from tests._parity import check_bf16, check_f32

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

_PLANS = {}


def _plan(schedule, theta_seed, sign_seed, int8=False):
    key = (schedule, theta_seed, sign_seed, int8)
    if key not in _PLANS:
        d = int(np.prod(schedule))
        theta = W.draw_theta(O.theta_count(schedule), 0.2236, theta_seed)
        if int8:
            codes, scales = W.quantize_theta_int8(theta, O.stage_theta_counts(schedule))
            gp = H.Plan(d, schedule, codes=codes, scales=scales, sign_seed=sign_seed).materialize()
            op = O.make_plan(d, schedule, codes=codes, scales=scales, sign_seed=sign_seed)
        else:
            gp = H.Plan(d, schedule, theta=theta, sign_seed=sign_seed).materialize()
            op = O.make_plan(d, schedule, theta, sign_seed=sign_seed)
        _PLANS[key] = (gp, O.Transform(op))
    return _PLANS[key]


def _rows(d, rows, seed, dtype):
    rng = np.random.default_rng([d, rows, seed])
    x = rng.standard_normal((rows, d))
    x[rng.random((rows, d)) < 0.01] *= 20.0
    if dtype == "bf16":
        enc = W.encode_bf16(x)
        return W.decode_bf16(enc), torch.from_numpy(enc.view(np.int16)).view(torch.bfloat16).to(DEV)
    xf = x.astype(np.float32)
    return xf.astype(np.float64), torch.from_numpy(xf).to(DEV)


def _host(t):
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def _run(monkeypatch, kernel, gp, x, direction, out_dtype=None):
    monkeypatch.setenv("HARP_KERNEL", kernel)
    y = torch.empty(x.shape, dtype=out_dtype or x.dtype, device=DEV)
    gp.apply_ex(x, y, direction=direction)
    assert H.last_kernel() == ("harp_cluster_kernel" if kernel == "cluster" else "harp_tiled_kernel")
    torch.cuda.synchronize()
    return y


SCHEDULES = [((8, 8, 8, 8), False), ((8, 8, 8, 5, 2), False), ((8, 8, 8, 8, 2), True), ((8, 8, 8, 2), False),
             ((8, 8, 8), False), ((2, 8, 8, 4, 2), False), ((8, 7, 8, 8), False)]


@pytest.mark.parametrize("schedule,int8", SCHEDULES)
@pytest.mark.parametrize("direction", ["forward", "inverse"])
@pytest.mark.parametrize("rows", [1, 5, 16, 100])
def test_cluster_bf16_matches_oracle_and_tiled(monkeypatch, schedule, int8, direction, rows):
    """Every element within one bf16 step (or the fp32 floor) of the oracle.  The share of
    elements held to the floor is a statistic of the sample (below 1e-4): it is taken over this
    case's rows together with a 128-row batch of the same plan, since a handful of rows has
    fewer elements than one such element's share needs."""
    gp, tr = _plan(schedule, 2201, 3201, int8)
    xf, x = _rows(gp.d, rows, 1, "bf16")
    y = _run(monkeypatch, "cluster", gp, x, direction)
    bf, b = _rows(gp.d, 128, 11, "bf16")
    yb = _run(monkeypatch, "cluster", gp, b, direction)
    xs = np.concatenate([xf, bf])
    check_bf16(np.concatenate([_host(y), _host(yb)]), tr.apply(xs, direction), np.linalg.norm(xs, axis=1),
               O.round_bf16, f"cluster {schedule} {direction} {rows}")
    yt = _run(monkeypatch, "tiled", gp, x, direction)
    assert np.array_equal(_host(y), _host(yt))
    gp.device_status()


@pytest.mark.parametrize("schedule,int8", SCHEDULES[:4])
@pytest.mark.parametrize("direction", ["forward", "inverse"])
def test_cluster_fp32_and_widening(monkeypatch, schedule, int8, direction):
    gp, tr = _plan(schedule, 2202, 3202, int8)
    xf, x = _rows(gp.d, 37, 2, "f32")
    y = _run(monkeypatch, "cluster", gp, x, direction)
    check_f32(_host(y).astype(np.float64), tr.apply(xf, direction), np.linalg.norm(xf, axis=1),
              f"cluster fp32 {schedule} {direction}")
    assert np.array_equal(_host(y), _host(_run(monkeypatch, "tiled", gp, x, direction)))
    xb, xbt = _rows(gp.d, 21, 3, "bf16")
    yw = _run(monkeypatch, "cluster", gp, xbt, direction, torch.float32)
    check_f32(_host(yw).astype(np.float64), tr.apply(xb, direction), np.linalg.norm(xb, axis=1),
              f"cluster bf16->fp32 {schedule} {direction}")
    assert np.array_equal(_host(yw), _host(_run(monkeypatch, "tiled", gp, xbt, direction, torch.float32)))


@pytest.mark.parametrize("direction", ["forward", "inverse"])
def test_cluster_many_tiles_ragged_and_in_place(monkeypatch, direction):
    """Several tiles of rows (each cluster one tile), a ragged last tile, padded rows, and in
    place, at the int8 d = 8192 workload's schedule."""
    gp, tr = _plan((8, 8, 8, 8, 2), 2203, 3203, True)
    rows, ld = 203, 8192 + 64
    xf, x0 = _rows(gp.d, rows, 4, "bf16")
    x = torch.zeros(rows, ld, dtype=torch.bfloat16, device=DEV)
    x[:, :gp.d] = x0
    v = x[:, :gp.d]
    monkeypatch.setenv("HARP_KERNEL", "cluster")
    gp.apply(v, v, direction=direction)
    assert H.last_kernel() == "harp_cluster_kernel"
    torch.cuda.synchronize()
    got = _host(x)
    check_bf16(got[:, :gp.d], tr.apply(xf, direction), np.linalg.norm(xf, axis=1), O.round_bf16, "in place")
    assert not got[:, gp.d:].any()                      # the padding is never written
    gp.device_status()


def test_cluster_declines_what_it_does_not_cover(monkeypatch):
    monkeypatch.setenv("HARP_KERNEL", "cluster")
    small, _ = _plan((8, 8), 2204, 3204)                # d = 64: no split with 8-pencil runs
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(H.HarpError) as e:
        small.apply(x)
    assert e.value.status == H.HARP_ERR_UNSUPPORTED
    gp, _ = _plan((8, 8, 8, 8), 2201, 3201)
    buf = torch.zeros(4 * 4096 + 8, dtype=torch.bfloat16, device=DEV)
    xu = buf[1:1 + 4 * 4096].view(4, 4096)                # rows not 16-byte aligned
    with pytest.raises(H.HarpError) as e:
        gp.apply(xu, torch.empty(4, 4096, dtype=torch.bfloat16, device=DEV))
    assert e.value.status == H.HARP_ERR_UNSUPPORTED
    monkeypatch.delenv("HARP_KERNEL")
    gp.apply(xu, torch.empty(4, 4096, dtype=torch.bfloat16, device=DEV))   # auto: another kernel
    assert H.last_kernel() != "harp_cluster_kernel"


def test_small_batches_take_the_cluster_kernel_by_default(monkeypatch):
    monkeypatch.delenv("HARP_KERNEL", raising=False)
    gp, tr = _plan((8, 8, 8, 8, 2), 2201, 3201, True)
    xf, x = _rows(gp.d, 16, 5, "bf16")
    y = gp.apply(x)
    assert H.last_kernel() == "harp_cluster_kernel"
    torch.cuda.synchronize()
    check_bf16(_host(y), tr.forward(xf), np.linalg.norm(xf, axis=1), O.round_bf16, "auto")


@pytest.mark.parametrize("rows", [1, 16])
def test_back_to_back_calls_wait_for_the_previous_kernel(monkeypatch, rows):
    """A call may start its prologue before the previous kernel of the stream ends (programmatic
    dependent launch), but reads rows only after that kernel is done.  A chain in which every
    call rotates the previous call's output, with torch kernels in between, run on one stream
    with no synchronization, equals the same chain synchronized after every step, bit for bit."""
    monkeypatch.setenv("HARP_KERNEL", "cluster")
    gp, _ = _plan((8, 8, 8, 8, 2), 2205, 3205, True)
    _, x = _rows(gp.d, rows, 6, "bf16")

    def chain(sync):
        a = x.clone()
        for k in range(12):
            b = gp.apply(a, direction="forward" if k % 3 else "inverse")
            if sync:
                torch.cuda.synchronize()
            a = b.mul(1.0) if k % 4 == 1 else b        # a torch kernel between two calls
        torch.cuda.synchronize()
        return _host(a)

    ref = chain(True)
    assert H.last_kernel() == "harp_cluster_kernel"
    for _ in range(3):
        assert np.array_equal(chain(False), ref)
    gp.device_status()
