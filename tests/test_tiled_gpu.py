"""GPU parity of the general tiled row kernel (forced with HARP_KERNEL=tiled) against
the float64 oracle: every workload schedule in both directions, schedules that use
each radix 2..8 (so every radix-set instantiation runs), ragged tiles, padded
leading dimensions, in-place calls; and its fallback rules."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from structured_rotations_b200 import harp as HB
from tests._parity import check_bf16, check_f32
from tests.test_parity_gpu import plans, to_dev, to_host, decode, check, run

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture
def tiled(monkeypatch):
    monkeypatch.setenv("HARP_KERNEL", "tiled")
    yield
    assert H.last_kernel() == "harp_tiled_kernel"


@pytest.mark.parametrize("name,direction", [
    ("d64", "forward"), ("d64", "inverse"), ("d64_hadamard", "forward"),
    ("d4096", "forward"), ("d4096", "inverse"), ("d5120", "forward"), ("d5120", "inverse"),
    ("d8192_int8", "forward"), ("d8192_int8", "inverse")])
@pytest.mark.parametrize("rows", [1, 5, 37, 300])
def test_workloads_full_compare(tiled, name, direction, rows):
    gp, tr = plans(name)
    enc = W.draw_encoded(W.get(name), 0, rows)
    out = run(gp, enc, direction)
    check(out, tr.apply(decode(enc), direction), decode(enc), f"tiled {name} {direction} rows={rows}")


def _plan_pair(schedule, seed):
    d = int(np.prod(schedule))
    theta = W.draw_theta(O.theta_count(schedule), 0.05, seed)
    gp = H.Plan(d, schedule, theta=theta, sign_seed=seed + 1)
    gp.materialize()
    return gp, O.Transform(O.make_plan(d, schedule, theta, sign_seed=seed + 1))


OTHER_SCHEDULES = [(5, 2, 8), (7, 8), (8, 5), (4, 4, 4), (3, 8), (6, 4), (2, 2, 2, 2),
                   (8, 7, 2), (2, 8, 8), (8, 8, 2, 3)]


@pytest.mark.parametrize("schedule", OTHER_SCHEDULES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_other_radices(tiled, schedule, dtype):
    gp, tr = _plan_pair(schedule, 900 + sum(schedule))
    d = int(np.prod(schedule))
    rng = np.random.default_rng(d)
    # enough elements that the share of near-zero outputs held to the fp32 bound
    # (rather than one bf16 step) is a meaningful statistic
    x = rng.standard_normal((max(53, 65536 // d), d))
    enc = W.encode_bf16(x) if dtype == "bf16" else x.astype(np.float32)
    xf = decode(enc)
    for direction in ("forward", "inverse"):
        out = run(gp, enc, direction)
        check(out, tr.apply(xf, direction), xf, f"tiled {schedule} {dtype} {direction}")


@pytest.mark.parametrize("name", ["d64", "d5120", "d8192_int8"])
def test_same_bits_as_the_simple_kernel(monkeypatch, name):
    """Both kernels sum each output as fma(B[k][l], x_l, acc) over l = 0..b-1 from 0, so
    their fp32 results agree bit for bit."""
    gp, _ = plans(name)
    enc = W.draw_encoded(W.get(name), 0, 41)
    outs = {}
    for kernel in ("tiled", "simple"):
        monkeypatch.setenv("HARP_KERNEL", kernel)
        for direction in ("forward", "inverse"):
            x = to_dev(enc)
            if x.dtype == torch.bfloat16:
                x = x.float()
            outs[kernel, direction] = to_host(gp.apply(x, direction=direction))
    for direction in ("forward", "inverse"):
        np.testing.assert_array_equal(outs["tiled", direction], outs["simple", direction])


@pytest.mark.parametrize("name", ["d5120", "d8192_int8", "d64"])
def test_in_place(tiled, name):
    gp, tr = plans(name)
    enc = W.draw_encoded(W.get(name), 0, 23)
    x = to_dev(enc)
    gp.apply(x, x, direction="inverse")
    torch.cuda.synchronize()
    check(to_host(x), tr.inverse(decode(enc)), decode(enc), f"tiled {name} in place")


@pytest.mark.parametrize("name,pad", [("d5120", 8), ("d8192_int8", 64), ("d64", 4)])
def test_padded_rows_and_guard_bands(tiled, name, pad):
    gp, tr = plans(name)
    w = W.get(name)
    rows, d = 29, w.d
    ld = d + pad
    enc = W.draw_encoded(w, 0, rows)
    canary = 0x7FC1 if enc.dtype == np.uint16 else np.float32(-123.25)
    buf_x = np.full(rows * ld + 64, canary, dtype=enc.dtype)
    buf_x[:rows * ld].reshape(rows, ld)[:, :d] = enc
    buf_y = np.full(rows * ld + 64, canary, dtype=enc.dtype)
    tx, ty = to_dev(buf_x), to_dev(buf_y)
    gp.apply(tx[:rows * ld].view(rows, ld)[:, :d], ty[:rows * ld].view(rows, ld)[:, :d])
    torch.cuda.synchronize()
    got = to_host(ty)
    body = got[:rows * ld].reshape(rows, ld)
    check(np.ascontiguousarray(body[:, :d]), tr.forward(decode(enc)), decode(enc), f"tiled {name} ld={ld}")
    assert np.all(body[:, d:] == canary) and np.all(got[rows * ld:] == canary)
    np.testing.assert_array_equal(to_host(tx), buf_x)


def test_shapes_outside_the_tiled_kernel_fall_back(monkeypatch):
    gp, tr = _plan_pair((3, 3), 77)            # d = 9 is not a multiple of 8
    x = np.random.default_rng(1).standard_normal((40, 9)).astype(np.float32)
    monkeypatch.delenv("HARP_KERNEL", raising=False)
    out = run(gp, x, "forward")
    assert H.last_kernel() == "apply_simple_kernel"
    check(out, tr.forward(x.astype(np.float64)), x.astype(np.float64), "d=9 fallback")
    monkeypatch.setenv("HARP_KERNEL", "tiled")
    with pytest.raises(HB.HarpError) as e:
        gp.apply(to_dev(x))
    assert e.value.status == HB.HARP_ERR_UNSUPPORTED


def test_default_dispatch_takes_the_tiled_kernel_for_d5120_and_c5(monkeypatch):
    """Batches of many rows (small ones take the cluster kernel, tests/test_cluster_gpu.py)."""
    monkeypatch.delenv("HARP_KERNEL", raising=False)
    for name, direction in (("d5120", "forward"), ("d8192_int8", "inverse"), ("d4096", "inverse")):
        gp, _ = plans(name)
        run(gp, W.draw_encoded(W.get(name), 0, 1024), direction)
        assert H.last_kernel() == "harp_tiled_kernel", name
        gp.device_status()


@pytest.mark.parametrize("name", ["d5120", "d8192_int8"])
@pytest.mark.parametrize("direction", ["forward", "inverse"])
def test_slab_mode_matches_whole_rows(monkeypatch, name, direction):
    """Slab mode (HARP_TILED_SLAB=1): schedules ending in radix 2 at large d run as CTA pairs
    that each hold half of every row (the last stage exchanged through distributed shared
    memory); the result is the same, bit for bit, as whole rows in one CTA, and matches the
    oracle."""
    gp, tr = plans(name)
    enc = W.draw_encoded(W.get(name), 0, 301)
    monkeypatch.setenv("HARP_KERNEL", "tiled")
    monkeypatch.setenv("HARP_TILED_SLAB", "1")
    a = run(gp, enc, direction)
    monkeypatch.setenv("HARP_TILED_SLAB", "0")
    b = run(gp, enc, direction)
    np.testing.assert_array_equal(a, b)
    check(a, tr.apply(decode(enc), direction), decode(enc), f"slab {name} {direction}")
    gp.device_status()


@pytest.mark.parametrize("schedule", [(8, 8, 8, 8, 8), (8, 8, 8, 8, 7)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_largest_dimensions_single_row_subtiles(tiled, schedule, dtype):
    """d = 32768 (the largest the library takes) and 28672: fp32 tiles of 4 rows no longer
    fit in shared memory, so the tiled kernel holds one row per sub-tile."""
    gp, tr = _plan_pair(schedule, 500 + schedule[-1])
    d = int(np.prod(schedule))
    x = np.random.default_rng(d).standard_normal((6, d))
    enc = W.encode_bf16(x) if dtype == "bf16" else x.astype(np.float32)
    xf = decode(enc)
    for direction in ("forward", "inverse"):
        out = run(gp, enc, direction)
        check(out, tr.apply(xf, direction), xf, f"d={d} {dtype} {direction}")


@pytest.mark.parametrize("schedule", [(2,), (3,), (2, 2), (16,), (16, 3), (12, 5)])
def test_degenerate_and_large_radix_schedules(monkeypatch, schedule):
    """One stage, d = 2, radices above 8: the simple kernel takes them."""
    monkeypatch.delenv("HARP_KERNEL", raising=False)
    gp, tr = _plan_pair(schedule, 600 + sum(schedule))
    d = int(np.prod(schedule))
    x = np.random.default_rng(d + 1).standard_normal((257, d)).astype(np.float32)
    xf = x.astype(np.float64)
    for direction in ("forward", "inverse"):
        out = run(gp, x, direction)
        check(out, tr.apply(xf, direction), xf, f"{schedule} {direction}")
    assert H.last_kernel() == "apply_simple_kernel"


@pytest.mark.parametrize("schedule", [(8, 8, 8, 8, 2), (2, 8, 8, 8, 8, 2), (8, 4, 8, 8, 4)])
@pytest.mark.parametrize("direction", ["forward", "inverse"])
def test_stages_fused_into_fill_and_drain_match_separate_passes(monkeypatch, schedule, direction):
    """At d = 8192 (a tile is one 4-row sub-tile) the radix-8 stride-1 stage and the radix-2
    stride-d/2 stage run inside the tile's fill and drain; the result is the same, bit for bit,
    as with every stage a pass of its own (HARP_TILED_NOFUSE=1), and matches the oracle."""
    d = int(np.prod(schedule))
    theta = W.draw_theta(O.theta_count(schedule), 0.2236, 77)
    gp = H.Plan(d, schedule, theta=theta, sign_seed=78).materialize()
    tr = O.Transform(O.make_plan(d, schedule, theta, sign_seed=78))
    rng = np.random.default_rng(d + len(schedule))
    enc = W.encode_bf16(rng.standard_normal((203, d)))
    monkeypatch.setenv("HARP_KERNEL", "tiled")
    a = run(gp, enc, direction)
    monkeypatch.setenv("HARP_TILED_NOFUSE", "1")
    b = run(gp, enc, direction)
    assert np.array_equal(a, b)
    xf = W.decode_bf16(enc)
    check(a, tr.apply(xf, direction), xf, f"fused {schedule} {direction}")
    gp.device_status()
