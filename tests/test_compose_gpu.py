"""GPU parity of composite plans (harp_plan_compose: T = T_{k-1} ... T_0 applied in one pass
over the rows, the composition of independent rotations the RHT-composition results quoted
with the HARP pages call for): against the float64 oracle (Composed) for two and three
plans of every workload shape in both directions; bit for bit against applying the plans
one after another with fp32 intermediates on the tiled kernel (the composite runs the same
stages in the same order, only without the round trips); the fused quantizer and the
two-sided rotation on composites; and the calls that decline a composite."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from structured_rotations_b200 import harp as HB
from tests.test_parity_gpu import DEV, to_dev, to_host, decode, check

pytestmark = pytest.mark.gpu


def _pair(schedule, seed, sigma=0.05):
    d = int(np.prod(schedule))
    theta = W.draw_theta(O.theta_count(schedule), sigma, seed)
    gp = H.Plan(d, schedule, theta=theta, sign_seed=seed + 100).materialize()
    return gp, O.Transform(O.make_plan(d, schedule, theta.astype(np.float32).astype(np.float64),
                                       sign_seed=seed + 100))


CASES = {
    "d4096 x2": [(8, 8, 8, 8), (8, 8, 8, 8)],
    "d5120 x2": [(8, 8, 8, 5, 2), (2, 5, 8, 8, 8)],
    "d8192 x3": [(8, 8, 8, 8, 2), (2, 8, 8, 8, 8), (8, 8, 2, 8, 8)],
    "d64 x3": [(8, 8), (2, 2, 2, 2, 2, 2), (4, 2, 8)],
}


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("direction", ["forward", "inverse"])
@pytest.mark.parametrize("rows", [29, 700])
def test_composite_vs_oracle(case, direction, rows):
    pairs = [_pair(s, 31 + 7 * i) for i, s in enumerate(CASES[case])]
    comp = H.Plan.compose([p for p, _ in pairs])
    oc = O.Composed([t for _, t in pairs])
    d = comp.d
    x = W.encode_bf16(np.random.default_rng(d + rows).standard_normal((rows, d)))
    y = comp.apply(to_dev(x), direction=direction)
    torch.cuda.synchronize()
    check(to_host(y), oc.apply(decode(x), direction), decode(x), f"{case} {direction} rows={rows}")


@pytest.mark.parametrize("case", ["d4096 x2", "d5120 x2", "d8192 x3"])
@pytest.mark.parametrize("direction", ["forward", "inverse"])
def test_composite_equals_the_plans_in_turn_bit_for_bit(monkeypatch, case, direction):
    monkeypatch.setenv("HARP_KERNEL", "tiled")
    plans = [_pair(s, 51 + 3 * i)[0] for i, s in enumerate(CASES[case])]
    comp = H.Plan.compose(plans)
    d, rows = comp.d, 300
    x = to_dev(W.encode_bf16(np.random.default_rng(d).standard_normal((rows, d))))
    y = comp.apply(x, direction=direction)
    assert H.last_kernel() == "harp_tiled_kernel"
    order = plans if direction == "forward" else plans[::-1]
    z = torch.empty(rows, d, dtype=torch.float32, device=DEV)
    order[0].apply_ex(x, z, direction=direction)
    for p in order[1:]:
        z = p.apply(z, direction=direction)
    ref = z.to(torch.bfloat16)                  # round to nearest even, as the kernel's bf16 store
    torch.cuda.synchronize()
    assert torch.equal(y, ref)


def test_composite_quantizer_and_host_path():
    pairs = [_pair(s, 71 + i) for i, s in enumerate(CASES["d4096 x2"])]
    comp = H.Plan.compose([p for p, _ in pairs])
    oc = O.Composed([t for _, t in pairs])
    x = W.encode_bf16(np.random.default_rng(5).standard_normal((40, 4096)))
    q, s = comp.apply_quant(to_dev(x), 128)
    torch.cuda.synchronize()
    y = oc.forward(decode(x)).reshape(40, -1, 128)
    deq = q.cpu().numpy().astype(np.float64).reshape(40, -1, 128) * s.cpu().numpy()[..., None]
    tol = 0.5 * s.cpu().numpy()[..., None] * (1 + 1e-4) + 2e-6 * np.linalg.norm(decode(x), axis=1)[:, None, None]
    assert (np.abs(deq - y) <= tol).all()
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = comp.apply_host(xh)
    check(yh.view(torch.int16).numpy().view(np.uint16), oc.forward(decode(x)), decode(x), "host path")


def test_composite_as_a_side_of_the_two_sided_rotation():
    pu, tu = _pair((8, 8, 4), 81)
    v1, t1 = _pair((8, 8, 2), 82)
    v2, t2 = _pair((2, 8, 8), 83)
    pv = H.Plan.compose([v1, v2])
    w = W.encode_bf16(np.random.default_rng(9).standard_normal((pu.d, pv.d)) * 0.02)
    out = H.apply_two_sided(pu, pv, to_dev(w))
    torch.cuda.synchronize()
    wf = decode(w)
    want = tu.inverse(O.Composed([t1, t2]).inverse(wf).T).T
    tau = np.full(pu.d, np.max(np.linalg.norm(wf, axis=1)))
    from tests._parity import check_bf16
    check_bf16(to_host(out), want, tau, O.round_bf16, "two-sided with a composite V")


def test_composite_declines_and_limits():
    a, _ = _pair((8, 8, 8, 8), 91)
    b, _ = _pair((8, 8, 8, 8), 92)
    comp = H.Plan.compose([a, b])
    a.close()                                   # the composite keeps its own copy of the blocks
    x = torch.zeros(4, 4096, dtype=torch.float32, device=DEV)
    with pytest.raises(HB.HarpError) as e:
        comp.grad_theta(x, x)
    assert e.value.status == HB.HARP_ERR_UNSUPPORTED
    with pytest.raises(HB.HarpError) as e:
        comp.apply_columns(torch.zeros(4096, 8, device=DEV))
    assert e.value.status == HB.HARP_ERR_UNSUPPORTED
    five = [_pair((8, 8, 8, 8), 93 + i)[0] for i in range(5)]   # 20 stages > 16
    with pytest.raises(HB.HarpError) as e:
        H.Plan.compose(five)
    assert e.value.status == HB.HARP_ERR_SCHEDULE
    other = _pair((8, 8, 8), 99)[0]
    with pytest.raises(HB.HarpError) as e:
        H.Plan.compose([b, other])
    assert e.value.status == HB.HARP_ERR_INVALID_ARG
    y = comp.apply(to_dev(W.encode_bf16(np.ones((2, 4096)))))
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
