"""GPU parity of the fit's evaluation terms (HARP technical summary §2.3 Optimization
Objective: L_fit = L_diag + lambda_bd R_bd(Theta_V), described in words; the readings are
the oracle's): the rotated Hessian proxy H' = T_V^T H T_V (the two-sided rotation with U = V),
the off-block energy behind R_bd (harp_off_block_energy) and the diagonal-weighted
quantization error L_diag (harp_l_diag), against the float64 oracle on seeded inputs.

Tolerances.  The two reduction kernels square and sum in double and take the quantizer's
decisions in the same double operations as its definition, so on the same input they agree
with the oracle to summation order (relative 1e-12).  Through the rotations, H' and W' carry
the fp32 transform's error (about 1e-6 of a row's norm per element); both terms are smooth
in their input (the squared quantization error is continuous across a rounding tie), so a
relative 1e-6 perturbation moves them by a few 1e-6: held to 2e-5 (R_bd) and 1e-4 (L_diag).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from structured_rotations_b200 import harp as HB

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _plans(schedule, theta_seed, sign_seed, sigma=0.2236):
    d = int(np.prod(schedule))
    theta = W.draw_theta(O.theta_count(schedule), sigma, theta_seed)
    gp = H.Plan(d, schedule, theta=theta, sign_seed=sign_seed).materialize()
    return gp, O.make_plan(d, schedule, theta, sign_seed=sign_seed)


def _dev(a, dtype):
    if dtype == "bf16":
        return torch.from_numpy(W.encode_bf16(a).view(np.int16)).view(torch.bfloat16).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def _vals(a, dtype):
    """float64 values of `a` as stored in dtype."""
    return W.decode_bf16(W.encode_bf16(a)) if dtype == "bf16" else np.asarray(a, np.float32).astype(np.float64)


@pytest.mark.parametrize("n,q,dtype,pad", [(512, 128, "f32", 0), (512, 8, "bf16", 0), (640, 64, "f32", 3),
                                           (4096, 128, "f32", 0), (96, 32, "bf16", 1), (60, 6, "f32", 0)])
def test_off_block_energy_matches_its_definition(n, q, dtype, pad):
    """The same stored values in both: a seeded matrix with a few heavy entries, padded
    rows (pad > 0 turns the 16-byte vector path off)."""
    rng = np.random.default_rng([n, q, pad])
    a = rng.standard_normal((n, n)) * np.exp(rng.standard_normal((n, n)))
    vals = _vals(a, dtype)
    full = np.zeros((n, n + pad))
    full[:, :n] = vals
    t = _dev(full, dtype)[:, :n]
    got = H.off_block_energy(t, q).cpu().numpy()
    assert got[1] == pytest.approx(float(np.sum(vals * vals)), rel=1e-12)
    assert got[0] / got[1] == pytest.approx(O.off_block_energy(vals, q), rel=1e-12)


def test_off_block_energy_closed_forms():
    """Block-diagonal input: no off-block energy; a constant matrix: 1 - q / n."""
    n, q = 256, 32
    blocks = np.zeros((n, n))
    for b in range(n // q):
        blocks[b * q:(b + 1) * q, b * q:(b + 1) * q] = 1.5
    assert H.off_block_energy(_dev(blocks, "f32"), q).cpu().numpy()[0] == 0.0
    e = H.off_block_energy(_dev(np.ones((n, n)), "f32"), q).cpu().numpy()
    assert e[0] / e[1] == pytest.approx(1 - q / n, rel=1e-15)


@pytest.mark.parametrize("rows,cols,qblock,dtype", [(64, 512, 32, "f32"), (33, 1024, 128, "bf16"),
                                                    (8, 256, 256, "f32"), (17, 640, 64, "bf16")])
def test_l_diag_matches_its_definition(rows, cols, qblock, dtype):
    """The same stored W' and H' in both, with hand-placed exact ties (w / s = k + 1/2, which
    round half to even), an all-zero block and a block whose maximum is negative."""
    rng = np.random.default_rng([rows, cols, qblock])
    w = 0.02 * rng.standard_normal((rows, cols))
    w[0, :qblock] = 0.0                                          # zero block: exact, no error
    tie = np.zeros(qblock)
    tie[0] = 127.0
    tie[1:6] = [0.5, 1.5, -2.5, 3.5, 126.5]                      # scale 1: every one a tie
    w[1, :qblock] = tie / 64.0                                   # exact in bf16 and fp32
    w[2, qblock:2 * qblock] = -np.abs(w[2, qblock:2 * qblock])
    wv = _vals(w, dtype)
    h = W.draw_hessian(cols, 5)
    got = H.l_diag(_dev(wv, dtype), _dev(h, "f32"), qblock).cpu().numpy()[0]
    want = O.l_diag(wv, h, qblock)
    assert want > 0
    assert got == pytest.approx(want, rel=1e-12)


def test_l_diag_of_exactly_representable_weights_is_zero():
    codes = np.random.default_rng(1).integers(-127, 128, size=(16, 256)).astype(np.float64)
    codes[:, ::32] = 127.0                                       # every block's maximum is 127
    w = codes / 256.0                                            # scale 1/256: exact
    h = W.draw_hessian(256, 2)
    assert H.l_diag(_dev(w, "f32"), _dev(h, "f32"), 32).cpu().numpy()[0] == 0.0


def test_fit_term_argument_errors():
    t = torch.zeros(64, 64, device=DEV)
    out = torch.zeros(2, dtype=torch.float64, device=DEV)
    L = H.lib()
    s = torch.cuda.current_stream().cuda_stream
    assert L.harp_off_block_energy(t.data_ptr(), 64, 64, HB.HARP_F32, 48, out.data_ptr(), s) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_off_block_energy(t.data_ptr(), 64, 63, HB.HARP_F32, 8, out.data_ptr(), s) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_off_block_energy(t.data_ptr(), 64, 64, 9, 8, out.data_ptr(), s) == HB.HARP_ERR_UNSUPPORTED
    assert L.harp_off_block_energy(t.data_ptr(), 64, 64, HB.HARP_F32, 8, t.data_ptr(), s) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_l_diag(t.data_ptr(), 64, 64, 64, HB.HARP_F32, t.data_ptr(), 64, 48, out.data_ptr(), s) \
        == HB.HARP_ERR_INVALID_ARG
    assert L.harp_l_diag(t.data_ptr(), 64, 64, 64, HB.HARP_F32, t.data_ptr(), 64, 128, out.data_ptr(), s) \
        == HB.HARP_ERR_INVALID_ARG                               # 128 does not divide 64
    assert L.harp_l_diag(t.data_ptr(), 64, 64, 64, HB.HARP_F32, t.data_ptr(), 64, 32, t.data_ptr(), s) \
        == HB.HARP_ERR_INVALID_ARG                               # out inside w
    assert L.harp_l_diag(None, 0, 64, 64, HB.HARP_F32, t.data_ptr(), 64, 32, out.data_ptr(), s) == HB.HARP_OK
    torch.cuda.synchronize()
    assert out.cpu().numpy()[0] == 0.0


@pytest.mark.parametrize("schedule,q", [((8, 8, 8, 8), 128), ((8, 8, 8, 5, 2), 128), ((8, 8, 2), 16)])
def test_r_bd_through_the_rotated_hessian(schedule, q):
    """R_bd(Theta_V) on a seeded SPD Hessian proxy: H' = T_V^T H T_V by the two-sided
    rotation (fp32 in and out), then the off-block energy, against the oracle's r_bd."""
    gp, op = _plans(schedule, 2101, 3101)
    n = gp.d
    h = W.draw_hessian(n, 7)
    hp = H.apply_two_sided(gp, gp, _dev(h, "f32"))
    e = H.off_block_energy(hp, q).cpu().numpy()
    ref_rot = O.rotated_hessian(op, h)
    got_rot = hp.cpu().numpy().astype(np.float64)
    assert np.abs(got_rot - ref_rot).max() <= 1e-5 * np.abs(ref_rot).max()
    want = O.off_block_energy(ref_rot, q)                       # = O.r_bd(op, h, q), not recomputed
    assert 0.0 < want < 1.0
    assert e[0] / e[1] == pytest.approx(want, rel=2e-5)
    # rotation keeps the total energy (the oracle's pin, here on the GPU path)
    assert e[1] == pytest.approx(float(np.sum(h * h)), rel=1e-5)


@pytest.mark.parametrize("u_sched,v_sched,qblock", [((8, 8, 7), (8, 8, 2), 32), ((8, 8, 8, 8), (8, 8, 8, 5, 2), 128)])
def test_l_diag_through_the_rotations(u_sched, v_sched, qblock):
    """L_diag on W' = T_U^T W T_V (fp32 two-sided rotation of a seeded weight with outlier
    columns) weighted by diag(H'), H' = T_V^T H T_V, against the oracle's chain."""
    pu, opu = _plans(u_sched, 2102, 3102)
    pv, opv = _plans(v_sched, 2103, 3103)
    n_out, n_in = pu.d, pv.d
    rng = np.random.default_rng([n_out, n_in])
    w = 0.02 * rng.standard_normal((n_out, n_in))
    w[:, rng.choice(n_in, 4, replace=False)] *= 30.0
    w = w.astype(np.float32).astype(np.float64)
    h = W.draw_hessian(n_in, 9)
    wp = H.apply_two_sided(pu, pv, _dev(w, "f32"))
    hp = H.apply_two_sided(pv, pv, _dev(h, "f32"))
    got = H.l_diag(wp, hp, qblock).cpu().numpy()[0]
    want = O.l_diag(O.two_sided(opu, opv, w), O.rotated_hessian(opv, h), qblock)
    assert got == pytest.approx(want, rel=1e-4)
