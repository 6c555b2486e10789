"""GPU parity of the fused quantizer (harp_apply_quant: the row transform with a blockwise
int8 round-to-nearest quantizer on its output, HARP technical summary §2.4: a drop-in
preprocessing step in front of a blockwise quantizer).

Against the float64 oracle (y = T x, then quantize_blocks): a scale differs from the
oracle's by at most what the fp32 row transform may move the block maximum (2e-6 |x| of
the row, the row transform's parity bound) over 127, plus half an fp32 ulp; a code equals
the oracle's wherever the oracle's y / s lies farther than the fp32 error band from a
rounding tie (k + 1/2), and differs by at most one inside that band.  Against the kernel's
own fp32 rows (the tiled kernel with fp32 output, the same stage arithmetic) the epilogue
is checked bit for bit, both sides deciding in fp32 (the kernel forms y * (127 / a), one
more fp32 rounding than y / s, which the oracle band's 2^-23 |y / s| term covers)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from structured_rotations_b200 import harp as HB
from tests.test_parity_gpu import DEV, plans, to_dev, decode

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


def _check(q_gpu, s_gpu, y64, x64, qblock, what):
    rows, d = y64.shape
    q_o, s_o = O.quantize_blocks(y64, qblock)
    tau = 2e-6 * np.linalg.norm(x64, axis=1)[:, None]
    ds = np.abs(s_gpu.astype(np.float64) - s_o)
    s_bound = tau / 127 + 2 * U * s_o
    assert np.all(ds <= s_bound), f"{what}: scale off by {np.max(ds - s_bound):.3e} beyond the bound"
    t = y64.reshape(rows, -1, qblock) / np.where(s_o > 0, s_o, 1.0)[..., None]
    band = 2 * ((tau[..., None] + np.abs(t) * s_bound[..., None]) / np.where(s_o > 0, s_o, 1.0)[..., None]
                + np.abs(t) * 2 * U)
    near_tie = np.abs(np.abs(t - np.floor(t)) - 0.5) <= band
    dq = np.abs(q_gpu.reshape(rows, -1, qblock).astype(int) - q_o.reshape(rows, -1, qblock).astype(int))
    assert np.all(dq[~near_tie] == 0), f"{what}: {int(np.sum(dq[~near_tie] != 0))} codes differ away from ties"
    assert np.all(dq[near_tie] <= 1), f"{what}: a code near a tie differs by more than one"


@pytest.mark.parametrize("name", ["d4096", "d5120", "d8192_int8"])
@pytest.mark.parametrize("direction", ["forward", "inverse"])
@pytest.mark.parametrize("rows,qblock", [(37, 32), (37, 256), (700, 128)])
def test_quant_vs_oracle(name, direction, rows, qblock):
    # 37 rows take one-row sub-tiles, 700 rows (more than 4 per SM) 4-row sub-tiles
    gp, tr = plans(name)
    xe = W.draw_encoded(W.get(name), 0, rows)
    q, s = gp.apply_quant(to_dev(xe), qblock, direction)
    torch.cuda.synchronize()
    # d = 4096 forward takes the specialized kernel's quantizing variant
    fast = name == "d4096" and direction == "forward"
    assert H.last_kernel() == ("harp_fast_d4096_fwd_kernel" if fast else "harp_tiled_kernel")
    x64 = decode(xe)
    _check(q.cpu().numpy(), s.cpu().numpy(), tr.apply(x64, direction), x64, qblock, f"{name} {direction} {rows}")


@pytest.mark.parametrize("qblock", [32, 64, 128, 256])
@pytest.mark.parametrize("rows", [32, 45, 1000])
def test_fast_kernel_quantizer_vs_oracle(monkeypatch, rows, qblock):
    """d = 4096 (8,8,8,8) forward on the specialized kernel: each CTA of a pair holds half of
    every quantizer block of 64 coordinates or more (its 32 pencils), so the block maxima are
    exchanged between the two; a zero row (scale 0, codes 0), a one-hot row and ragged last
    tiles included."""
    monkeypatch.setenv("HARP_KERNEL", "fast")
    gp, tr = plans("d4096")
    xe = W.draw_encoded(W.get("d4096"), 0, rows)
    xe[3] = 0
    xe[7] = 0
    xe[7, 1234] = W.encode_bf16(np.array([5.0]))[0]
    q, s = gp.apply_quant(to_dev(xe), qblock)
    torch.cuda.synchronize()
    assert H.last_kernel() == "harp_fast_d4096_fwd_kernel"
    x64 = decode(xe)
    qh, sh = q.cpu().numpy(), s.cpu().numpy()
    _check(qh, sh, tr.forward(x64), x64, qblock, f"fast rows={rows} qblock={qblock}")
    assert np.all(qh[3] == 0) and np.all(sh[3] == 0)
    gp.device_status()


def test_fast_kernel_quantizer_padded_outputs(monkeypatch):
    """Padded code and scale rows: the kernel writes exactly rows x 4096 codes and
    rows x 4096 / qblock scales."""
    monkeypatch.setenv("HARP_KERNEL", "fast")
    gp, tr = plans("d4096")
    rows = 77
    xe = W.draw_encoded(W.get("d4096"), 0, rows)
    qp = torch.full((rows, 4096 + 48), 5, dtype=torch.int8, device=DEV)
    sp = torch.full((rows, 40), -1.0, device=DEV)
    gp.apply_quant(to_dev(xe), 128, q=qp[:, :4096], scales=sp[:, :32])
    torch.cuda.synchronize()
    assert H.last_kernel() == "harp_fast_d4096_fwd_kernel"
    x64 = decode(xe)
    _check(qp[:, :4096].cpu().numpy(), sp[:, :32].cpu().numpy(), tr.forward(x64), x64, 128, "fast padded")
    assert torch.all(qp[:, 4096:] == 5) and torch.all(sp[:, 32:] == -1.0)
    gp.device_status()


def test_quant_full_size_on_sampled_rows():
    """C2 in the bench's launch configuration (65,536 rows, qblock 128), sampled rows."""
    gp, tr = plans("d4096")
    w = W.get("d4096")
    xe = W.draw_encoded(w, 0, w.rows)
    q, s = gp.apply_quant(to_dev(xe), 128)
    torch.cuda.synchronize()
    idx = W.sample_rows(w.rows, 48)
    x64 = decode(xe[idx])
    _check(q.cpu().numpy()[idx], s.cpu().numpy()[idx], tr.forward(x64), x64, 128, "C2 sampled rows")


@pytest.mark.parametrize("rows", [5, 700])
@pytest.mark.parametrize("qblock", [32, 64, 128, 256])
def test_epilogue_matches_the_kernels_own_fp32_rows_bit_for_bit(monkeypatch, rows, qblock):
    monkeypatch.setenv("HARP_KERNEL", "tiled")
    gp, _ = plans("d5120")
    x = to_dev(W.draw_encoded(W.get("d5120"), 0, rows))
    y32 = torch.empty(rows, gp.d, dtype=torch.float32, device=DEV)
    gp.apply_ex(x, y32)
    q, s = gp.apply_quant(x, qblock)
    torch.cuda.synchronize()
    y = y32.cpu().numpy().reshape(rows, -1, qblock)
    # the kernel's fp32 steps: s = a / 127 and q = rne(y * (127 / a)), each operation rounded
    # to nearest in fp32 (numpy float32 arithmetic rounds the same way)
    amax = np.max(np.abs(y), axis=2)
    s_ref = (amax / np.float32(127)).astype(np.float32)
    inv = np.where(amax > 0, np.float32(127) / np.where(amax > 0, amax, np.float32(1)), np.float32(0))
    q_ref = np.rint((y * inv[..., None]).astype(np.float32)).clip(-127, 127).astype(np.int8)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref.reshape(rows, -1))


def test_quant_padded_rows_and_empty_batch():
    gp, tr = plans("d4096")
    xe = W.draw_encoded(W.get("d4096"), 0, 9)
    xp = torch.zeros(9, 4096 + 64, dtype=torch.bfloat16, device=DEV)
    xp[:, :4096] = to_dev(xe)
    qp = torch.full((9, 4096 + 32), 5, dtype=torch.int8, device=DEV)
    sp = torch.full((9, 40), -1.0, device=DEV)
    gp.apply_quant(xp[:, :4096], 128, q=qp[:, :4096], scales=sp[:, :32])
    torch.cuda.synchronize()
    x64 = decode(xe)
    _check(qp[:, :4096].cpu().numpy(), sp[:, :32].cpu().numpy(), tr.forward(x64), x64, 128, "padded")
    assert torch.all(qp[:, 4096:] == 5) and torch.all(sp[:, 32:] == -1.0)
    gp.apply_quant(torch.empty(0, 4096, dtype=torch.bfloat16, device=DEV), 128)


def test_quant_argument_errors():
    gp, _ = plans("d4096")
    x = torch.zeros(4, 4096, dtype=torch.bfloat16, device=DEV)
    for qb in (48, 512):
        with pytest.raises(HB.HarpError) as e:
            gp.apply_quant(x, qb)
        assert e.value.status == HB.HARP_ERR_INVALID_ARG
    odd = H.Plan(96, (8, 4, 3), sign_seed=2).materialize()
    with pytest.raises(HB.HarpError) as e:                          # 64 does not divide 96
        odd.apply_quant(torch.zeros(2, 96, dtype=torch.bfloat16, device=DEV), 64)
    assert e.value.status == HB.HARP_ERR_INVALID_ARG
    with pytest.raises(HB.HarpError) as e:                          # fp32 rows
        gp.apply_quant(torch.zeros(4, 4096, device=DEV), 128)
    assert e.value.status == HB.HARP_ERR_UNSUPPORTED
    q = torch.empty(4, 4096 + 8, dtype=torch.int8, device=DEV)      # code rows not 16-byte aligned
    with pytest.raises(HB.HarpError) as e:
        gp.apply_quant(x, 128, q=q[:, :4096])
    assert e.value.status == HB.HARP_ERR_UNSUPPORTED
