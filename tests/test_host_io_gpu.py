"""GPU parity of harp_apply_host (host buffers in and out, chunks on three streams):
bit for bit against the device call when every chunk takes the same kernel, against the
oracle across a ragged last chunk, in place, with padded rows, and from pageable memory."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from tests.test_parity_gpu import plans, to_dev, to_host, decode, check

pytestmark = pytest.mark.gpu


def _host(enc, pin=True):
    t = torch.from_numpy(enc.view(np.int16)).view(torch.bfloat16) if enc.dtype == np.uint16 \
        else torch.from_numpy(np.ascontiguousarray(enc))
    return t.pin_memory() if pin else t.clone()


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()


@pytest.mark.parametrize("direction", ["forward", "inverse"])
def test_host_chunks_equal_the_device_call(direction):
    gp, _ = plans("d5120")
    enc = W.draw_encoded(W.get("d5120"), 0, 9000)            # three 32 MiB chunks, the last ragged
    yh = gp.apply_host(_host(enc), direction=direction)
    yd = gp.apply(to_dev(enc), direction=direction)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_bits(yh), to_host(yd))


def test_host_d4096_with_a_small_last_chunk_matches_the_oracle():
    gp, tr = plans("d4096")
    enc = W.draw_encoded(W.get("d4096"), 0, 8200)            # chunks of 4096, 4096 and 8 rows
    out = _bits(gp.apply_host(_host(enc)))
    idx = np.unique(np.concatenate([W.sample_rows(8200, 300), np.arange(8190, 8200)]))
    x = decode(enc[idx])
    check(out[idx], tr.forward(x), x, "host d4096")


def test_host_in_place_padded_and_pageable():
    gp, tr = plans("d5120")
    w = W.get("d5120")
    rows, d, pad = 3100, w.d, 24
    enc = W.draw_encoded(w, 0, rows)
    buf = np.zeros((rows, d + pad), dtype=np.uint16)
    buf[:, :d] = enc
    buf[:, d:] = 0x7FC1
    for pin in (True, False):
        t = _host(buf, pin=pin)
        view = t[:, :d]
        gp.apply_host(view, view, direction="inverse")
        got = _bits(t)
        assert np.all(got[:, d:] == 0x7FC1)
        x = decode(enc)
        check(np.ascontiguousarray(got[:, :d]), tr.inverse(x), x, f"host in place pinned={pin}")
