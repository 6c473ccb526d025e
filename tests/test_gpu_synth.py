"""The device generator equals the NumPy generator byte for byte."""
import numpy as np
import pytest
import torch

import synth
import synth.gpu as sg

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,lognormal", [(128, False), (512, True)])
def test_gpu_mxfp4_rows_equal_numpy(n, lognormal):
    rows = 1000
    c = torch.zeros((rows, n // 2), dtype=torch.uint8, device="cuda")
    s = torch.zeros((rows, n // 32), dtype=torch.uint8, device="cuda")
    sg.mxfp4_rows_into(c, s, 11, synth.T_MAIN_CODES, synth.T_MAIN_SCALES, 3, 2, 40, rows, n, lognormal)
    nk = synth.stream_key(11, synth.T_ROWNORM, 3, 0) if lognormal else None
    hc, hs = synth.mxfp4_rows(11, synth.T_MAIN_CODES, synth.T_MAIN_SCALES, 3, 2, 40, rows, n, nk)
    assert np.array_equal(c.cpu().numpy(), hc) and np.array_equal(s.cpu().numpy(), hs)


def test_gpu_e4m3_and_normal_equal_numpy():
    w = torch.zeros((300, 512), dtype=torch.uint8, device="cuda")
    sg.e4m3_rows_into(w, 5, synth.T_WIN, 1, 2, 7, 300)
    assert np.array_equal(w.cpu().numpy(), synth.e4m3_rows(5, synth.T_WIN, 1, 2, 7, 300))
    x = torch.zeros(100000, dtype=torch.bfloat16, device="cuda")
    sg.normal_bf16_into(x, 5, synth.T_RAW, 0, 0)
    assert np.array_equal(x.view(torch.int16).cpu().numpy().view(np.uint16), synth.normal_bf16(5, synth.T_RAW, 0, 0, 100000))
