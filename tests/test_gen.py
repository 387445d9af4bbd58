"""Seeded input generators: shapes, determinism and code ranges."""

import torch

from gen import LINEAR_CONFIGS, LinearSpec, make_linear_case
from gen.workloads import _quant_mxfp4, _rne_e2m1_index


def test_c0_shapes_and_determinism():
    spec = LINEAR_CONFIGS["c0"]
    a, b = make_linear_case(spec), make_linear_case(spec)
    assert a["X"].shape == (64, 256) and a["X"].dtype == torch.bfloat16
    assert a["codes"].shape == (384, 128) and a["scales"].shape == (8, 384)
    assert a["Q"].shape == (3, 8, 32 * 31 // 2)
    for k in ("X", "codes", "scales", "Q"):
        assert torch.equal(a[k], b[k])
    nib = torch.stack([a["codes"] & 0xF, a["codes"] >> 4], -1)
    assert int((nib == 8).sum()) == 0          # symmetric range [-7, 7]
    s = a["scales"].float()
    assert float(s.min()) >= 0.0099 and float(s.max()) <= 0.0501


def test_fp8_and_mxfp4_shapes():
    sp = LinearSpec("t", M=8, K=128, splits=(64, 32), fmt="fp8", group=0, b=32, q_sigma=0.02, backward=True)
    c = make_linear_case(sp)
    assert c["codes"].shape == (96, 128) and c["scales"].shape == (96,) and c["dY"].shape == (8, 96)
    sp = sp.with_(fmt="mxfp4", group=32)
    c = make_linear_case(sp)
    assert c["codes"].shape == (96, 64) and c["scales"].shape == (4, 96) and c["scales"].dtype == torch.uint8


def test_e2m1_encoder_rounds_to_nearest_even():
    a = torch.tensor([0.0, 0.25, 0.26, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.1, 9.0])
    assert _rne_e2m1_index(a).tolist() == [0, 0, 1, 2, 2, 4, 4, 6, 6, 7, 7]
    codes, e8 = _quant_mxfp4(torch.randn(4, 64))
    assert codes.shape == (4, 32) and e8.shape == (2, 4)
