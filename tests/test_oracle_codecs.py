"""Pins for oracle.codecs: element decoders, bf16 rounding, group-wise dequant.

Every expected value here comes from outside the oracle: torch's own fp8/e8m0
decoders and fp32->bf16 conversion, int8 sign extension, the OCP spec tables
stored under tests/golden/, or torch CPU arithmetic on the same codes.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import codecs
from gen import LinearSpec, make_linear_case
from npcase import raw

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_e4m3_all_codes_match_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().double().numpy()
    got = codecs.E4M3_TABLE
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


def test_e4m3_named_codes_from_ocp_spec():
    g = _golden("ocp_fp8_e4m3.json")
    for code, val in g["named_codes"].items():
        assert codecs.E4M3_TABLE[int(code, 16)] == val
    for code in g["nan_codes"]:
        assert np.isnan(codecs.E4M3_TABLE[int(code, 16)])
    assert np.nanmax(codecs.E4M3_TABLE) == 448.0


def test_e2m1_table_from_ocp_spec():
    g = _golden("ocp_fp4_e2m1.json")
    mags = np.array(g["codes_0_to_7_magnitude"])
    assert np.array_equal(codecs.E2M1_TABLE[:8], mags)
    assert np.array_equal(codecs.E2M1_TABLE[8:], -mags)


def test_e2m1_agrees_with_e4m3_on_shared_values():
    # e2m1 (s, e2, m1), bias 1, is the e4m3 code (s, e2 + 6, m1 << 2) for e2 >= 1;
    # the subnormal 0.5 is e4m3 (s, 6, 0).  The e4m3 decoder is pinned to torch.
    for c in range(16):
        s, e2, m1 = c >> 3, (c >> 1) & 3, c & 1
        if e2 == 0 and m1 == 0:
            c8 = s << 7
        elif e2 == 0:
            c8 = (s << 7) | (6 << 3)
        else:
            c8 = (s << 7) | ((e2 + 6) << 3) | (m1 << 2)
        assert codecs.E2M1_TABLE[c] == codecs.E4M3_TABLE[c8]


def test_e8m0_all_codes_match_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).float().double().numpy()
    got = codecs.E8M0_TABLE
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


def test_int4_matches_int8_sign_extension():
    for n in range(16):
        assert codecs.INT4_TABLE[n] == int(np.int8(np.uint8(n << 4).view(np.int8)) >> 4)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 2**32, size=200000, dtype=np.uint64).astype(np.uint32)
    # exact ties (low half 0x8000) with even and odd kept halves, and near-overflow values
    ties = (rng.integers(0, 2**16, size=20000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    special = np.array([0x7F7FFFFF, 0x7F7F8000, 0xFF7FFFFF, 0x00000001, 0x80008000, 0x3F808000, 0x3F818000,
                        0x7F800000, 0xFF800000, 0x7FC00000, 0x7F800001], dtype=np.uint32)
    x = np.concatenate([bits, ties, special]).view(np.float32)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = codecs.f32_to_bf16_bits(x)
    nan = np.isnan(x)
    assert np.array_equal(ref[~nan], got[~nan])
    assert np.all(np.isnan(codecs.bf16_bits_to_f64(got[nan])))


def test_bf16_to_f64_roundtrip():
    t = torch.randn(10000).to(torch.bfloat16)
    got = codecs.bf16_bits_to_f64(raw(t))
    assert np.array_equal(got, t.double().numpy())


def _torch_unpack_int4(codes: torch.Tensor) -> torch.Tensor:
    lo = (codes & 0xF).to(torch.int16)
    hi = (codes >> 4).to(torch.int16)
    q = torch.stack([lo, hi], dim=-1).flatten(-2)
    return torch.where(q >= 8, q - 16, q)


@pytest.mark.parametrize("group,w_mode", [(32, "codes"), (128, "normal"), (32, "normal")])
def test_int4_dequant_matches_torch(group, w_mode):
    spec = LinearSpec("t", M=4, K=256, splits=(96, 40), fmt="int4", group=group, b=32, q_sigma=0.01,
                      w_mode=w_mode, seed=11)
    case = make_linear_case(spec)
    q = _torch_unpack_int4(case["codes"]).float()                       # [N][K]
    s = case["scales"].float().t().repeat_interleave(group, dim=1)      # [N][K]
    ref = (q * s).to(torch.bfloat16)
    got = codecs.dequant_bits("int4", raw(case["codes"]), raw(case["scales"]), spec.K, group)
    assert np.array_equal(got, raw(ref))


def test_fp8_dequant_matches_torch():
    spec = LinearSpec("t", M=4, K=192, splits=(64, 72), fmt="fp8", group=0, b=32, q_sigma=0.01, seed=12)
    case = make_linear_case(spec)
    v = case["codes"].view(torch.float8_e4m3fn).float()
    ref = (v * case["scales"].unsqueeze(1)).to(torch.bfloat16)         # fp32 product, then bf16
    got = codecs.dequant_bits("fp8", raw(case["codes"]), raw(case["scales"]), spec.K, 0)
    assert np.array_equal(got, raw(ref))


def test_mxfp4_dequant_matches_torch():
    spec = LinearSpec("t", M=4, K=256, splits=(64, 40), fmt="mxfp4", group=32, b=32, q_sigma=0.01, seed=13)
    case = make_linear_case(spec)
    mags = torch.tensor(_golden("ocp_fp4_e2m1.json")["codes_0_to_7_magnitude"])
    table = torch.cat([mags, -mags])
    nib = torch.stack([case["codes"] & 0xF, case["codes"] >> 4], dim=-1).flatten(-2).long()
    v = table[nib]
    x = case["scales"].view(torch.float8_e8m0fnu).float().t().repeat_interleave(32, dim=1)
    ref = (v * x).to(torch.bfloat16)
    got = codecs.dequant_bits("mxfp4", raw(case["codes"]), raw(case["scales"]), spec.K, 32)
    assert np.array_equal(got, raw(ref))


def test_dequant_row_and_column_windows():
    spec = LinearSpec("t", M=4, K=256, splits=(50,), fmt="int4", group=32, b=32, q_sigma=0.01, seed=14)
    case = make_linear_case(spec)
    full = codecs.dequant_bits("int4", raw(case["codes"]), raw(case["scales"]), 256, 32)
    rows = np.array([3, 17, 49])
    part = codecs.dequant_bits("int4", raw(case["codes"]), raw(case["scales"]), 256, 32, rows=rows, k0=64, k1=160)
    assert np.array_equal(part, full[rows][:, 64:160])
