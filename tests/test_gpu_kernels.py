"""Single steps of the path on the GPU, through the C ABI, against the oracle:
bit-exact dequantisation, Cayley forward/backward, block rotation, and the
bounded-wait error path."""

import numpy as np
import pytest
import torch

from gen import LinearSpec, make_linear_case
from gpu_util import TOL, device_weight, f64, rel_err
from npcase import linear_np, raw
from oracle import codecs, oft_ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def oft():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import orthogonal_fine_tuning_b200 as m
    return m


DQ_CASES = [
    ("int4", 32, "codes", 384, 256),
    ("int4", 128, "normal", 200, 512),
    ("int4", 64, "normal", 72, 192),
    ("fp8", 0, "normal", 136, 352),
    ("mxfp4", 32, "normal", 264, 224),
]


@pytest.mark.parametrize("fmt,group,mode,N,K", DQ_CASES)
@pytest.mark.parametrize("transpose", [False, True])
def test_dequant_bit_exact(oft, fmt, group, mode, N, K, transpose):
    spec = LinearSpec("dq", M=1, K=K, splits=(N,), fmt=fmt, group=group, b=32, q_sigma=0.0, w_mode=mode, seed=N)
    case = make_linear_case(spec)
    W = device_weight(case, "cuda")
    out = oft.oft_dequant_weight(W, transpose=transpose)
    torch.cuda.synchronize()
    got = raw(out)
    ref = codecs.dequant_bits(fmt, raw(case["codes"]), raw(case["scales"]), K, group)
    if transpose:
        ref = ref.T
    assert got.shape == ref.shape
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("b,sigma", [(16, 0.05), (32, 0.02), (32, 0.5), (64, 0.02), (64, 0.5)])
def test_cayley_forward(oft, b, sigma):
    g = torch.Generator().manual_seed(b)
    Q = (torch.randn(3, 7, b * (b - 1) // 2, generator=g) * sigma).to(torch.bfloat16)
    R = oft.oft_build_rotation(Q.cuda(), b)
    ref = oft_ref.rotations(raw(Q), b)
    got = f64(R)
    assert np.abs(got - ref).max() < 2e-5 * max(1.0, sigma * b)
    I = np.eye(b)
    assert np.abs(np.swapaxes(got, -1, -2) @ got - I).max() < 1e-4


@pytest.mark.parametrize("b,sigma", [(16, 0.05), (32, 0.05), (64, 0.05), (32, 0.5)])
def test_cayley_forward_many_blocks(oft, b, sigma):
    """Launches of many blocks take the unrolled pivot loop; same result bar (also with
    a large Q, whose pivots grow well above 1)."""
    g = torch.Generator().manual_seed(100 + b)
    Q = (torch.randn(4101, b * (b - 1) // 2, generator=g) * sigma).to(torch.bfloat16)
    R = oft.oft_build_rotation(Q.cuda(), b)
    ref = oft_ref.rotations(raw(Q), b)
    got = f64(R)
    assert np.abs(got - ref).max() < 2e-5 * max(1.0, sigma * b)
    I = np.eye(b)
    assert np.abs(np.swapaxes(got, -1, -2) @ got - I).max() < 1e-4


@pytest.mark.parametrize("nblocks", [5, 4100])
def test_cayley_zero_is_identity(oft, nblocks):
    """Q = 0 gives R = I exactly, for the small-launch and the many-block forms."""
    Q = torch.zeros(nblocks, 32 * 31 // 2, dtype=torch.bfloat16, device="cuda")
    R = oft.oft_build_rotation(Q, 32)
    assert torch.equal(R.cpu(), torch.eye(32).expand(nblocks, 32, 32))


@pytest.mark.parametrize("b", [16, 32, 64])
def test_cayley_backward(oft, b):
    g = torch.Generator().manual_seed(100 + b)
    Q = (torch.randn(4, b * (b - 1) // 2, generator=g) * 0.05).to(torch.bfloat16)
    G = torch.randn(4, b, b, generator=g)
    R = oft.oft_build_rotation(Q.cuda(), b)
    dq = oft.oft_cayley_backward(R, G.cuda(), b)
    Rr = oft_ref.rotations(raw(Q), b)
    T = np.swapaxes(np.eye(b) + Rr, -1, -2)
    D = 0.5 * T @ G.double().numpy() @ T
    ref = oft_ref.pack_upper(D, b) - oft_ref.pack_upper(np.swapaxes(D, -1, -2), b)
    assert rel_err(f64(dq), ref) < 1e-4


@pytest.mark.parametrize("M,K,P,b", [(64, 256, 3, 32), (131, 192, 2, 64), (1, 64, 1, 16), (200, 352, 4, 32)])
def test_rotate(oft, M, K, P, b):
    spec = LinearSpec("r", M=M, K=K, splits=(8,) * P, fmt="int4", group=32, b=b, q_sigma=0.05, seed=M)
    case = make_linear_case(spec)
    c = linear_np(case)
    R = oft.oft_build_rotation(case["Q"].cuda(), b)
    Xr = oft.oft_rotate(case["X"].cuda(), R, b)
    Rr = oft_ref.rotations(c["Q"], b)
    X = codecs.bf16_bits_to_f64(c["X"])
    for p in range(P):
        assert rel_err(f64(Xr[p]), oft_ref.rotate(X, Rr[p])) < TOL


def test_bounded_wait_reports_timeout_and_context_survives(oft):
    oft.oft_debug_bounded_wait(2000)          # 2 ms: a barrier nothing completes
    with pytest.raises(oft.OFTError) as ei:
        oft.oft_check_device()
    assert ei.value.code == 4
    oft.oft_check_device()                    # the word was cleared
    Q = torch.zeros(2, 32 * 31 // 2, dtype=torch.bfloat16, device="cuda")
    R = oft.oft_build_rotation(Q, 32)         # the context is still usable
    assert torch.equal(R.cpu(), torch.eye(32).expand(2, 32, 32))


# The fused GEMM decodes the weight inside its producer warps, so its decode is
# checked through the GEMM itself: with Q = 0 (R = I exactly) and one-hot
# activations, every output is a single product 1 * w accumulated with exact
# zeros, so the forward returns deq(W)^T and the backward's dX returns deq(W)
# value for value.  Scales cover the decode's special paths: FP8 channel scales
# too large to carry the 2^120 of the bit-pattern decode (and negative ones),
# MXFP4 exponents on both sides of the two-step factor (kept where every value
# and product stays finite and normal).
FUSED_DQ_CASES = [
    ("int4", 32, 256, (136, 120)),
    ("int4", 128, 384, (200, 56)),
    ("fp8", 0, 256, (136, 64, 40)),
    ("mxfp4", 32, 256, (264, 8)),
]


def _extreme_scales(fmt, scales, seed):
    g = torch.Generator().manual_seed(seed)
    if fmt == "fp8":
        s = scales.clone()
        big = torch.tensor([200.0, -1000.0, 3.0e4, 128.0, -0.75])
        idx = torch.arange(0, s.numel(), 5)
        s[idx] = big[torch.arange(idx.numel()) % big.numel()]
        s[1::11] = -s[1::11]
        return s
    if fmt == "mxfp4":
        return torch.randint(2, 253, scales.shape, generator=g).to(torch.uint8)
    s = scales.clone()
    s[1::7] = -s[1::7]
    return s


@pytest.mark.parametrize("fmt,group,K,splits", FUSED_DQ_CASES, ids=[f"{c[0]}-{c[2]}" for c in FUSED_DQ_CASES])
def test_fused_decode_exact_through_gemm(oft, fmt, group, K, splits):
    N = sum(splits)
    spec = LinearSpec("fdq", M=K, K=K, splits=splits, fmt=fmt, group=group, b=32, q_sigma=0.0, w_mode="normal",
                      seed=K + N)
    case = make_linear_case(spec, q_zero=True)
    case["scales"] = _extreme_scales(fmt, case["scales"], N)
    W = device_weight(case, "cuda")
    ref = codecs.dequant(fmt, raw(case["codes"]), raw(case["scales"]), K, group)  # [N][K] float64
    assert np.all(np.isfinite(ref))
    R = oft.oft_build_rotation(case["Q"].cuda(), spec.b)
    eye_k = torch.eye(K, dtype=torch.bfloat16, device="cuda")
    Y = oft.oft_linear_fwd(eye_k, W, splits, spec.b, R)
    dX, _ = oft.oft_linear_bwd(torch.eye(N, dtype=torch.bfloat16, device="cuda"),
                               torch.zeros(N, K, dtype=torch.bfloat16, device="cuda"), W, splits, spec.b, R)
    oft.oft_check_device()
    np.testing.assert_array_equal(f64(Y), ref.T)
    np.testing.assert_array_equal(f64(dX), ref)
