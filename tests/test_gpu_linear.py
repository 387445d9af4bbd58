"""Split-projection OFT linear, forward and backward, on the GPU through the C
ABI, against the float64 oracle.  Small and ragged shapes are compared element
by element; the full-size workloads are compared in full (the fused-QKV FP8
workload) or on sampled tokens, columns and rotation blocks."""

import numpy as np
import pytest
import torch

from gen import LINEAR_CONFIGS, LinearSpec, make_linear_case
from gpu_util import TOL, OracleLinear, device_weight, f64, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def oft():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import orthogonal_fine_tuning_b200 as m
    return m


def _run(oft, case, backward):
    spec = case["spec"]
    W = device_weight(case, "cuda")
    X, Q = case["X"].cuda(), case["Q"].cuda()
    R = oft.oft_build_rotation(Q, spec.b)
    Y = oft.oft_linear_fwd(X, W, spec.splits, spec.b, R)
    out = dict(Y=Y)
    if backward:
        out["dX"], out["dQ"] = oft.oft_linear_bwd(case["dY"].cuda(), X, W, spec.splits, spec.b, R)
    oft.oft_check_device()
    return out


SMALL = [
    # name, M, K, splits, fmt, group, b
    ("c0", 64, 256, (128, 128, 128), "int4", 32, 32),
    ("ragged-fp8", 300, 352, (264, 8, 136), "fp8", 0, 32),
    ("ragged-mxfp4", 129, 192, (520, 264), "mxfp4", 32, 64),
    ("one-token", 1, 128, (8,), "int4", 128, 16),
    ("four-splits", 257, 512, (64, 136, 256, 40), "int4", 64, 64),
    ("wide-k", 130, 1024, (384,), "fp8", 0, 16),
    ("small-m-mxfp4", 37, 2048, (264, 1032), "mxfp4", 32, 64),
    ("small-m-fp8", 64, 1536, (256, 128, 128), "fp8", 0, 32),
    # 80 tiles of 256 x 256 on 74 CTA pairs (a second, partial wave), ragged in both
    # tokens and columns
    ("wave-tail", 1000, 256, (2560, 2440), "int4", 32, 32),
]


@pytest.fixture(params=[1, 2, 3, 4], ids=["one-cta", "pair", "plain-pair", "plain"])
def gemm_mode(oft, request):
    """Every GEMM path: the fused-dequant one-CTA kernel, the 2-SM pair, and the bf16
    weight copy with the plain tcgen05 GEMM on 2-SM pairs or on one CTA per tile."""
    oft.oft_set_gemm_mode(request.param)
    yield request.param
    oft.oft_set_gemm_mode(0)


@pytest.mark.parametrize("name,M,K,splits,fmt,group,b", SMALL, ids=[s[0] for s in SMALL])
def test_small_fwd_bwd(oft, gemm_mode, name, M, K, splits, fmt, group, b):
    spec = LinearSpec(name, M=M, K=K, splits=splits, fmt=fmt, group=group, b=b, q_sigma=0.05,
                      w_mode="codes" if name == "c0" else "normal", backward=True, seed=len(name) + M)
    case = make_linear_case(spec)
    got = _run(oft, case, True)
    ref = OracleLinear(case)
    assert rel_err(f64(got["Y"]), ref.fwd()) < TOL
    dX, dq = ref.bwd()
    assert rel_err(f64(got["dX"]), dX) < TOL
    assert rel_err(f64(got["dQ"]), dq) < TOL


def test_q_zero_reduces_to_base_gemm(oft):
    spec = LinearSpec("q0", M=190, K=256, splits=(136, 120), fmt="int4", group=32, b=32, q_sigma=0.0, seed=9)
    case = make_linear_case(spec, q_zero=True)
    got = _run(oft, case, False)
    ref = OracleLinear(case)
    base = ref.X @ ref.Wt.T                       # plain dequantised GEMM
    assert rel_err(f64(got["Y"]), base) < TOL
    # and the GPU base path itself: rotation by I leaves X unchanged bit for bit
    R = oft.oft_build_rotation(case["Q"].cuda(), 32)
    Xr = oft.oft_rotate(case["X"].cuda(), R, 32)
    assert torch.equal(Xr[0].cpu(), case["X"]) and torch.equal(Xr[1].cpu(), case["X"])


def test_c0_forward(oft):
    case = make_linear_case(LINEAR_CONFIGS["c0"])
    got = _run(oft, case, False)
    assert rel_err(f64(got["Y"]), OracleLinear(case).fwd()) < TOL


def test_c1_full_fwd_bwd(oft):
    """Dense fused-QKV FP8 workload (4096 x 2560 -> 4096/1024/1024, b=32), every output."""
    case = make_linear_case(LINEAR_CONFIGS["c1"])
    got = _run(oft, case, True)
    ref = OracleLinear(case)
    assert rel_err(f64(got["Y"]), ref.fwd()) < TOL
    dX, dq = ref.bwd()
    assert rel_err(f64(got["dX"]), dX) < TOL
    assert rel_err(f64(got["dQ"]), dq) < TOL


def _sample(n, k, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=k, replace=False)]))


def test_c2_sampled_fwd(oft):
    """Gated-MLP gate/up INT4-g128 workload (8192 x 4096 -> 2 x 12288, b=64), sampled outputs."""
    case = make_linear_case(LINEAR_CONFIGS["c2"])
    got = _run(oft, case, False)
    ref = OracleLinear(case)
    rows, cols = _sample(8192, 96, 1), _sample(24576, 768, 2)
    assert rel_err(f64(got["Y"])[rows][:, cols], ref.fwd(rows=rows, cols=cols)) < TOL


def test_c4_sampled_fwd_bwd(oft):
    """Large MXFP4 training step (16384 x 7168 -> 12288/3072/3072, b=64): sampled Y
    and dX rows; dQ of every rotation block of the K sub-projection (112 blocks, all
    16384 tokens: the whole longest-first backward schedule feeds them) and of sampled
    blocks of the other two."""
    case = make_linear_case(LINEAR_CONFIGS["c4"])
    got = _run(oft, case, True)
    ref = OracleLinear(case)
    rows, cols = _sample(16384, 64, 3), _sample(18432, 2048, 4)
    assert rel_err(f64(got["Y"])[rows][:, cols], ref.fwd(rows=rows, cols=cols)) < TOL
    drows = _sample(16384, 64, 5)
    assert rel_err(f64(got["dX"])[drows], ref.dx_rows(drows)) < TOL
    dQ = f64(got["dQ"])
    assert rel_err(dQ[1], ref.dq_split(1)) < TOL
    for p, j in [(0, 0), (0, 111), (2, 3), (2, 110)]:
        assert rel_err(dQ[p, j], ref.dq_block(p, j)) < TOL


@pytest.mark.parametrize("name,M,K,splits,fmt,group,b", SMALL, ids=[s[0] for s in SMALL])
def test_weight_side_forward(oft, name, M, K, splits, fmt, group, b):
    """The weight-side variant, Y_p = X (R_p deq(W_p)), against the same oracle."""
    spec = LinearSpec(name, M=M, K=K, splits=splits, fmt=fmt, group=group, b=b, q_sigma=0.05,
                      w_mode="codes" if name == "c0" else "normal", seed=len(name) + M + 1)
    case = make_linear_case(spec)
    W = device_weight(case, "cuda")
    R = oft.oft_build_rotation(case["Q"].cuda(), b)
    Y = oft.oft_linear_fwd_weight_side(case["X"].cuda(), W, splits, b, R)
    oft.oft_check_device()
    assert rel_err(f64(Y), OracleLinear(case).fwd()) < TOL


def test_weight_side_c2_sampled(oft):
    """Gate/up INT4-g128 workload through the weight-side variant, sampled outputs."""
    case = make_linear_case(LINEAR_CONFIGS["c2"])
    spec = case["spec"]
    W = device_weight(case, "cuda")
    R = oft.oft_build_rotation(case["Q"].cuda(), spec.b)
    Y = oft.oft_linear_fwd_weight_side(case["X"].cuda(), W, spec.splits, spec.b, R)
    oft.oft_check_device()
    rows, cols = _sample(8192, 64, 11), _sample(24576, 512, 12)
    assert rel_err(f64(Y)[rows][:, cols], OracleLinear(case).fwd(rows=rows, cols=cols)) < TOL
