"""The small-M forward (1 to 128 tokens: the decode / rollout shape) on the GPU
through the C ABI.  The library runs it on the split-K, weight-stream kernel
(gemm mode 0 picks it); here it is compared with the float64
oracle element by element on ragged shapes, token counts that are not multiples
of 16, reductions that end inside a code tile, several units per CTA and split
counts from 1 to 8, and value for value (one-hot tokens, Q = 0) for the decode
itself.  The decode-like workloads (the fused-QKV FP8 and MXFP4 weights at 64
tokens) are compared on sampled columns."""

import numpy as np
import pytest
import torch

from gen import LINEAR_CONFIGS, LinearSpec, make_linear_case
from gpu_util import TOL, OracleLinear, device_weight, f64, rel_err
from npcase import linear_np
from oracle import codecs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def oft():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import orthogonal_fine_tuning_b200 as m
    return m


def _fwd(oft, case):
    spec = case["spec"]
    W = device_weight(case, "cuda")
    X, Q = case["X"].cuda(), case["Q"].cuda()
    R = oft.oft_build_rotation(Q, spec.b)
    Y = oft.oft_linear_fwd(X, W, spec.splits, spec.b, R)
    oft.oft_check_device()
    return Y


CASES = [
    # name, M, K, splits, fmt, group, b
    ("int4-g32", 64, 512, (256, 128, 128), "int4", 32, 32),
    ("int4-g128-ragged", 37, 384, (264, 8, 136), "int4", 128, 32),
    ("int4-g64-k-tail", 16, 320, (200, 56), "int4", 64, 16),
    ("fp8", 64, 1536, (256, 128, 128), "fp8", 0, 32),
    ("fp8-k-tail", 128, 160, (136, 64, 40), "fp8", 0, 32),
    ("mxfp4", 37, 2048, (264, 1032), "mxfp4", 32, 64),
    ("mxfp4-one-token", 1, 768, (512, 256), "mxfp4", 32, 64),
    ("mxfp4-128", 128, 1024, (640, 384), "mxfp4", 32, 64),
    ("int4-many-tiles", 24, 1024, (12288, 4096), "int4", 128, 64),   # 128 tiles: one split
    ("fp8-deep", 48, 4096, (384, 128), "fp8", 0, 64),                 # 4 tiles: eight splits
]


@pytest.mark.parametrize("name,M,K,splits,fmt,group,b", CASES, ids=[c[0] for c in CASES])
def test_small_m_forward(oft, name, M, K, splits, fmt, group, b):
    spec = LinearSpec(name, M=M, K=K, splits=splits, fmt=fmt, group=group, b=b, q_sigma=0.05,
                      seed=M + K + len(splits))
    case = make_linear_case(spec)
    Y = _fwd(oft, case)
    assert rel_err(f64(Y), OracleLinear(case).fwd()) < TOL


@pytest.mark.parametrize("M", [1, 16, 37, 64, 128])
@pytest.mark.parametrize("fmt,group", [("int4", 32), ("fp8", 0), ("mxfp4", 32)])
def test_small_m_token_counts(oft, M, fmt, group):
    spec = LinearSpec("tok", M=M, K=1024, splits=(384, 136, 8), fmt=fmt, group=group, b=32, q_sigma=0.05,
                      seed=M * 3 + len(fmt))
    case = make_linear_case(spec)
    Y = _fwd(oft, case)
    assert rel_err(f64(Y), OracleLinear(case).fwd()) < TOL


@pytest.mark.parametrize("fmt,group,K,extreme", [("int4", 32, 352, False), ("int4", 128, 512, False),
                                                 ("fp8", 0, 320, False), ("mxfp4", 32, 512, False),
                                                 ("mxfp4", 32, 768, True)])
def test_small_m_decode_exact(oft, fmt, group, K, extreme):
    """One-hot tokens with Q = 0 (R = I exactly): token m selects input feature k_m, so
    Y[m][n] = deq(W)[n][k_m] -- a single product 1 * w summed with exact zeros, split-K
    partials included.  Every k of the reduction is covered by windows of 64 tokens.
    The extreme case draws e8m0 exponents over 2..252, so both the one-step and the
    two-step scale factors of the MXFP4 decode are exercised."""
    splits = (264, 136)
    N = sum(splits)
    spec = LinearSpec("ex", M=64, K=K, splits=splits, fmt=fmt, group=group, b=32, q_sigma=0.0, seed=K + N)
    case = make_linear_case(spec, q_zero=True)
    if extreme:
        g = torch.Generator().manual_seed(K)
        case["scales"] = torch.randint(2, 253, case["scales"].shape, generator=g).to(torch.uint8)
    c = linear_np(case)
    ref = codecs.dequant(fmt, c["codes"], c["scales"], K, group)     # float64 [N][K]
    W = device_weight(case, "cuda")
    R = oft.oft_build_rotation(case["Q"].cuda(), spec.b)
    for k0 in range(0, K, 64):
        ks = [min(K - 1, k0 + m) for m in range(64)]
        X = torch.zeros(64, K, dtype=torch.bfloat16)
        X[torch.arange(64), torch.tensor(ks)] = 1.0
        Y = oft.oft_linear_fwd(X.cuda(), W, splits, spec.b, R)
        oft.oft_check_device()
        np.testing.assert_array_equal(f64(Y), ref[:, ks].T)


@pytest.mark.parametrize("name", ["c1-m64", "c4-m64"])
def test_decode_workloads_sampled(oft, name):
    """The fused-QKV FP8 weights and the MXFP4 training-step weights at 64 tokens."""
    base = LINEAR_CONFIGS[name[:2]]
    spec = base.with_(M=64, backward=False)
    case = make_linear_case(spec)
    Y = f64(_fwd(oft, case))
    rng = np.random.default_rng(7)
    N = spec.N
    bounds = np.cumsum((0,) + tuple(spec.splits))
    cols = np.unique(np.concatenate([bounds[:-1], bounds[1:] - 1, rng.choice(N, 96, replace=False)]))
    ref = OracleLinear(case).fwd(cols=cols)
    assert rel_err(Y[:, cols], ref) < TOL


def test_small_m_repeat_is_deterministic(oft):
    """Split-K partials are summed in split order by whichever CTA finishes a tile last,
    so two calls give the same bits."""
    spec = LinearSpec("det", M=64, K=4096, splits=(512, 256), fmt="fp8", group=0, b=32, q_sigma=0.05, seed=5)
    case = make_linear_case(spec)
    W = device_weight(case, "cuda")
    X, R = case["X"].cuda(), oft.oft_build_rotation(case["Q"].cuda(), spec.b)
    Y1 = oft.oft_linear_fwd(X, W, spec.splits, spec.b, R)
    Y2 = oft.oft_linear_fwd(X, W, spec.splits, spec.b, R)
    oft.oft_check_device()
    assert torch.equal(Y1, Y2)
