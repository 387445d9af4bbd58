"""oft_linear_fwd_noalloc: the split-projection forward for callers that cannot
allocate device memory or hand over a workspace -- a runtime whose memory pool
already owns the free HBM, or a plugin interface that passes only inputs and
outputs.  Its scratch is the library's fixed device array, so its output must
match the workspace-based oft_linear_fwd, call after call (the array keeps the
previous call's contents).  This file is collected last on purpose."""

import ctypes

import pytest
import torch

from gen import LINEAR_CONFIGS, LinearSpec, make_linear_case
from gpu_util import TOL, device_weight, f64, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def oft():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import orthogonal_fine_tuning_b200 as m
    return m


def _both(oft, case):
    spec = case["spec"]
    W = device_weight(case, "cuda")
    X, Q = case["X"].cuda(), case["Q"].cuda()
    R = oft.oft_build_rotation(Q, spec.b)
    Y_ws = oft.oft_linear_fwd(X, W, spec.splits, spec.b, R)
    Y_na = torch.full_like(Y_ws, float("nan"))
    oft.oft_linear_fwd_noalloc(X, W, spec.splits, spec.b, R, Y_na)
    oft.oft_check_device()
    return Y_ws, Y_na


def test_noalloc_matches_workspace_forward_on_consecutive_calls(oft):
    cases = [
        make_linear_case(LINEAR_CONFIGS["c0"]),
        make_linear_case(LinearSpec("na", M=300, K=352, splits=(264, 8, 136), fmt="fp8", group=0, b=32,
                                    q_sigma=0.05, seed=21)),
    ]
    for case in cases:                      # two calls in a row, different shapes and formats
        Y_ws, Y_na = _both(oft, case)
        assert rel_err(f64(Y_na), f64(Y_ws)) < TOL
        assert torch.equal(Y_na, Y_ws)      # same kernels on the same inputs


from orthogonal_fine_tuning_b200 import _lib, binding  # noqa: E402


def _fwd_with_workspace(oft, X, W, splits, b, R, Y, nbytes):
    """oft_linear_fwd through the C ABI with a caller workspace of exactly `nbytes`
    (the binding would grow a workspace smaller than the size query asks for)."""
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    cw, cs = W.c(), binding._split(splits)
    binding._check(binding._L.oft_linear_fwd(binding._ptr(X), X.shape[0], ctypes.byref(cw), ctypes.byref(cs), b,
                                              binding._ptr(R), binding._ptr(Y), binding._ptr(ws), nbytes,
                                              binding._stream(None)))
    return Y


def test_noalloc_large_token_paths(oft):
    """From 2048 tokens: a shape whose bf16 weight copy fits beside X' in the array
    (the bf16-weight path, with the weight dequantised on the side stream into the
    array), and one where only X' fits (the fused-decode path), each called twice in
    a row with the other in between; both match oft_linear_fwd given a workspace of
    the array's size."""
    specs = [LinearSpec("na_plain", M=2048, K=1024, splits=(512, 256, 256), fmt="int4", group=32, b=32,
                        q_sigma=0.05, seed=31),
             LinearSpec("na_fused", M=2048, K=2560, splits=(4096, 1024, 1024), fmt="fp8", group=0, b=32,
                        q_sigma=0.02, seed=32)]
    runs = []
    for spec in specs:
        case = make_linear_case(spec)
        W = device_weight(case, "cuda")
        X, R = case["X"].cuda(), oft.oft_build_rotation(case["Q"].cuda(), spec.b)
        Y_ref = _fwd_with_workspace(oft, X, W, spec.splits, spec.b, R,
                                    torch.empty(spec.M, spec.N, dtype=torch.bfloat16, device="cuda"),
                                    _lib.OFT_NOALLOC_SCRATCH_BYTES)
        runs.append((spec, X, W, R, Y_ref))
    for _ in range(2):
        for spec, X, W, R, Y_ref in runs:
            Y = torch.full_like(Y_ref, float("nan"))
            oft.oft_linear_fwd_noalloc(X, W, spec.splits, spec.b, R, Y)
            oft.oft_check_device()
            assert torch.equal(Y, Y_ref), spec.name


def test_noalloc_rejects_shapes_beyond_its_scratch(oft):
    spec = LINEAR_CONFIGS["c1"]             # 4096 x 2560 x 3 splits: X' alone is ~63 MB
    case = make_linear_case(spec.with_(M=8))
    W = device_weight(case, "cuda")
    X = torch.zeros(4096, spec.K, dtype=torch.bfloat16, device="cuda")
    R = torch.zeros(spec.P, spec.K // spec.b, spec.b, spec.b, device="cuda")
    Y = torch.empty(4096, spec.N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(oft.OFTError) as ei:
        oft.oft_linear_fwd_noalloc(X, W, spec.splits, spec.b, R, Y)
    assert ei.value.code == 5 and "scratch" in str(ei.value)
