"""oft_linear_fwd_noalloc: the split-projection forward for callers that cannot
allocate device memory or hand over a workspace -- a runtime whose memory pool
already owns the free HBM, or a plugin interface that passes only inputs and
outputs.  Its scratch is the library's fixed device array, so its output must
match the workspace-based oft_linear_fwd, call after call (the array keeps the
previous call's contents).  This file is collected last on purpose."""

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


def test_noalloc_rejects_shapes_beyond_its_scratch(oft):
    spec = LINEAR_CONFIGS["c1"]             # 4096 x 2560 -> 6144 needs ~94 MB of scratch
    case = make_linear_case(spec.with_(M=8))
    W = device_weight(case, "cuda")
    X = torch.zeros(4096, spec.K, dtype=torch.bfloat16, device="cuda")
    R = torch.zeros(spec.P, spec.K // spec.b, spec.b, spec.b, device="cuda")
    Y = torch.empty(4096, spec.N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(oft.OFTError) as ei:
        oft.oft_linear_fwd_noalloc(X, W, spec.splits, spec.b, R, Y)
    assert ei.value.code == 5 and "scratch" in str(ei.value)
