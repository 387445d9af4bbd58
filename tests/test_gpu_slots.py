"""Double-buffered adapter slots: an upload into the inactive slot, made while the
active slot serves a forward, becomes visible to compute only after activate(), and
the rotations it builds equal the library's rotation build of the same Q."""

import pytest
import torch

from gen import LinearSpec, make_linear_case
from gpu_util import device_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def oft():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import orthogonal_fine_tuning_b200 as m
    return m


def test_upload_then_activate(oft):
    spec = LinearSpec("slots", M=300, K=512, splits=(256, 128, 128), fmt="fp8", group=0, b=32, q_sigma=0.05, seed=3)
    case = make_linear_case(spec)
    W = device_weight(case, "cuda")
    X = case["X"].cuda()
    g = torch.Generator().manual_seed(5)
    q1 = case["Q"].pin_memory()
    q2 = (torch.randn(case["Q"].shape, generator=g) * 0.05).to(torch.bfloat16).pin_memory()
    slots = oft.AdapterSlots(tuple(case["Q"].shape), spec.b, "cuda")
    with pytest.raises(RuntimeError):
        slots.activate()
    slots.upload(q1)
    Q, R = slots.activate()
    assert torch.equal(Q.cpu(), q1)
    assert torch.equal(R, oft.oft_build_rotation(q1.cuda(), spec.b))
    y1 = oft.oft_linear_fwd(X, W, spec.splits, spec.b, R)
    # stage q2 while the forward on slot 1 is queued; compute still sees q1 until activate()
    slots.upload(q2)
    y1b = oft.oft_linear_fwd(X, W, spec.splits, spec.b, slots.current()[1])
    Q2, R2 = slots.activate()
    y2 = oft.oft_linear_fwd(X, W, spec.splits, spec.b, R2)
    torch.cuda.synchronize()
    oft.oft_check_device()
    assert torch.equal(y1, y1b)
    assert torch.equal(Q2.cpu(), q2)
    ref2 = oft.oft_linear_fwd(X, W, spec.splits, spec.b, oft.oft_build_rotation(q2.cuda(), spec.b))
    assert torch.equal(y2, ref2)
    assert not torch.equal(y2, y1)
    # and back: the first slot is reused once compute has moved off it
    slots.upload(q1)
    _, R3 = slots.activate()
    assert torch.equal(oft.oft_linear_fwd(X, W, spec.splits, spec.b, R3), y1)
