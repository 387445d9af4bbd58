"""Full MoE expert layer on the GPU through the C ABI (moe_chunked_oft_layer_fwd):
gate/up, SwiGLU and the down projection with its own OFT adapter, every expert weight
INT4 and dequantised chunk by chunk, against the float64 oracle; ragged small cases
and the Kimi-like expert layer sampled."""

import numpy as np
import pytest
import torch

from gen import MOE_CONFIGS, MoESpec, make_moe_case, make_moe_down
from gpu_util import TOL, f64, rel_err
from npcase import raw
from oracle import moe_ref

pytestmark = pytest.mark.gpu

# Two GEMMs in series, each with a bf16 operand (X R for gate/up, h R_down for down),
# then the bf16 output: twice the single-GEMM bar.  On the first small case the
# float64 emulation of exactly this rounding chain lands at 3.12e-2 of the reference
# RMS, the same figure the GPU result gives (the output there has max/RMS = 6.5).
TOL_LAYER = 2 * TOL


@pytest.fixture(scope="module")
def oft():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import orthogonal_fine_tuning_b200 as m
    return m


def _layer(oft, case, down):
    spec = case["spec"]
    W = oft.Weight("int4", case["codes"], case["scales"], spec.K, 2 * spec.n_proj, spec.group, n_experts=spec.E)
    Wd = oft.Weight("int4", down["down_codes"], down["down_scales"], spec.n_proj, spec.K, spec.group,
                    n_experts=spec.E)
    Y = oft.moe_chunked_oft_layer_fwd(case["X"], case["logits"], W, Wd, spec.b, case["Q"], down["Q_down"],
                                      spec.top_k, spec.chunk)
    oft.oft_check_device()
    return Y


def _to(d, dev):
    return {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in d.items()}


class _Rows:
    """Expert-indexed view of a device tensor, copied to the host on demand."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return raw(self.t[int(e)])


@pytest.mark.parametrize("T,E,top_k,chunk,b,K,n", [
    (120, 10, 3, 4, 32, 256, 96),   # three chunks, the last partial
    (77, 9, 2, 2, 16, 256, 64),
    (64, 6, 1, 3, 64, 256, 128),
    (50, 7, 2, 3, 32, 160, 64),     # hidden size not a multiple of 64
    (300, 40, 4, 16, 32, 128, 64),  # idle experts, one full chunk
])
def test_small_moe_layer(oft, T, E, top_k, chunk, b, K, n):
    spec = MoESpec("sl", T=T, K=K, E=E, n_proj=n, top_k=top_k, chunk=chunk, group=32, b=b, q_sigma=0.05,
                   seed=5 * T + E)
    case, down = make_moe_case(spec), make_moe_down(spec)
    Y = _layer(oft, _to(case, "cuda"), _to(down, "cuda"))
    bank = moe_ref.ExpertBank(raw(case["codes"]), raw(case["scales"]), K, spec.group, n)
    dbank = moe_ref.DownBank(raw(down["down_codes"]), raw(down["down_scales"]), n, spec.group)
    Yref = moe_ref.moe_layer_direct(raw(case["X"]), raw(case["logits"]), bank, dbank, raw(case["Q"]),
                                    raw(down["Q_down"]), b, top_k)
    assert rel_err(f64(Y), Yref) < TOL_LAYER


def test_c3_layer_sampled(oft):
    """Kimi-like expert layer (4096 tokens, hidden 7168, 384 experts of 2 x 2048 gate/up
    and 2048 -> 7168 down, INT4 g32, top-8, chunks of 16, b = 32), sampled tokens."""
    spec = MOE_CONFIGS["c3"]
    case = make_moe_case(spec, device="cuda")
    down = make_moe_down(spec, device="cuda")
    Y = _layer(oft, case, down)
    toks = [0, 1777, spec.T - 1]
    bank = moe_ref.ExpertBank(_Rows(case["codes"]), _Rows(case["scales"]), spec.K, spec.group, spec.n_proj)
    dbank = moe_ref.DownBank(_Rows(down["down_codes"]), _Rows(down["down_scales"]), spec.n_proj, spec.group)
    Yref = moe_ref.moe_layer_direct(raw(case["X"]), raw(case["logits"]), bank, dbank, raw(case["Q"]),
                                    raw(down["Q_down"]), spec.b, spec.top_k, tokens=toks)
    assert rel_err(f64(Y)[toks], Yref) < TOL_LAYER
