"""MoE adapter backward on the GPU through the C ABI (moe_chunked_oft_bwd) against
the float64 oracle: dX, the per-expert dq (zero for idle experts) and the router
logit gradient, on ragged small cases and, sampled, on the Kimi-like expert layer."""

import numpy as np
import pytest
import torch

from gen import MOE_CONFIGS, MoESpec, make_moe_case, make_moe_grad
from gpu_util import TOL, f64, rel_err
from npcase import raw
from oracle import moe_ref
from oracle.codecs import bf16_bits_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def oft():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import orthogonal_fine_tuning_b200 as m
    return m


def _bwd(oft, case, dY, want_dlogits=True):
    spec = case["spec"]
    W = oft.Weight("int4", case["codes"], case["scales"], spec.K, 2 * spec.n_proj, spec.group, n_experts=spec.E)
    out = oft.moe_chunked_oft_bwd(dY, case["X"], case["logits"], W, spec.b, case["Q"], spec.top_k, spec.chunk,
                                  want_dlogits=want_dlogits)
    oft.oft_check_device()
    return out


def _to(case, dev):
    return {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in case.items()}


@pytest.mark.parametrize("T,E,top_k,chunk,b,K,n", [
    (120, 10, 3, 4, 32, 256, 96),   # three chunks, the last partial
    (77, 9, 2, 2, 16, 256, 64),
    (64, 6, 1, 3, 64, 256, 128),    # k = 1: the logit gradient vanishes
    (50, 7, 2, 3, 32, 160, 72),     # hidden and projection widths not multiples of 64
    (300, 40, 4, 16, 32, 128, 64),  # idle experts (dq must be zero), one full chunk
    (600, 4, 2, 2, 32, 192, 64),    # experts of about 300 rows: several row tiles per unit
    (96, 8, 2, 4, 32, 4096, 32),    # wide hidden: several (expert, column group) units per CTA
    (96, 8, 2, 4, 64, 4096, 32),
    (96, 8, 3, 4, 16, 2048, 32),
])
def test_small_moe_backward(oft, T, E, top_k, chunk, b, K, n):
    spec = MoESpec("sb", T=T, K=K, E=E, n_proj=n, top_k=top_k, chunk=chunk, group=32, b=b, q_sigma=0.05,
                   seed=3 * T + E)
    case = make_moe_case(spec)
    dY = make_moe_grad(spec)
    out = _bwd(oft, _to(case, "cuda"), dY.cuda())
    bank = moe_ref.ExpertBank(raw(case["codes"]), raw(case["scales"]), K, spec.group, n)
    dX, dq, dlog, _ = moe_ref.moe_bwd_direct(bf16_bits_to_f64(raw(dY)), raw(case["X"]), raw(case["logits"]), bank,
                                             raw(case["Q"]), b, top_k, E)
    assert rel_err(f64(out["dX"]), dX) < TOL
    got_dq = f64(out["dQ"])
    assert rel_err(got_dq, dq) < TOL
    idle = ~np.isin(np.arange(E), moe_ref.topk(raw(case["logits"]), top_k)[0])
    assert not got_dq[idle].any()
    got_dl = f64(out["dlogits"])
    if top_k == 1:
        assert not got_dl.any()
    else:
        assert rel_err(got_dl, dlog) < TOL
    # unselected logits get exactly zero
    sel = np.zeros((T, E), dtype=bool)
    np.put_along_axis(sel, moe_ref.topk(raw(case["logits"]), top_k)[0].astype(np.int64), True, axis=1)
    assert not got_dl[~sel].any()


def test_backward_is_deterministic_and_dlogits_optional(oft):
    spec = MoESpec("sd", T=150, K=192, E=12, n_proj=64, top_k=3, chunk=4, group=32, b=32, q_sigma=0.05, seed=4)
    case = _to(make_moe_case(spec), "cuda")
    dY = make_moe_grad(spec).cuda()
    a = _bwd(oft, case, dY)
    b = _bwd(oft, case, dY)
    c = _bwd(oft, case, dY, want_dlogits=False)
    for k in ("dX", "dQ", "dlogits"):
        assert torch.equal(a[k], b[k]), k
    assert torch.equal(a["dX"], c["dX"]) and torch.equal(a["dQ"], c["dQ"])


class _Rows:
    """Expert-indexed view of a device tensor, copied to the host on demand."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return raw(self.t[int(e)])


def test_c3_backward_sampled(oft):
    """Kimi-like expert layer (4096 tokens, hidden 7168, 384 INT4-g32 experts of
    2 x 2048, top-8, chunks of 16, b = 32): dX and dlogits on sampled tokens, dq
    of two lightly loaded experts (computed from all of their tokens), and the full
    dq of a heavily loaded expert (the eighth most loaded, over a thousand routed
    tokens, several 128-row tiles of its grouped GEMM)."""
    spec = MOE_CONFIGS["c3"]
    case = make_moe_case(spec, device="cuda")
    dY = make_moe_grad(spec, device="cuda")
    out = _bwd(oft, case, dY)
    logits = raw(case["logits"])
    idx, _ = moe_ref.topk(logits, spec.top_k)
    counts = np.bincount(idx.reshape(-1), minlength=spec.E)
    light = [int(e) for e in np.nonzero((counts >= 2) & (counts <= 4))[0][:2]]
    assert len(light) == 2
    toks = set([0, spec.T - 1, 1234])
    for e in light:
        toks |= set(np.nonzero((idx == e).any(axis=1))[0].tolist())
    toks = sorted(toks)
    bank = moe_ref.ExpertBank(_Rows(case["codes"]), _Rows(case["scales"]), spec.K, spec.group, spec.n_proj)
    dX, dq, dlog, _ = moe_ref.moe_bwd_direct(bf16_bits_to_f64(raw(dY)), raw(case["X"]), logits, bank, raw(case["Q"]),
                                             spec.b, spec.top_k, spec.E, tokens=toks)
    assert rel_err(f64(out["dX"])[toks], dX[toks]) < TOL
    assert rel_err(f64(out["dlogits"])[toks], dlog[toks]) < TOL
    got_dq = f64(out["dQ"])
    for e in light:
        assert rel_err(got_dq[e], dq[e]) < TOL
    idle = counts == 0
    assert not got_dq[idle].any()
    heavy = int(np.argsort(-counts, kind="stable")[7])
    assert counts[heavy] > 1000
    dq_h = moe_ref.expert_dq(heavy, bf16_bits_to_f64(raw(dY)), raw(case["X"]), logits, bank, raw(case["Q"]), spec.b,
                             spec.top_k)
    assert rel_err(got_dq[heavy], dq_h) < TOL
