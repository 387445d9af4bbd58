"""Active-expert MoE OFT forward on the GPU through the C ABI, in both variants:
chunked (experts dequantised chunk by chunk into a bf16 buffer) and fused
(decoded inside the grouped GEMM).  Routing, buckets and chunk table bit-exact
against the oracle; Y within tolerance."""

import numpy as np
import pytest
import torch

from gen import MOE_CONFIGS, MoESpec, make_moe_case
from gpu_util import TOL, f64, rel_err
from npcase import raw
from oracle import moe_ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def oft():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import orthogonal_fine_tuning_b200 as m
    return m


def _run(oft, case, fused=False):
    spec = case["spec"]
    W = oft.Weight("int4", case["codes"], case["scales"], spec.K, 2 * spec.n_proj, spec.group, n_experts=spec.E)
    fwd = oft.moe_fused_oft_fwd if fused else oft.moe_chunked_oft_fwd
    out = fwd(case["X"], case["logits"], W, spec.b, case["Q"], spec.top_k, spec.chunk)
    oft.oft_check_device()
    return out


@pytest.fixture(params=[False, True], ids=["chunked", "fused"])
def fused(request):
    return request.param


def _check_routing(out, logits_np, spec):
    idx, w = moe_ref.topk(logits_np, spec.top_k)
    counts, offsets, bucket = moe_ref.buckets(idx, spec.E)
    n_active, table = moe_ref.chunk_table(counts, spec.chunk, spec.E)
    assert np.array_equal(out["topk_idx"].cpu().numpy(), idx)
    assert np.array_equal(out["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(out["bucket"].cpu().numpy(), bucket)
    assert int(out["n_active"].item()) == n_active
    assert np.array_equal(out["chunk_table"].cpu().numpy(), table)
    assert rel_err(out["topk_w"].cpu().double().numpy(), w) < 1e-5
    return idx


def _to(case, dev):
    return {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in case.items()}


@pytest.mark.parametrize("T,E,top_k,chunk,b,K", [(200, 24, 4, 4, 32, 256), (77, 9, 3, 2, 16, 256), (64, 5, 1, 3, 64, 256),
                                                  (50, 7, 2, 3, 32, 160)])
def test_small_moe(oft, fused, T, E, top_k, chunk, b, K):
    spec = MoESpec("s", T=T, K=K, E=E, n_proj=48, top_k=top_k, chunk=chunk, group=32, b=b, q_sigma=0.05,
                   seed=T + E)
    case = make_moe_case(spec)
    out = _run(oft, _to(case, "cuda"), fused)
    _check_routing(out, raw(case["logits"]), spec)
    bank = moe_ref.ExpertBank(raw(case["codes"]), raw(case["scales"]), spec.K, spec.group, spec.n_proj)
    Yref, _ = moe_ref.moe_fwd_chunked(raw(case["X"]), raw(case["logits"]), bank, raw(case["Q"]), b, top_k, chunk, E)
    assert rel_err(f64(out["Y"]), Yref) < TOL


def test_ties_in_logits_go_to_lower_expert(oft):
    spec = MoESpec("t", T=64, K=128, E=16, n_proj=16, top_k=4, chunk=4, group=32, b=32, q_sigma=0.05, seed=1)
    case = make_moe_case(spec)
    g = torch.Generator().manual_seed(0)
    case["logits"] = torch.randint(-2, 3, (64, 16), generator=g).float()
    out = _run(oft, _to(case, "cuda"))
    _check_routing(out, raw(case["logits"]), spec)


def test_non_finite_logits(oft, fused):
    """A diverging router: rows of NaN, -inf and +inf logits.  NaN ranks as -inf, so
    every index stays a real expert; routing is bit-exact with the oracle, the weights
    follow the softmax's limits, and Y stays within tolerance."""
    spec = MoESpec("nf", T=96, K=128, E=12, n_proj=32, top_k=4, chunk=3, group=32, b=32, q_sigma=0.05, seed=11)
    case = make_moe_case(spec)
    g = torch.Generator().manual_seed(5)
    lg = torch.randn(spec.T, spec.E, generator=g)
    u = torch.rand(spec.T, spec.E, generator=g)
    lg[u < 0.25] = float("nan")
    lg[(u >= 0.25) & (u < 0.35)] = float("-inf")
    lg[(u >= 0.35) & (u < 0.40)] = float("inf")
    lg[0] = float("nan")
    lg[1] = float("-inf")
    lg[2, :] = float("nan")
    lg[2, 7] = 0.5
    case["logits"] = lg
    out = _run(oft, _to(case, "cuda"), fused)
    idx = _check_routing(out, raw(case["logits"]), spec)
    assert idx.min() >= 0 and idx.max() < spec.E
    _, w = moe_ref.topk(raw(case["logits"]), spec.top_k)
    assert np.array_equal(out["topk_w"].cpu().numpy()[:2], w[:2].astype(np.float32))
    bank = moe_ref.ExpertBank(raw(case["codes"]), raw(case["scales"]), spec.K, spec.group, spec.n_proj)
    Yref, _ = moe_ref.moe_fwd_chunked(raw(case["X"]), raw(case["logits"]), bank, raw(case["Q"]), spec.b, spec.top_k,
                                      spec.chunk, spec.E)
    Y = f64(out["Y"])
    assert np.all(np.isfinite(Y))
    assert rel_err(Y, Yref) < TOL


def test_c3_full_routing_and_sampled_output(oft, fused):
    """Kimi-like expert layer: 4096 tokens, hidden 7168, 384 INT4-g32 experts of
    2 x 2048, top-8 over Zipf-biased logits, chunks of 16, b=32."""
    spec = MOE_CONFIGS["c3"]
    case = make_moe_case(spec, device="cuda")
    out = _run(oft, case, fused)
    logits = raw(case["logits"])
    _check_routing(out, logits, spec)
    rng = np.random.default_rng(0)
    toks = np.unique(np.concatenate([[0, spec.T - 1], rng.choice(spec.T, 14, replace=False)]))
    cols = np.unique(np.concatenate([[0, 2047, 2048, 4095], rng.choice(4096, 60, replace=False)]))
    # oracle inputs: the generated expert codes for the experts these tokens use
    idx, _ = moe_ref.topk(logits, spec.top_k)
    used = np.unique(idx[toks])
    codes = np.zeros((spec.E,) + tuple(case["codes"].shape[1:]), dtype=np.uint8)
    scales = np.zeros((spec.E,) + tuple(case["scales"].shape[1:]), dtype=np.uint16)
    for e in used:
        codes[e] = raw(case["codes"][int(e)])
        scales[e] = raw(case["scales"][int(e)])
    bank = moe_ref.ExpertBank(codes, scales, spec.K, spec.group, spec.n_proj)
    Yref = moe_ref.moe_fwd_direct(raw(case["X"]), logits, bank, raw(case["Q"]), spec.b, spec.top_k,
                                  tokens=toks, cols=cols)
    assert rel_err(f64(out["Y"])[toks][:, cols], Yref) < TOL


def test_fused_matches_chunked(oft):
    """Both variants compute the same product: identical routing, Y within tolerance
    of each other on a ragged case (hidden size not a multiple of 64, experts with
    a single token)."""
    spec = MoESpec("fc", T=90, K=160, E=13, n_proj=40, top_k=3, chunk=5, group=32, b=32, q_sigma=0.05, seed=77)
    case = _to(make_moe_case(spec), "cuda")
    a, f = _run(oft, case, False), _run(oft, case, True)
    for k in ("topk_idx", "offsets", "bucket", "chunk_table", "n_active"):
        assert torch.equal(a[k], f[k]), k
    assert rel_err(f64(f["Y"]), f64(a["Y"])) < TOL
