"""Bit-exact dequantisation on the MoE paths, through the C ABI.

The chunked MoE calls dequantise each chunk of active experts into a transient
bf16 buffer (the forward's [chunk][N][K] buffer, the backward's transposed
[chunk][2][K][N/2] one, and the full layer's down projections through the first),
and the fused variant decodes the INT4 codes inside the grouped GEMM.  Each decoded
value must equal bf16_rne(q * s) exactly (the canonical decode of the oracle's
codecs), so these tests compare with np.array_equal, not a tolerance."""

import numpy as np
import pytest
import torch

from gen import MoESpec, make_moe_case
from gpu_util import f64
from npcase import raw
from oracle import codecs, moe_ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def oft():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import orthogonal_fine_tuning_b200 as m
    return m


def _random_bank(E, N, K, group, seed):
    """Every code byte and signed scales, so all 16 nibbles (-8 included) and both
    scale signs reach the decoder."""
    g = torch.Generator().manual_seed(seed)
    codes = torch.randint(0, 256, (E, N, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    scales = (torch.rand(E, K // group, N, generator=g) * 0.09 + 0.01)
    sign = torch.where(torch.rand(E, K // group, N, generator=g) < 0.3, -1.0, 1.0)
    return codes, (scales * sign).to(torch.bfloat16)


def _table(E, chunk, seed):
    """A chunk table over a random subset of the experts (ascending), -1 padded."""
    rng = np.random.default_rng(seed)
    active = np.sort(rng.choice(E, size=max(1, E - E // 3), replace=False))
    n_chunks = (E + chunk - 1) // chunk
    t = np.full((n_chunks, chunk), -1, dtype=np.int32)
    for c in range(0, len(active), chunk):
        part = active[c:c + chunk]
        t[c // chunk, :len(part)] = part
    return t


# (E, N = gate + up rows, K, group, chunk): ragged N and K (not multiples of 64),
# groups 32/64/128, a partial last chunk, and the MoE workload's d_in with its bank stride
CASES = [(7, 96, 160, 32, 3), (5, 48, 256, 64, 2), (9, 208, 384, 128, 4), (4, 64, 7168, 32, 2)]


@pytest.mark.parametrize("E,N,K,group,chunk", CASES, ids=[f"E{c[0]}-N{c[1]}-K{c[2]}-g{c[3]}" for c in CASES])
@pytest.mark.parametrize("transpose", [False, True], ids=["rows", "transposed"])
def test_chunk_dequant_bit_exact(oft, E, N, K, group, chunk, transpose):
    codes, scales = _random_bank(E, N, K, group, seed=E * 1000 + K)
    W = oft.Weight("int4", codes.cuda(), scales.cuda(), K, N, group, n_experts=E)
    table = _table(E, chunk, seed=N)
    ct = torch.from_numpy(table).cuda()
    craw, sraw = raw(codes), raw(scales)
    for c in range(table.shape[0]):
        out = oft.oft_moe_chunk_dequant(W, ct, c, chunk, transpose=transpose)
        oft.oft_check_device()
        got = raw(out)
        for s, e in enumerate(table[c]):
            if e < 0:
                continue
            ref = codecs.dequant_bits("int4", craw[e], sraw[e], K, group)      # uint16 [N][K]
            if transpose:
                n = N // 2
                want = np.stack([ref[:n].T, ref[n:].T])                         # [2][K][n]
            else:
                want = ref
            assert np.array_equal(got[s], want), (c, s, int(e))


def test_chunk_dequant_leaves_empty_slots(oft):
    E, N, K, group, chunk = 3, 32, 64, 32, 4
    codes, scales = _random_bank(E, N, K, group, seed=3)
    W = oft.Weight("int4", codes.cuda(), scales.cuda(), K, N, group, n_experts=E)
    ct = torch.tensor([[2, -1, 0, -1]], dtype=torch.int32, device="cuda")
    fill = torch.full((chunk, N, K), 1.5, dtype=torch.bfloat16, device="cuda")
    oft.oft_moe_chunk_dequant(W, ct, 0, chunk, out=fill)
    oft.oft_check_device()
    got = raw(fill)
    one_five = raw(torch.tensor([1.5], dtype=torch.bfloat16))[0]
    assert np.all(got[1] == one_five) and np.all(got[3] == one_five)
    assert np.array_equal(got[0], codecs.dequant_bits("int4", raw(codes)[2], raw(scales)[2], K, group))
    assert np.array_equal(got[2], codecs.dequant_bits("int4", raw(codes)[0], raw(scales)[0], K, group))


# Through the grouped GEMMs: with Q = 0 (R = I exactly), k = 1 (weight exactly 1) and
# one-hot activations, token (e, k) routed to expert e returns row k of deq(W_e)^T,
# i.e. Y[(e, k), r] = deq(W_e)[r][k] -- a single product 1 * w accumulated with exact
# zeros.  This covers the fused variant's in-GEMM INT4 decode in MoE mode (expert
# bank stride, per-expert scale rows, gate/up halves) and the chunked variant's
# buffer + grouped GEMM, value for value.
@pytest.mark.parametrize("fused", [False, True], ids=["chunked", "fused"])
@pytest.mark.parametrize("K,group,n_proj", [(256, 32, 48), (192, 64, 40), (384, 128, 24)])
def test_moe_decode_exact_through_gemm(oft, fused, K, group, n_proj):
    E = 5
    N = 2 * n_proj
    spec = MoESpec("ex", T=E * K, K=K, E=E, n_proj=n_proj, top_k=1, chunk=2, group=group, b=32, q_sigma=0.0,
                   seed=K + n_proj)
    case = make_moe_case(spec)
    codes, scales = _random_bank(E, N, K, group, seed=K * 7 + n_proj)
    case["codes"], case["scales"] = codes, scales
    case["Q"] = torch.zeros_like(case["Q"])
    X = torch.zeros(E * K, K, dtype=torch.bfloat16)
    X[torch.arange(E * K), torch.arange(E * K) % K] = 1.0
    logits = torch.full((E * K, E), -4.0)
    logits[torch.arange(E * K), torch.arange(E * K) // K] = 4.0
    W = oft.Weight("int4", codes.cuda(), scales.cuda(), K, N, group, n_experts=E)
    fwd = oft.moe_fused_oft_fwd if fused else oft.moe_chunked_oft_fwd
    out = fwd(X.cuda(), logits.cuda(), W, spec.b, case["Q"].cuda(), 1, spec.chunk)
    oft.oft_check_device()
    idx, w = moe_ref.topk(raw(logits), 1)
    assert np.array_equal(out["topk_idx"].cpu().numpy(), idx)
    assert np.all(out["topk_w"].cpu().numpy() == 1.0)
    Y = f64(out["Y"])
    for e in range(E):
        ref = codecs.dequant("int4", raw(codes)[e], raw(scales)[e], K, group)   # float64 [N][K]
        np.testing.assert_array_equal(Y[e * K:(e + 1) * K], ref.T)
