"""Seeded synthetic workloads.

Shapes and distributions follow the five synthetic workloads that define the
hot path of OFT over a frozen low-precision base ("Orbit" adapter-first RL
post-training, chooseai.io news 4086, sections "技术原理" and "对低精度 MoE 模型的专门优化";
m.xxlwj.com 771001, section "技术细节").  Where a distribution is not fixed by
the workload description, the choice made here is documented on the field.

Storage layouts (shared with the C ABI, include/oft.h):
  * X, dY: bf16 row-major [tokens][features].
  * Weights are stored transposed, one row per output channel: W^T [d_out][d_in].
      - INT4:  codes uint8 [N][K/2], k even in the low nibble, two's complement;
               scales bf16 [K/G][N] (k-group major).
      - FP8:   codes uint8 [N][K] (OCP e4m3fn); scales fp32 [N] (per output channel).
      - MXFP4: codes uint8 [N][K/2] (OCP e2m1, k even in the low nibble);
               scales uint8 [K/32][N] (OCP e8m0).
  * Q (adapter): bf16 packed strict upper triangle, row-major within a block:
      [P splits][K/b blocks][b(b-1)/2].
  * MoE experts: the same per-expert layouts with a leading [E] dimension; the
    gate rows come first (0..n_proj-1), then the up rows.

Nothing here dequantises, rotates or multiplies: the quantisers below only turn
a drawn dense weight into codes and scales (the inverse direction).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

FMT_INT4 = "int4"
FMT_FP8 = "fp8"
FMT_MXFP4 = "mxfp4"


def split_offsets(splits: Sequence[int]):
    """Start column of each sub-projection in the fused output."""
    offs, acc = [], 0
    for n in splits:
        offs.append(acc)
        acc += n
    return offs


@dataclasses.dataclass(frozen=True)
class LinearSpec:
    name: str
    M: int                      # tokens
    K: int                      # d_in
    splits: tuple               # d_out of each sub-projection, in fused order
    fmt: str                    # "int4" | "fp8" | "mxfp4"
    group: int                  # INT4 group (32/128) along d_in; MXFP4: 32; FP8: 0
    b: int                      # OFT block size
    q_sigma: float              # std of the packed upper entries of Q
    w_mode: str = "normal"      # "codes": INT4 codes U{-7..7}, scales U(lo,hi);
                                # "normal": W ~ N(0, w_sigma), then quantised
    w_sigma: float = 0.02
    scale_lo: float = 0.01
    scale_hi: float = 0.05
    backward: bool = False
    seed: int = 0

    @property
    def N(self) -> int:
        return int(sum(self.splits))

    @property
    def P(self) -> int:
        return len(self.splits)

    def with_(self, **kw) -> "LinearSpec":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class MoESpec:
    name: str
    T: int                      # tokens
    K: int                      # hidden (d_in)
    E: int                      # experts
    n_proj: int                 # d_out of each of gate and up
    top_k: int
    chunk: int
    group: int                  # INT4 group along d_in
    b: int
    q_sigma: float
    zipf_s: float = 1.1
    w_sigma: float = 0.02
    seed: int = 0

    def with_(self, **kw) -> "MoESpec":
        return dataclasses.replace(self, **kw)


# The five synthetic workloads (index = position in the workload list).
LINEAR_CONFIGS = {
    # tiny fused-QKV, forward only; codes and scales drawn directly
    "c0": LinearSpec("c0", M=64, K=256, splits=(128, 128, 128), fmt=FMT_INT4, group=32, b=32,
                     q_sigma=0.01, w_mode="codes"),
    # dense fused-QKV fwd+bwd, 4B-class shape, FP8 per-channel
    "c1": LinearSpec("c1", M=4096, K=2560, splits=(4096, 1024, 1024), fmt=FMT_FP8, group=0, b=32,
                     q_sigma=0.02, backward=True, seed=1),
    # gated-MLP gate/up fwd, INT4 group 128
    "c2": LinearSpec("c2", M=8192, K=4096, splits=(12288, 12288), fmt=FMT_INT4, group=128, b=64,
                     q_sigma=0.01, seed=2),
    # large training step fwd+bwd, MXFP4
    "c4": LinearSpec("c4", M=16384, K=7168, splits=(12288, 3072, 3072), fmt=FMT_MXFP4, group=32, b=64,
                     q_sigma=0.02, backward=True, seed=4),
}

MOE_CONFIGS = {
    # Kimi-like expert layer, active-expert-chunked
    "c3": MoESpec("c3", T=4096, K=7168, E=384, n_proj=2048, top_k=8, chunk=16, group=32, b=32,
                  q_sigma=0.01, seed=3),
}


# ----------------------------------------------------------------------------
# quantisers (generator side only)
# ----------------------------------------------------------------------------

def _pack_nibbles(q: torch.Tensor) -> torch.Tensor:
    """int8 [N][K] with values in [-8,7] -> uint8 [N][K/2], even k in the low nibble."""
    u = (q.to(torch.int16) & 0xF).to(torch.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).contiguous()


def _quant_int4(w: torch.Tensor, group: int):
    """w fp32 [N][K] -> (codes uint8 [N][K/2], scales bf16 [K/G][N]).

    Symmetric absmax quantiser: s = bf16(absmax_g / 7), q = clamp(rne(w/s), -7, 7).
    """
    N, K = w.shape
    wg = w.view(N, K // group, group)
    amax = wg.abs().amax(dim=-1)
    s = (amax / 7.0).to(torch.bfloat16)
    s = torch.where(amax == 0, torch.ones_like(s), s)
    q = torch.round(wg / s.float().unsqueeze(-1)).clamp_(-7, 7).to(torch.int8).view(N, K)
    return _pack_nibbles(q), s.t().contiguous()


def _quant_fp8(w: torch.Tensor):
    """w fp32 [N][K] -> (codes uint8 [N][K] e4m3fn, scales fp32 [N])."""
    amax = w.abs().amax(dim=1)
    s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    v = (w / s.unsqueeze(1)).clamp_(-448.0, 448.0)
    codes = v.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    return codes, s.contiguous()


def _rne_e2m1_index(a: torch.Tensor) -> torch.Tensor:
    """|v| -> index into the e2m1 magnitude grid {0,.5,1,1.5,2,3,4,6}, round to
    nearest with ties to the even code, saturating at 6."""
    idx = ((a > 0.25).to(torch.uint8) + (a >= 0.75).to(torch.uint8) + (a > 1.25).to(torch.uint8)
           + (a >= 1.75).to(torch.uint8) + (a > 2.5).to(torch.uint8) + (a >= 3.5).to(torch.uint8)
           + (a > 5.0).to(torch.uint8))
    return idx


def _quant_mxfp4(w: torch.Tensor):
    """w fp32 [N][K] -> (codes uint8 [N][K/2], scales uint8 e8m0 [K/32][N]).

    Shared exponent per 32 along d_in: floor(log2(absmax)) - 2 (emax of e2m1),
    then each element rounded to e2m1 with saturation.
    """
    N, K = w.shape
    wg = w.view(N, K // 32, 32)
    amax = wg.abs().amax(dim=-1)
    e = torch.floor(torch.log2(torch.where(amax > 0, amax, torch.ones_like(amax)))) - 2.0
    e8 = torch.where(amax > 0, (e + 127.0).clamp(0, 254), torch.full_like(e, 127.0))
    x = torch.pow(2.0, (e8 - 127.0).double()).float()
    v = wg / x.unsqueeze(-1)
    idx = _rne_e2m1_index(v.abs())
    code = idx | ((v < 0).to(torch.uint8) << 3)
    codes = _pack_nibbles(code.view(N, K).to(torch.int8))
    return codes, e8.to(torch.uint8).t().contiguous()


def _draw_weight(spec: LinearSpec, N: int, g: torch.Generator, device):
    K = spec.K
    if spec.w_mode == "codes":
        assert spec.fmt == FMT_INT4
        q = torch.randint(-7, 8, (N, K), generator=g, device=device, dtype=torch.int8)
        s = torch.empty(K // spec.group, N, device=device).uniform_(spec.scale_lo, spec.scale_hi, generator=g)
        return _pack_nibbles(q), s.to(torch.bfloat16).contiguous()
    w = torch.randn(N, K, generator=g, device=device) * spec.w_sigma
    if spec.fmt == FMT_INT4:
        return _quant_int4(w, spec.group)
    if spec.fmt == FMT_FP8:
        return _quant_fp8(w)
    if spec.fmt == FMT_MXFP4:
        return _quant_mxfp4(w)
    raise ValueError(spec.fmt)


def _draw_q(P: int, K: int, b: int, sigma: float, g: torch.Generator, device, lead=()):
    n = b * (b - 1) // 2
    q = torch.randn(*lead, P, K // b, n, generator=g, device=device) * sigma
    return q.to(torch.bfloat16).contiguous()


def make_linear_case(spec: LinearSpec, device="cpu", q_zero: bool = False):
    """Draw one OFT-linear problem.  Returns a dict of tensors on `device`."""
    g = torch.Generator(device=device)
    g.manual_seed(1000 + spec.seed)
    x = torch.randn(spec.M, spec.K, generator=g, device=device).to(torch.bfloat16)
    codes, scales = _draw_weight(spec, spec.N, g, device)
    q = _draw_q(spec.P, spec.K, spec.b, spec.q_sigma, g, device)
    if q_zero:
        q = torch.zeros_like(q)
    case = dict(spec=spec, X=x, codes=codes, scales=scales, Q=q)
    if spec.backward:
        case["dY"] = torch.randn(spec.M, spec.N, generator=g, device=device).to(torch.bfloat16)
    return case


def make_moe_router(spec: MoESpec, device="cpu"):
    """Router logits fp32 [T][E]: N(0,1) noise plus ln p_rank(e), where
    p_r is Zipf(s) over ranks 1..E and a seeded permutation assigns ranks."""
    g = torch.Generator(device="cpu")
    g.manual_seed(7000 + spec.seed)
    perm = torch.randperm(spec.E, generator=g)
    ranks = torch.arange(1, spec.E + 1, dtype=torch.float64)
    p = ranks.pow(-spec.zipf_s)
    p = p / p.sum()
    bias = torch.log(p)[perm].to(torch.float32)
    noise = torch.randn(spec.T, spec.E, generator=g)
    return (noise + bias.unsqueeze(0)).to(torch.float32).contiguous().to(device)


def make_moe_grad(spec: MoESpec, device="cpu"):
    """Upstream gradient of the MoE layer output, bf16 [T][2 n_proj] (gate | up)."""
    g = torch.Generator(device=device)
    g.manual_seed(9000 + spec.seed)
    return torch.randn(spec.T, 2 * spec.n_proj, generator=g, device=device).to(torch.bfloat16)


def make_moe_down(spec: MoESpec, device="cpu", experts: Optional[Sequence[int]] = None):
    """Down projections of a full expert layer (d_in = n_proj, d_out = K) and their
    adapters: codes uint8 [E][K][n_proj/2], scales bf16 [E][n_proj/G][K] (INT4, group
    G along n_proj), Q_down bf16 [E][n_proj/b][b(b-1)/2].  One generator per expert,
    as for the gate/up bank."""
    g = torch.Generator(device=device)
    g.manual_seed(5000 + spec.seed)
    qd = _draw_q(1, spec.n_proj, spec.b, spec.q_sigma, g, device, lead=(spec.E,))[:, 0].contiguous()
    codes = torch.zeros(spec.E, spec.K, spec.n_proj // 2, dtype=torch.uint8, device=device)
    scales = torch.ones(spec.E, spec.n_proj // spec.group, spec.K, dtype=torch.bfloat16, device=device)
    wspec = LinearSpec("down", M=0, K=spec.n_proj, splits=(spec.K,), fmt=FMT_INT4, group=spec.group, b=spec.b,
                       q_sigma=0.0, w_sigma=spec.w_sigma)
    ge = torch.Generator(device=device)
    for e in (range(spec.E) if experts is None else experts):
        ge.manual_seed(200000 + 1000 * spec.seed + e)
        c, s_ = _draw_weight(wspec, spec.K, ge, device)
        codes[e].copy_(c)
        scales[e].copy_(s_)
    return dict(down_codes=codes, down_scales=scales, Q_down=qd)


def make_moe_case(spec: MoESpec, device="cpu", experts: Optional[Sequence[int]] = None):
    """Draw one chunked-MoE OFT problem.

    Each expert's weight is drawn from its own generator seeded with the expert id,
    on `device`, so that large expert banks are drawn where they will live.
    `experts` (optional) restricts which experts get non-zero weights drawn; the
    rest stay zero (used by small CPU tests only).
    """
    g = torch.Generator(device=device)
    g.manual_seed(3000 + spec.seed)
    x = torch.randn(spec.T, spec.K, generator=g, device=device).to(torch.bfloat16)
    q = _draw_q(2, spec.K, spec.b, spec.q_sigma, g, device, lead=(spec.E,))
    N = 2 * spec.n_proj
    codes = torch.zeros(spec.E, N, spec.K // 2, dtype=torch.uint8, device=device)
    scales = torch.ones(spec.E, spec.K // spec.group, N, dtype=torch.bfloat16, device=device)
    wspec = LinearSpec("expert", M=0, K=spec.K, splits=(N,), fmt=FMT_INT4, group=spec.group, b=spec.b,
                       q_sigma=0.0, w_sigma=spec.w_sigma)
    ge = torch.Generator(device=device)
    for e in (range(spec.E) if experts is None else experts):
        ge.manual_seed(100000 + 1000 * spec.seed + e)
        c, s = _draw_weight(wspec, N, ge, device)
        codes[e].copy_(c)
        scales[e].copy_(s)
    logits = make_moe_router(spec, device=device)
    return dict(spec=spec, X=x, logits=logits, codes=codes, scales=scales, Q=q)
