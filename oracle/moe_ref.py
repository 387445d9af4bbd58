"""Active-expert-chunked MoE OFT forward (float64 oracle).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

The pages describe it as: the experts that the router selects are grouped into
fixed-size chunks; each chunk is dequantised transiently, fed to a grouped GEMM,
and its high-precision copy is released afterwards, so that peak transient
memory stays bounded by one chunk (m.xxlwj.com 771001, section "技术细节",
paragraph "Active-expert-chunked dequantization"; chooseai.io news 4086,
section "对低精度 MoE 模型的专门优化").  The routing itself is not specified; the
readings taken here are:

  * top-k by logit, descending; ties go to the lower expert index; the slot
    order k is the rank;
  * gating weights are a softmax over the k selected logits (they sum to 1);
  * non-finite logits (a diverging router): NaN ranks as -inf; where selected
    values are infinite the weights are the softmax's limit -- if the largest
    selected logit is +inf, the selected +inf entries share the weight equally
    and the others get 0; if it is -inf (all k selected are -inf or NaN), each
    gets 1/k;
  * each expert e has gate and up projections with independent OFT rotations
    (split-projection applied to the expert's fused gate/up tensor):
        Y_tk = [ (X_t R_e,gate) W_e,gate  |  (X_t R_e,up) W_e,up ]
  * the layer output is Y_t = sum_k w_tk Y_tk in slot order (the gate/up linear
    outputs; no activation and no down projection);
  * bucket order: entries (t, k) sorted by expert, stable in (t, k); active
    experts are those with a non-zero count, ascending; chunk c holds
    active[c*C : (c+1)*C], the last one possibly partial.

Full expert layer (the step after the gate/up output above): each expert also has
a down projection W_e,down (d_in = n, d_out = K) with its own OFT rotation on its
input, and the gated activation between them is SwiGLU:

  h_tk  = silu(g_tk) * u_tk,            [g_tk | u_tk] = Y_tk,  silu(x) = x sigmoid(x)
  Z_tk  = (h_tk R_e,down) W_e,down
  Y_t   = sum_k w_tk Z_tk

Backward (the pages train these expert layers through the adapter only; the
frozen expert weights get no gradient).  With D_p,tk = dY_p[t] W_e,p^T (e =
idx[t, k], p = gate / up):

  dX[t]          = sum_k w_tk sum_p D_p,tk R_e,p^T            (blockwise)
  G_e,p,blk      = sum_{(t,k): idx = e} X[t]_blk^T (w_tk D_p,tk,blk)
  dq_e,p         = Cayley backward of G_e,p (oft_ref.cayley_grad); zero for
                   experts no token selected
  dw_tk          = <dY[t], Y_tk> = sum_p <D_p,tk, X[t] R_e,p>
  dlogit[t, e_k] = w_tk (dw_tk - sum_j w_tj dw_tj)   (softmax over the selected
                   logits); zero for logits that were not selected (top-k is
                   piecewise constant in the logits)

Pins (tests/test_oracle_moe.py, tests/test_oracle_moe_bwd.py): top-k against a
brute-force Python sort; buckets against a dictionary build; chunked order
equals the direct per-token sum; weights sum to one; a router that sends every
token to one expert with k = 1 reduces to the split-projection linear of
oft_ref (forward and backward); central finite differences of the forward for
dX, dq and the logits; dw equals the inner product of dY with the per-slot
expert outputs; each token's logit gradient sums to zero; one expert's dq from
its own entries (expert_dq) equals the full backward's.
"""

from __future__ import annotations

import numpy as np

from .codecs import bf16_bits_to_f64, dequant
from .oft_ref import cayley_grad, packed_len, rotate, rotate_t, rotations


def topk(logits: np.ndarray, k: int):
    """logits fp32 [T][E] -> (idx int32 [T][k], w float64 [T][k]).

    NaN ranks as -inf; the weights follow the limits stated in the module
    docstring when a selected logit is infinite."""
    logits = np.asarray(logits, dtype=np.float32)
    v = np.where(np.isnan(logits), np.float32(-np.inf), logits)
    order = np.argsort(-v, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(v, order, axis=1).astype(np.float64)
    mx = sel.max(axis=1)
    w = np.empty_like(sel)
    fin = np.isfinite(mx)
    z = np.exp(sel[fin] - mx[fin, None])
    w[fin] = z / z.sum(axis=1, keepdims=True)
    top = mx == np.inf
    hit = (sel[top] == np.inf).astype(np.float64)
    w[top] = hit / hit.sum(axis=1, keepdims=True)
    w[mx == -np.inf] = 1.0 / k
    return order.astype(np.int32), w


def buckets(idx: np.ndarray, E: int):
    """idx [T][k] -> (counts [E], offsets [E+1], bucket [T*k]).

    bucket lists the flat entries t*k + slot grouped by expert, each expert's
    entries in increasing (t, slot)."""
    flat = np.asarray(idx).reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    bucket = np.argsort(flat, kind="stable").astype(np.int32)
    return counts, offsets, bucket


def chunk_table(counts: np.ndarray, chunk: int, E: int):
    """Active experts (count > 0) ascending, cut into chunks of `chunk`.

    Returns (n_active, table int32 [ceil(E/chunk)][chunk]) padded with -1."""
    active = np.nonzero(np.asarray(counts) > 0)[0].astype(np.int32)
    n_chunks_max = (E + chunk - 1) // chunk
    table = np.full((n_chunks_max, chunk), -1, dtype=np.int32)
    for c in range(0, len(active), chunk):
        part = active[c:c + chunk]
        table[c // chunk, : len(part)] = part
    return len(active), table


class ExpertBank:
    """Dequantises expert weights on demand from stored INT4 codes/scales.

    codes uint8 [E][2n][K/2], scales bf16 bits [E][K/G][2n]; rows 0..n-1 are the
    gate projection, n..2n-1 the up projection."""

    def __init__(self, codes, scales_bits, K: int, group: int, n_proj: int):
        self.codes, self.scales, self.K, self.group, self.n = codes, scales_bits, K, group, n_proj

    def weight_t(self, e: int, rows=None) -> np.ndarray:
        return dequant("int4", self.codes[e], self.scales[e], self.K, self.group, rows=rows)


def expert_outputs(X: np.ndarray, e: int, bank: ExpertBank, Qe_bits: np.ndarray, b: int, cols=None, R=None):
    """Y_tk for tokens X [m][K] routed to expert e: [m][2n] (or the given columns).

    Qe_bits: packed bf16 bits [2][K/b][b(b-1)/2] for (gate, up); or R, the
    expert's rotations [2][K/b][b][b] given directly (then Qe_bits is unused)."""
    n = bank.n
    if R is None:
        R = rotations(Qe_bits, b)                               # [2][K/b][b][b]
    cols = np.arange(2 * n) if cols is None else np.asarray(cols)
    out = np.empty((X.shape[0], len(cols)))
    for proj in (0, 1):
        sel = np.nonzero((cols >= proj * n) & (cols < (proj + 1) * n))[0]
        if len(sel) == 0:
            continue
        Wt = bank.weight_t(e, rows=cols[sel])
        out[:, sel] = rotate(X, R[proj]) @ Wt.T
    return out


def moe_fwd_direct(X_bits, logits, bank: ExpertBank, Q_bits, b: int, top_k: int, tokens=None, cols=None):
    """Y[t] = sum_k w_tk Y_tk, computed token by token in slot order.

    tokens/cols optionally restrict the rows/columns computed (for sampled
    checks of large problems)."""
    X = bf16_bits_to_f64(X_bits)
    idx, w = topk(logits, top_k)
    T = X.shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    ncols = 2 * bank.n if cols is None else len(cols)
    Y = np.zeros((len(tokens), ncols))
    for i, t in enumerate(tokens):
        for k in range(top_k):
            e = int(idx[t, k])
            Y[i] += w[t, k] * expert_outputs(X[t:t + 1], e, bank, Q_bits[e], b, cols)[0]
    return Y


def moe_fwd_chunked(X_bits, logits, bank: ExpertBank, Q_bits, b: int, top_k: int, chunk: int, E: int):
    """The same result computed in the method's order: route, bucket, walk the
    chunks of active experts, compute each expert's bucket rows (its grouped-GEMM
    rows), then combine per token in slot order.  Returns (Y, routing dict)."""
    X = bf16_bits_to_f64(X_bits)
    T = X.shape[0]
    idx, w = topk(logits, top_k)
    counts, offsets, bucket = buckets(idx, E)
    n_active, table = chunk_table(counts, chunk, E)
    Ytk = np.zeros((T * top_k, 2 * bank.n))
    for c in range(table.shape[0]):
        for e in table[c]:
            if e < 0:
                continue
            ent = bucket[offsets[e]:offsets[e + 1]]
            Ytk[offsets[e]:offsets[e + 1]] = expert_outputs(X[ent // top_k], int(e), bank, Q_bits[e], b)
    pos = np.empty(T * top_k, dtype=np.int64)
    pos[bucket] = np.arange(T * top_k)
    Y = np.zeros((T, 2 * bank.n))
    for k in range(top_k):
        Y += w[:, k:k + 1] * Ytk[pos[np.arange(T) * top_k + k]]
    routing = dict(idx=idx, w=w, counts=counts, offsets=offsets, bucket=bucket, n_active=n_active, table=table)
    return Y, routing


def moe_bwd_direct(dY: np.ndarray, X_bits, logits, bank: ExpertBank, Q_bits, b: int, top_k: int, E: int,
                   tokens=None):
    """Backward of moe_fwd_direct, token by token in slot order.

    dY float64 [T][2n] (gate | up columns).  Returns (dX [T][K],
    dq [E][2][K/b][b(b-1)/2], dlogits [T][E], dw [T][top_k]).
    `tokens` (optional) restricts the work to those tokens, for sampled checks of
    large problems: the rows of dX, dlogits and dw of the other tokens stay zero,
    and dq_e is complete only for experts all of whose tokens are listed."""
    X = bf16_bits_to_f64(X_bits)
    idx, w = topk(logits, top_k)
    T, K = X.shape
    n, nb = bank.n, K // b
    dX = np.zeros((T, K))
    G = np.zeros((E, 2, nb, b, b))
    dw = np.zeros((T, top_k))
    Rs, Ws = {}, {}
    tokens = range(T) if tokens is None else [int(t) for t in tokens]
    for t in tokens:
        for k in range(top_k):
            e = int(idx[t, k])
            if e not in Rs:
                Rs[e], Ws[e] = rotations(Q_bits[e], b), bank.weight_t(e)
            for p in (0, 1):
                D = dY[t, p * n:(p + 1) * n] @ Ws[e][p * n:(p + 1) * n]      # dY_p[t] W_e,p^T, [K]
                dw[t, k] += D @ rotate(X[t:t + 1], Rs[e][p])[0]
                dX[t] += w[t, k] * rotate_t(D[None], Rs[e][p])[0]
                G[e, p] += w[t, k] * np.einsum("ji,jk->jik", X[t].reshape(nb, b), D.reshape(nb, b))
    dq = np.zeros((E, 2, nb, packed_len(b)))
    for e in Rs:
        for p in (0, 1):
            dq[e, p] = cayley_grad(G[e, p], Rs[e][p], b)
    dlogits = np.zeros((T, E))
    s = (w * dw).sum(axis=1)
    for t in tokens:
        for k in range(top_k):
            dlogits[t, idx[t, k]] = w[t, k] * (dw[t, k] - s[t])
    return dX, dq, dlogits, dw


def expert_dq(e: int, dY: np.ndarray, X_bits, logits, bank: ExpertBank, Q_bits, b: int, top_k: int):
    """dq_e [2][K/b][b(b-1)/2] of one expert, from the (t, k) entries routed to it
    only: the same sums as moe_bwd_direct's G_e,p (slot order within each token,
    tokens ascending), batched over the expert's tokens, then the Cayley backward.
    For checks of a heavily loaded expert at full size, where moe_bwd_direct would
    also work through every other expert of those tokens."""
    X = bf16_bits_to_f64(X_bits)
    idx, w = topk(logits, top_k)
    T, K = X.shape
    n, nb = bank.n, K // b
    ts, ks = np.nonzero(idx == e)                  # entries in (t, k) order
    R = rotations(Q_bits[e], b)
    Wt = bank.weight_t(e)
    dq = np.zeros((2, nb, packed_len(b)))
    for p in (0, 1):
        D = dY[ts, p * n:(p + 1) * n] @ Wt[p * n:(p + 1) * n]           # [entries][K]
        wD = w[ts, ks][:, None] * D
        G = np.einsum("mji,mjk->jik", X[ts].reshape(-1, nb, b), wD.reshape(-1, nb, b))
        dq[p] = cayley_grad(G, R[p], b)
    return dq


def silu(x):
    """x * sigmoid(x); sigmoid from exp(-|x|) on both branches, so neither overflows
    nor cancels: 1 / (1 + e^-x) for x >= 0, e^x / (1 + e^x) for x < 0."""
    x = np.asarray(x, dtype=np.float64)
    z = np.exp(-np.abs(x))
    sig = np.where(x >= 0, 1.0 / (1.0 + z), z / (1.0 + z))
    return x * sig


class DownBank(ExpertBank):
    """INT4 down projections: codes uint8 [E][K][n/2], scales bf16 bits [E][n/G][K];
    weight_t(e) is deq(W_e,down)^T [K][n] (one row per output channel)."""

    def __init__(self, codes, scales_bits, n: int, group: int):
        super().__init__(codes, scales_bits, n, group, 0)

    def weight_t(self, e: int, rows=None) -> np.ndarray:
        return dequant("int4", self.codes[e], self.scales[e], self.K, self.group, rows=rows)


def expert_layer(X: np.ndarray, e: int, bank: ExpertBank, down: DownBank, Qe_bits, Qd_bits, b: int):
    """Z for tokens X [m][K] through expert e: [m][K] = (silu(g) u R_e,down) W_e,down."""
    Y = expert_outputs(X, e, bank, Qe_bits, b)
    n = bank.n
    h = silu(Y[:, :n]) * Y[:, n:]
    Rd = rotations(Qd_bits, b)                                  # [n/b][b][b]
    return rotate(h, Rd) @ down.weight_t(e).T


def moe_layer_direct(X_bits, logits, bank: ExpertBank, down: DownBank, Q_bits, Qd_bits, b: int, top_k: int,
                     tokens=None):
    """Y[t] = sum_k w_tk Z_tk for the full expert layer, token by token in slot order.

    Q_bits: gate/up adapters [E][2][K/b][b(b-1)/2]; Qd_bits: down adapters
    [E][n/b][b(b-1)/2].  `tokens` optionally restricts the rows computed."""
    X = bf16_bits_to_f64(X_bits)
    idx, w = topk(logits, top_k)
    T, K = X.shape
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    Y = np.zeros((len(tokens), K))
    for i, t in enumerate(tokens):
        for k in range(top_k):
            e = int(idx[t, k])
            Y[i] += w[t, k] * expert_layer(X[t:t + 1], e, bank, down, Q_bits[e], Qd_bits[e], b)[0]
    return Y
