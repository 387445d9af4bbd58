"""OFT-adapted linear: Cayley rotation, split-projection forward, adapter backward.

TEST INFRASTRUCTURE ONLY -- see the package docstring.

The pages fix the method at the level of concepts: a frozen low-precision base
with a BF16 OFT adapter carrying all gradients (chooseai.io news 4086, section
"技术原理：低精度基座 + BF16 适配器 + OFT"), one independent orthogonal rotation per
sub-projection of a fused QKV or gate/up tensor (same page, sections
"适配器优先架构的五大设计特性" item "自定义适配器核函数" and "OFT 相比 LoRA 的架构优势"
item "分投影适配器支持"), and a backward that skips the frozen base's weight
gradient (m.xxlwj.com 771001, section "技术细节", the DeepSeek V4 paragraph).
The formulas are the standard OFT definition:

  Q_blk     skew-symmetric b x b, parameterised by its strict upper triangle
  R_blk     = (I + Q_blk)(I - Q_blk)^-1              (Cayley map)
  R_p       = blockdiag(R_p,0 ... R_p,K/b-1)          one per sub-projection p
  y_p       = W_p^T (R_p^T x)  for a column token x;  row-major:  X'_p = X R_p,
  Y_p       = X'_p W_p,  Y = [Y_0 | Y_1 | ...]        (W_p = deq(W)[:, cols of p])

Backward (no gradient for the frozen W):
  dX'_p     = dY_p W_p^T
  dX        = sum_p dX'_p R_p^T
  G_p,blk   = X_blk^T dX'_p,blk                        (dL/dR_p,blk)
  dQ_full   = 1/2 (I + R)^T G (I + R)^T               (Cayley backward)
  dq_ij     = dQ_full[i, j] - dQ_full[j, i]   for i < j

Derivation of the Cayley backward: with A = I - Q, R = A^-1 (I + Q) and
dR = A^-1 dQ (I + R); hence dL/dQ = A^-T G (I + R)^T, and A^-T = (I + Q)^-1 =
((I + R)/2)^T because I + R = 2 A^-1.  Q_ij = q, Q_ji = -q projects it onto q.

Pins (tests/test_oracle_oft.py): Q = 0 gives R = I and the plain base GEMM;
R^T R = I and det R = +1; R(-Q) = R(Q)^T; the b = 2 closed form; the Cayley
power series I + 2Q + 2Q^2 + ...; a hand-computed rotation golden value that
fixes the R versus R^T convention; row-norm preservation; split equals
separately adapted layers concatenated; central finite differences for dX
and dQ; dq = 2(G - G^T) at Q = 0.
"""

from __future__ import annotations

import numpy as np

from .codecs import bf16_bits_to_f64, dequant


def packed_len(b: int) -> int:
    return b * (b - 1) // 2


def unpack_skew(qp: np.ndarray, b: int) -> np.ndarray:
    """[..., b(b-1)/2] strict-upper entries (row-major) -> skew [..., b, b]."""
    qp = np.asarray(qp, dtype=np.float64)
    iu, ju = np.triu_indices(b, 1)
    Q = np.zeros(qp.shape[:-1] + (b, b), dtype=np.float64)
    Q[..., iu, ju] = qp
    Q[..., ju, iu] = -qp
    return Q


def pack_upper(A: np.ndarray, b: int) -> np.ndarray:
    """[..., b, b] -> its strict upper triangle, row-major."""
    iu, ju = np.triu_indices(b, 1)
    return np.asarray(A)[..., iu, ju]


def cayley(Q: np.ndarray) -> np.ndarray:
    """R = (I + Q)(I - Q)^-1 for a stack of skew blocks [..., b, b].

    The two factors commute, so R also equals (I - Q)^-1 (I + Q), which is the
    solution of (I - Q) R = (I + Q)."""
    b = Q.shape[-1]
    I = np.eye(b)
    return np.linalg.solve(I - Q, np.broadcast_to(I, Q.shape) + Q)


def rotations(qp_bits_or_values, b: int, is_bits: bool = True) -> np.ndarray:
    """Packed Q (bf16 bits, or float values) [..., K/b, b(b-1)/2] -> R [..., K/b, b, b]."""
    qv = bf16_bits_to_f64(qp_bits_or_values) if is_bits else np.asarray(qp_bits_or_values, dtype=np.float64)
    return cayley(unpack_skew(qv, b))


def rotate(X: np.ndarray, R: np.ndarray) -> np.ndarray:
    """X' = X blockdiag(R): X [M][K], R [K/b][b][b]."""
    M, K = X.shape
    nb, b, _ = R.shape
    assert nb * b == K
    return np.einsum("mji,jik->mjk", X.reshape(M, nb, b), R).reshape(M, K)


def rotate_t(D: np.ndarray, R: np.ndarray) -> np.ndarray:
    """D blockdiag(R)^T."""
    M, K = D.shape
    nb, b, _ = R.shape
    return np.einsum("mjk,jik->mji", D.reshape(M, nb, b), R).reshape(M, K)


def split_bounds(splits):
    out, acc = [], 0
    for n in splits:
        out.append((acc, acc + n))
        acc += n
    return out


def linear_fwd(X: np.ndarray, Wt: np.ndarray, splits, R: np.ndarray) -> np.ndarray:
    """Y = [ (X R_p) W_p ]_p.  X [M][K] float64; Wt = deq(W)^T [N][K]; R [P][K/b][b][b]."""
    outs = []
    for p, (n0, n1) in enumerate(split_bounds(splits)):
        outs.append(rotate(X, R[p]) @ Wt[n0:n1].T)
    return np.concatenate(outs, axis=1)


def cayley_grad(G: np.ndarray, R: np.ndarray, b: int) -> np.ndarray:
    """dL/dR = G per block [nb][b][b] -> dq [nb][b(b-1)/2] (Cayley backward).

    dQ_full = 1/2 (I + R)^T G (I + R)^T, then dq_ij = dQ_full[i, j] - dQ_full[j, i]."""
    T = np.swapaxes(np.eye(b) + R, -1, -2)
    dQf = 0.5 * T @ G @ T
    return pack_upper(dQf, b) - pack_upper(np.swapaxes(dQf, -1, -2), b)


def linear_bwd(dY: np.ndarray, X: np.ndarray, Wt: np.ndarray, splits, R: np.ndarray, b: int,
               return_parts: bool = False):
    """Adapter backward.  Returns dX [M][K] and dq [P][K/b][b(b-1)/2]."""
    M, K = X.shape
    nb = K // b
    dX = np.zeros((M, K))
    dq, parts = [], []
    for p, (n0, n1) in enumerate(split_bounds(splits)):
        dXp = dY[:, n0:n1] @ Wt[n0:n1]                       # dY_p W_p^T
        dX += rotate_t(dXp, R[p])
        G = np.einsum("mji,mjk->jik", X.reshape(M, nb, b), dXp.reshape(M, nb, b))
        dq.append(cayley_grad(G, R[p], b))
        parts.append(dict(dXp=dXp, G=G))
    dq = np.stack(dq)
    if return_parts:
        return dX, dq, parts
    return dX, dq


# ----------------------------------------------------------------------------
# convenience wrappers over generator outputs (numpy arrays of raw storage)
# ----------------------------------------------------------------------------


def weight_t(case_np: dict, rows=None, k0: int = 0, k1=None) -> np.ndarray:
    """deq(W)^T [N][K] in float64 from a case holding fmt/codes/scales/K/group."""
    return dequant(case_np["fmt"], case_np["codes"], case_np["scales"], case_np["K"], case_np["group"],
                   rows=rows, k0=k0, k1=k1)
