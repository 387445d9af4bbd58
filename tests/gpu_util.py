"""Helpers shared by the GPU parity tests: move a generated case to the device,
call the library through the C ABI, and compare with the float64 oracle."""

import numpy as np
import torch

from npcase import linear_np, raw
from oracle import oft_ref
from oracle.codecs import bf16_bits_to_f64

TOL = 2e-2  # max-abs error relative to the reference RMS, for every floating-point result


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.abs(got - ref).max() / max(rms, 1e-300))


def f64(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return bf16_bits_to_f64(raw(t))
    return t.double().numpy()


def device_weight(case, dev):
    import orthogonal_fine_tuning_b200 as oft
    spec = case["spec"]
    return oft.Weight(spec.fmt, case["codes"].to(dev), case["scales"].to(dev), spec.K, spec.N, spec.group)


class OracleLinear:
    """Float64 reference for one generated linear case (optionally on a subset)."""

    def __init__(self, case):
        self.c = linear_np(case)
        self.spec = case["spec"]
        self.X = bf16_bits_to_f64(self.c["X"])
        self.R = oft_ref.rotations(self.c["Q"], self.spec.b)
        self._Wt = None

    @property
    def Wt(self):
        if self._Wt is None:
            self._Wt = oft_ref.weight_t(self.c)
        return self._Wt

    def fwd(self, rows=None, cols=None):
        X = self.X if rows is None else self.X[rows]
        if cols is None:
            return oft_ref.linear_fwd(X, self.Wt, self.spec.splits, self.R)
        cols = np.asarray(cols)
        out = np.empty((X.shape[0], len(cols)))
        for p, (n0, n1) in enumerate(oft_ref.split_bounds(self.spec.splits)):
            sel = np.nonzero((cols >= n0) & (cols < n1))[0]
            if len(sel):
                Wt = oft_ref.weight_t(self.c, rows=cols[sel])
                out[:, sel] = oft_ref.rotate(X, self.R[p]) @ Wt.T
        return out

    def bwd(self):
        dY = bf16_bits_to_f64(self.c["dY"])
        return oft_ref.linear_bwd(dY, self.X, self.Wt, self.spec.splits, self.R, self.spec.b)

    def dx_rows(self, rows):
        """dX for a subset of tokens (needs the whole weight)."""
        dY = bf16_bits_to_f64(self.c["dY"][rows])
        out = np.zeros((len(rows), self.spec.K))
        for p, (n0, n1) in enumerate(oft_ref.split_bounds(self.spec.splits)):
            out += oft_ref.rotate_t(dY[:, n0:n1] @ self.Wt[n0:n1], self.R[p])
        return out

    def dq_split(self, p):
        """dq of every rotation block of sub-projection p (needs every token): the
        oracle backward of that sub-projection alone."""
        b = self.spec.b
        n0, n1 = oft_ref.split_bounds(self.spec.splits)[p]
        dY = bf16_bits_to_f64(self.c["dY"][:, n0:n1])
        Wt = oft_ref.weight_t(self.c, rows=np.arange(n0, n1))                  # [N_p][K]
        _, dq = oft_ref.linear_bwd(dY, self.X, Wt, (n1 - n0,), self.R[p:p + 1], b)
        return dq[0]

    def dq_block(self, p, j):
        """dq of rotation block j of sub-projection p (needs every token)."""
        b = self.spec.b
        n0, n1 = oft_ref.split_bounds(self.spec.splits)[p]
        dY = bf16_bits_to_f64(self.c["dY"][:, n0:n1])
        Wt = oft_ref.weight_t(self.c, rows=np.arange(n0, n1), k0=j * b, k1=(j + 1) * b)   # [N_p][b]
        dXp = dY @ Wt                                                                       # [M][b]
        G = self.X[:, j * b:(j + 1) * b].T @ dXp
        T = (np.eye(b) + self.R[p, j]).T
        D = 0.5 * T @ G @ T
        iu, ju = np.triu_indices(b, 1)
        return D[iu, ju] - D[ju, iu]
