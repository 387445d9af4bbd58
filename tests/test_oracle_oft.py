"""Pins for oracle.oft_ref: Cayley build, split-projection forward, adapter backward.

Expected values come from closed forms (tests/golden/cayley_closed_forms.json),
the Cayley power series, orthogonality invariants, special cases that reduce
to a plain matmul, and central finite differences of the forward.
"""

import json
import os

import numpy as np
import pytest

from oracle import oft_ref
from oracle.codecs import bf16_bits_to_f64
from gen import LinearSpec, make_linear_case
from npcase import linear_np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _golden():
    with open(os.path.join(GOLDEN, "cayley_closed_forms.json")) as f:
        return json.load(f)


def _rand_q(shape, b, sigma):
    return RNG.normal(0, sigma, size=shape + (b * (b - 1) // 2,))


def test_packing_order_b3():
    Q = oft_ref.unpack_skew(np.array([1.0, 2.0, 3.0]), 3)     # (0,1), (0,2), (1,2)
    assert np.array_equal(Q, np.array([[0, 1, 2], [-1, 0, 3], [-2, -3, 0]], dtype=float))


def test_cayley_zero_is_identity():
    for b in (2, 16, 32, 64):
        R = oft_ref.cayley(oft_ref.unpack_skew(np.zeros((3, b * (b - 1) // 2)), b))
        assert np.array_equal(R, np.broadcast_to(np.eye(b), R.shape))


def test_cayley_b2_closed_form():
    for case in _golden()["b2"]["cases"]:
        R = oft_ref.cayley(oft_ref.unpack_skew(np.array([case["a"]]), 2))
        np.testing.assert_allclose(R, np.array(case["R"]), rtol=0, atol=1e-15)


@pytest.mark.parametrize("b,sigma", [(16, 0.05), (32, 0.02), (64, 0.02), (64, 0.3)])
def test_cayley_orthogonal_det_and_transpose(b, sigma):
    Q = oft_ref.unpack_skew(_rand_q((4,), b, sigma), b)
    R = oft_ref.cayley(Q)
    I = np.eye(b)
    assert np.abs(np.swapaxes(R, -1, -2) @ R - I).max() < 1e-12
    assert np.abs(np.linalg.det(R) - 1.0).max() < 1e-12
    Rm = oft_ref.cayley(-Q)
    assert np.abs(Rm - np.swapaxes(R, -1, -2)).max() < 1e-14
    # I + R = 2 (I - Q)^-1
    assert np.abs(I + R - 2 * np.linalg.inv(I - Q)).max() < 1e-13


def test_cayley_power_series():
    # (I + Q)(I - Q)^-1 = I + 2 sum_{n>=1} Q^n for ||Q|| < 1
    b = 32
    Q = oft_ref.unpack_skew(_rand_q((2,), b, 0.01), b)
    S = np.broadcast_to(np.eye(b), Q.shape).copy()
    P = np.broadcast_to(np.eye(b), Q.shape).copy()
    for _ in range(40):
        P = P @ Q
        S = S + 2 * P
    assert np.abs(oft_ref.cayley(Q) - S).max() < 1e-14


def test_rotation_convention_golden():
    g = _golden()["convention"]
    R = oft_ref.cayley(oft_ref.unpack_skew(np.array([[g["a"]]]), 2))       # [1 block][2][2]
    X = np.array(g["X"])
    W = np.array(g["W_logical_din_by_dout"])
    Y = oft_ref.linear_fwd(X, W.T, (2,), R[None])
    np.testing.assert_allclose(Y, np.array(g["Y"]), rtol=0, atol=1e-15)


def _tiny_case(M=5, K=8, b=4, splits=(3, 2), sigma=0.3):
    X = RNG.normal(size=(M, K))
    Wt = RNG.normal(size=(sum(splits), K))
    qp = _rand_q((len(splits), K // b), b, sigma)
    dY = RNG.normal(size=(M, sum(splits)))
    return X, Wt, qp, dY


def test_forward_q_zero_is_base_gemm():
    spec = LinearSpec("t", M=37, K=128, splits=(64, 80), fmt="int4", group=32, b=32, q_sigma=0.0, seed=3)
    c = linear_np(make_linear_case(spec, q_zero=True))
    X = bf16_bits_to_f64(c["X"])
    Wt = oft_ref.weight_t(c)
    R = oft_ref.rotations(c["Q"].reshape(2, 4, -1), 32)
    assert np.array_equal(oft_ref.linear_fwd(X, Wt, spec.splits, R), X @ Wt.T)


def test_forward_row_norms_preserved():
    X = RNG.normal(size=(50, 256))
    R = oft_ref.cayley(oft_ref.unpack_skew(_rand_q((8,), 32, 0.1), 32))
    Xr = oft_ref.rotate(X, R)
    np.testing.assert_allclose(np.linalg.norm(Xr, axis=1), np.linalg.norm(X, axis=1), rtol=1e-12)
    # and block by block
    np.testing.assert_allclose(np.linalg.norm(Xr.reshape(50, 8, 32), axis=2),
                               np.linalg.norm(X.reshape(50, 8, 32), axis=2), rtol=1e-12)


def test_split_equals_separate_layers():
    X, Wt, qp, _ = _tiny_case(M=6, K=16, b=4, splits=(5, 3, 4))
    R = oft_ref.cayley(oft_ref.unpack_skew(qp, 4))
    Y = oft_ref.linear_fwd(X, Wt, (5, 3, 4), R)
    parts = [oft_ref.linear_fwd(X, Wt[0:5], (5,), R[0:1]),
             oft_ref.linear_fwd(X, Wt[5:8], (3,), R[1:2]),
             oft_ref.linear_fwd(X, Wt[8:12], (4,), R[2:3])]
    assert np.array_equal(Y, np.concatenate(parts, axis=1))


def test_forward_equals_dense_blockdiag():
    # the block-diagonal rotation equals multiplying by the full K x K matrix
    X, Wt, qp, _ = _tiny_case(M=4, K=12, b=4, splits=(7,))
    R = oft_ref.cayley(oft_ref.unpack_skew(qp, 4))[0]
    D = np.zeros((12, 12))
    for j in range(3):
        D[4 * j:4 * j + 4, 4 * j:4 * j + 4] = R[j]
    np.testing.assert_allclose(oft_ref.rotate(X, R), X @ D, rtol=0, atol=1e-14)


def _loss(X, Wt, qp, dY, splits, b):
    R = oft_ref.cayley(oft_ref.unpack_skew(qp, b))
    return float(np.sum(oft_ref.linear_fwd(X, Wt, splits, R) * dY))


def test_backward_finite_differences():
    b, splits = 4, (3, 2)
    X, Wt, qp, dY = _tiny_case(M=3, K=8, b=b, splits=splits, sigma=0.3)
    R = oft_ref.cayley(oft_ref.unpack_skew(qp, b))
    dX, dq = oft_ref.linear_bwd(dY, X, Wt, splits, R, b)
    h = 1e-6
    fdX = np.zeros_like(X)
    for i in np.ndindex(X.shape):
        Xp, Xm = X.copy(), X.copy()
        Xp[i] += h
        Xm[i] -= h
        fdX[i] = (_loss(Xp, Wt, qp, dY, splits, b) - _loss(Xm, Wt, qp, dY, splits, b)) / (2 * h)
    fdq = np.zeros_like(qp)
    for i in np.ndindex(qp.shape):
        qpp, qpm = qp.copy(), qp.copy()
        qpp[i] += h
        qpm[i] -= h
        fdq[i] = (_loss(X, Wt, qpp, dY, splits, b) - _loss(X, Wt, qpm, dY, splits, b)) / (2 * h)
    assert np.abs(dX - fdX).max() <= 1e-7 * np.abs(fdX).max()
    assert np.abs(dq - fdq).max() <= 1e-7 * np.abs(fdq).max()


def test_backward_q_zero_special_case():
    b, splits = 4, (3, 2)
    X, Wt, _, dY = _tiny_case(M=7, K=8, b=b, splits=splits)
    qp = np.zeros((2, 2, b * (b - 1) // 2))
    R = oft_ref.cayley(oft_ref.unpack_skew(qp, b))
    dX, dq, parts = oft_ref.linear_bwd(dY, X, Wt, splits, R, b, return_parts=True)
    iu, ju = np.triu_indices(b, 1)
    for p in range(2):
        G = parts[p]["G"]
        np.testing.assert_allclose(dq[p], 2 * (G[:, iu, ju] - G[:, ju, iu]), rtol=0, atol=1e-13)
    # with R = I the input gradient is the plain dY W
    np.testing.assert_allclose(dX, dY @ Wt, rtol=0, atol=1e-12)


def test_backward_symmetric_g_gives_zero_dq():
    # if X == dX' blockwise-symmetric contributions vanish: choose W, dY so that G is symmetric
    b = 4
    X = RNG.normal(size=(6, 4))
    Wt = np.eye(4)
    dY = X.copy()                         # dX' = dY W^T... = X, G = X^T X symmetric
    R = np.broadcast_to(np.eye(b), (1, 1, b, b))
    _, dq = oft_ref.linear_bwd(dY, X, Wt, (4,), R, b)
    assert np.abs(dq).max() < 1e-12
