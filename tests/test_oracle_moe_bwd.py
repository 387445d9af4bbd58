"""Pins for oracle.moe_ref.moe_bwd_direct (the MoE adapter backward).

The backward is checked against things it does not compute itself: central
finite differences of the float64 forward (for dX, the packed Q of every
selected expert, and the router logits), the dense split-projection backward
that one expert with k = 1 reduces to, and the inner products <dY[t], Y_tk>
of the forward's own per-slot outputs.
"""

import numpy as np

from oracle import moe_ref, oft_ref
from oracle.codecs import bf16_bits_to_f64
from gen import MoESpec, make_moe_case, make_moe_grad
from npcase import raw


def _tiny(**kw):
    base = dict(name="tiny", T=5, K=8, E=6, n_proj=3, top_k=2, chunk=2, group=4, b=4, q_sigma=0.3, seed=11)
    base.update(kw)
    return MoESpec(**base)


def _setup(spec):
    case = make_moe_case(spec)
    bank = moe_ref.ExpertBank(raw(case["codes"]), raw(case["scales"]), spec.K, spec.group, spec.n_proj)
    dY = bf16_bits_to_f64(raw(make_moe_grad(spec)))
    return case, bank, dY


def _loss(spec, bank, dY, X, qvals, lg, idx):
    """<dY, Y> for the float64 forward with the selection `idx` held fixed."""
    L = 0.0
    for t in range(spec.T):
        sel = lg[t, idx[t]]
        z = np.exp(sel - sel.max())
        w = z / z.sum()
        for k in range(spec.top_k):
            e = int(idx[t, k])
            R = oft_ref.rotations(qvals[e], spec.b, is_bits=False)
            L += w[k] * (dY[t] @ moe_ref.expert_outputs(X[t:t + 1], e, bank, None, spec.b, R=R)[0])
    return L


def test_backward_matches_finite_differences():
    spec = _tiny()
    case, bank, dY = _setup(spec)
    Xb, logits, Qb = raw(case["X"]), raw(case["logits"]), raw(case["Q"])
    dX, dq, dlog, _ = moe_ref.moe_bwd_direct(dY, Xb, logits, bank, Qb, spec.b, spec.top_k, spec.E)
    X = bf16_bits_to_f64(Xb)
    q = bf16_bits_to_f64(Qb)
    lg = logits.astype(np.float64)
    idx, _ = moe_ref.topk(logits, spec.top_k)
    h = 1e-6

    def fd(arr, pos):
        a0 = arr[pos]
        arr[pos] = a0 + h
        lp = _loss(spec, bank, dY, X, q, lg, idx)
        arr[pos] = a0 - h
        lm = _loss(spec, bank, dY, X, q, lg, idx)
        arr[pos] = a0
        return (lp - lm) / (2 * h)

    num_dX = np.array([[fd(X, (t, c)) for c in range(spec.K)] for t in range(spec.T)])
    assert np.abs(num_dX - dX).max() <= 1e-7 * np.abs(dX).max()
    active = sorted(set(idx.reshape(-1).tolist()))
    assert len(active) >= 3
    for e in range(spec.E):
        if e not in active:
            assert not dq[e].any()
            continue
        num = np.zeros_like(dq[e])
        for pos in np.ndindex(*dq[e].shape):
            num[pos] = fd(q, (e,) + pos)
        assert np.abs(num - dq[e]).max() <= 1e-7 * np.abs(dq).max()
    for t in range(spec.T):
        for e in range(spec.E):
            g = fd(lg, (t, e)) if e in idx[t] else 0.0
            assert abs(g - dlog[t, e]) <= 1e-7 * np.abs(dlog).max()


def test_dw_is_inner_product_with_slot_outputs():
    spec = _tiny(T=7, K=16, E=5, n_proj=4, top_k=3, b=8)
    case, bank, dY = _setup(spec)
    Xb, logits, Qb = raw(case["X"]), raw(case["logits"]), raw(case["Q"])
    _, _, dlog, dw = moe_ref.moe_bwd_direct(dY, Xb, logits, bank, Qb, spec.b, spec.top_k, spec.E)
    X = bf16_bits_to_f64(Xb)
    idx, _ = moe_ref.topk(logits, spec.top_k)
    for t in range(spec.T):
        for k in range(spec.top_k):
            e = int(idx[t, k])
            ytk = moe_ref.expert_outputs(X[t:t + 1], e, bank, Qb[e], spec.b)[0]
            assert abs(dw[t, k] - dY[t] @ ytk) <= 1e-12 * np.abs(dw).max()
    # softmax over the selected logits is shift-invariant: each row sums to zero
    assert np.abs(dlog.sum(axis=1)).max() <= 1e-12 * np.abs(dlog).max()


def test_single_expert_reduces_to_split_linear_backward():
    spec = _tiny(T=9, K=16, E=4, n_proj=5, top_k=1, b=8)
    case, bank, dY = _setup(spec)
    logits = np.full((spec.T, spec.E), -4.0, dtype=np.float32)
    logits[:, 1] = 4.0
    Xb, Qb = raw(case["X"]), raw(case["Q"])
    dX, dq, dlog, _ = moe_ref.moe_bwd_direct(dY, Xb, logits, bank, Qb, spec.b, 1, spec.E)
    X = bf16_bits_to_f64(Xb)
    R = oft_ref.rotations(Qb[1], spec.b)
    dXl, dql = oft_ref.linear_bwd(dY, X, bank.weight_t(1), (spec.n_proj, spec.n_proj), R, spec.b)
    assert np.abs(dX - dXl).max() <= 1e-12 * np.abs(dXl).max()
    assert np.abs(dq[1] - dql).max() <= 1e-12 * np.abs(dql).max()
    assert not dq[[0, 2, 3]].any()
    assert not dlog.any()


def test_token_subset_gives_the_same_rows_and_complete_experts():
    spec = _tiny(T=12, K=16, E=7, n_proj=4, top_k=2, b=8)
    case, bank, dY = _setup(spec)
    Xb, logits, Qb = raw(case["X"]), raw(case["logits"]), raw(case["Q"])
    full = moe_ref.moe_bwd_direct(dY, Xb, logits, bank, Qb, spec.b, spec.top_k, spec.E)
    idx, _ = moe_ref.topk(logits, spec.top_k)
    e = int(idx[3, 0])
    toks = sorted(set(np.nonzero((idx == e).any(axis=1))[0].tolist()) | {0, 5})
    part = moe_ref.moe_bwd_direct(dY, Xb, logits, bank, Qb, spec.b, spec.top_k, spec.E, tokens=toks)
    for a, b in zip(full, part):
        if a.shape[0] == spec.T:
            assert np.array_equal(a[toks], b[toks])
    assert np.abs(full[1][e] - part[1][e]).max() <= 1e-13 * np.abs(full[1][e]).max()


def test_expert_dq_equals_the_full_backward():
    """expert_dq, which works from one expert's routed entries only, gives the same dq
    as the token-by-token full backward, for heavily and lightly loaded experts."""
    spec = MoESpec("edq", T=60, K=64, E=7, n_proj=16, top_k=3, chunk=3, group=32, b=16, q_sigma=0.1, seed=12)
    case = make_moe_case(spec)
    bank = moe_ref.ExpertBank(raw(case["codes"]), raw(case["scales"]), spec.K, spec.group, spec.n_proj)
    rng = np.random.default_rng(3)
    dY = rng.standard_normal((spec.T, 2 * spec.n_proj))
    logits = raw(case["logits"])
    _, dq, _, _ = moe_ref.moe_bwd_direct(dY, raw(case["X"]), logits, bank, raw(case["Q"]), spec.b, spec.top_k,
                                         spec.E)
    idx, _ = moe_ref.topk(logits, spec.top_k)
    counts = np.bincount(idx.reshape(-1), minlength=spec.E)
    for e in range(spec.E):
        got = moe_ref.expert_dq(e, dY, raw(case["X"]), logits, bank, raw(case["Q"]), spec.b, spec.top_k)
        scale = max(np.abs(dq[e]).max(), 1e-300)
        assert np.abs(got - dq[e]).max() <= 1e-12 * scale, e
        assert (counts[e] == 0) == (not got.any())
