"""Pins for oracle.moe_ref: top-k + gating, bucketing, chunking, chunked forward."""

import numpy as np

from oracle import moe_ref, oft_ref
from oracle.codecs import bf16_bits_to_f64
from gen import MoESpec, make_moe_case, make_moe_router
from npcase import raw


def _small_spec(**kw):
    base = dict(name="m", T=40, K=64, E=12, n_proj=24, top_k=3, chunk=4, group=32, b=16, q_sigma=0.05, seed=5)
    base.update(kw)
    return MoESpec(**base)


def test_topk_matches_brute_force_with_ties():
    rng = np.random.default_rng(0)
    logits = rng.integers(-3, 4, size=(200, 10)).astype(np.float32)   # many ties
    idx, w = moe_ref.topk(logits, 4)
    for t in range(200):
        ref = sorted(range(10), key=lambda e: (-float(logits[t, e]), e))[:4]
        assert list(idx[t]) == ref
        z = np.exp(logits[t, ref].astype(np.float64) - logits[t, ref].max())
        np.testing.assert_allclose(w[t], z / z.sum(), rtol=1e-15)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-15)


def test_topk_non_finite_logits():
    """A diverging router: NaN ranks as -inf (ties to the lower id), every index is a
    real expert, and the weights are the softmax's limits: +inf entries share the
    weight, an all -inf / NaN selection is uniform."""
    nan, inf = np.float32(np.nan), np.float32(np.inf)
    rng = np.random.default_rng(4)
    E, k = 9, 4
    rows = [
        [nan] * E,                                             # all NaN
        [-inf] * E,                                            # all -inf
        [nan, -inf, 0.5, nan, -inf, nan, nan, nan, nan],       # one finite value
        [nan, 1.0, inf, 2.0, inf, nan, -inf, 0.0, 3.0],        # two +inf
        [-1.0, nan, -2.0, -3.0, -inf, nan, -0.5, nan, -inf],   # finite values mixed with NaN and -inf
        [nan, nan, 2.0, 2.0, nan, 2.0, -inf, 2.0, 2.0],        # ties among finite values
    ]
    rows += [list(np.where(rng.random(E) < 0.3, nan, rng.integers(-2, 3, E)).astype(np.float32))
             for _ in range(40)]
    logits = np.array(rows, dtype=np.float32)
    idx, w = moe_ref.topk(logits, k)
    for t in range(len(rows)):
        key = [(-np.inf if np.isnan(x) else float(x)) for x in logits[t]]
        ref = sorted(range(E), key=lambda e: (-key[e], e))[:k]
        assert list(idx[t]) == ref
        assert np.all((idx[t] >= 0) & (idx[t] < E))
        sel = np.array([key[e] for e in ref])
        if sel.max() == np.inf:
            want = (sel == np.inf) / np.sum(sel == np.inf)
        elif sel.max() == -np.inf:
            want = np.full(k, 1.0 / k)
        else:
            z = np.exp(sel - sel.max())
            want = z / z.sum()
        np.testing.assert_allclose(w[t], want, rtol=1e-15, atol=0)
        assert abs(w[t].sum() - 1.0) < 1e-15 and np.all(np.isfinite(w[t]))
    # closed forms of the special rows
    assert list(idx[0]) == [0, 1, 2, 3] and np.all(w[0] == 0.25)
    assert list(idx[1]) == [0, 1, 2, 3] and np.all(w[1] == 0.25)
    assert list(idx[2]) == [2, 0, 1, 3] and list(w[2]) == [1.0, 0.0, 0.0, 0.0]
    assert list(idx[3]) == [2, 4, 8, 3] and list(w[3]) == [0.5, 0.5, 0.0, 0.0]


def test_buckets_match_dictionary_build():
    rng = np.random.default_rng(1)
    T, k, E = 300, 4, 17
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    counts, offsets, bucket = moe_ref.buckets(idx, E)
    d = {e: [] for e in range(E)}
    for t in range(T):
        for s in range(k):
            d[int(idx[t, s])].append(t * k + s)
    flat = [x for e in range(E) for x in d[e]]
    assert list(bucket) == flat
    assert [len(d[e]) for e in range(E)] == list(counts)
    assert offsets[0] == 0 and offsets[-1] == T * k


def test_chunk_table():
    counts = np.array([0, 3, 0, 1, 5, 0, 2, 2, 0, 1])
    n, table = moe_ref.chunk_table(counts, 3, 10)
    assert n == 6
    assert table.tolist() == [[1, 3, 4], [6, 7, 9], [-1, -1, -1], [-1, -1, -1]]


def test_chunked_equals_direct():
    spec = _small_spec()
    case = make_moe_case(spec)
    bank = moe_ref.ExpertBank(raw(case["codes"]), raw(case["scales"]), spec.K, spec.group, spec.n_proj)
    Yc, routing = moe_ref.moe_fwd_chunked(raw(case["X"]), raw(case["logits"]), bank, raw(case["Q"]), spec.b,
                                          spec.top_k, spec.chunk, spec.E)
    Yd = moe_ref.moe_fwd_direct(raw(case["X"]), raw(case["logits"]), bank, raw(case["Q"]), spec.b, spec.top_k)
    assert np.abs(Yc - Yd).max() <= 1e-12 * np.abs(Yd).max()
    # sampled columns/tokens agree with the full computation
    toks, cols = np.array([0, 7, 39]), np.array([1, 5, 23, 24, 40])
    Ys = moe_ref.moe_fwd_direct(raw(case["X"]), raw(case["logits"]), bank, raw(case["Q"]), spec.b, spec.top_k,
                                tokens=toks, cols=cols)
    assert np.abs(Ys - Yd[toks][:, cols]).max() <= 1e-12 * np.abs(Yd).max()


def test_single_expert_reduces_to_split_linear():
    # every token routed to expert 2 with k = 1 (weight 1): the layer is the
    # split-projection linear with splits (gate, up) and the expert's rotations
    spec = _small_spec(top_k=1)
    case = make_moe_case(spec)
    logits = np.full((spec.T, spec.E), -5.0, dtype=np.float32)
    logits[:, 2] = 5.0
    bank = moe_ref.ExpertBank(raw(case["codes"]), raw(case["scales"]), spec.K, spec.group, spec.n_proj)
    Y, routing = moe_ref.moe_fwd_chunked(raw(case["X"]), logits, bank, raw(case["Q"]), spec.b, 1, spec.chunk,
                                         spec.E)
    assert routing["n_active"] == 1
    X = bf16_bits_to_f64(raw(case["X"]))
    R = oft_ref.rotations(raw(case["Q"])[2], spec.b)
    Yl = oft_ref.linear_fwd(X, bank.weight_t(2), (spec.n_proj, spec.n_proj), R)
    assert np.abs(Y - Yl).max() <= 1e-13 * np.abs(Yl).max()


def test_zipf_router_is_skewed():
    spec = MoESpec("z", T=4096, K=64, E=384, n_proj=8, top_k=8, chunk=16, group=32, b=32, q_sigma=0.01, seed=3)
    logits = make_moe_router(spec).numpy()
    idx, _ = moe_ref.topk(logits, 8)
    counts, _, _ = moe_ref.buckets(idx, spec.E)
    n_active = int((counts > 0).sum())
    # heavy head, many idle experts: the structure the chunked path must handle
    assert counts.max() > 1000 and 50 < n_active < 384
    assert int(np.median(counts)) <= 2
