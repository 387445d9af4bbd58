"""Pins for the full expert layer of oracle.moe_ref (gate/up, SwiGLU, down
projection with its own OFT rotation): SiLU against closed forms and a library
logistic function; one expert with k = 1 against two chained dense OFT linears of
oracle.oft_ref (themselves pinned); the top-k sum against its per-slot terms."""

import numpy as np
from scipy.special import expit

from oracle import moe_ref, oft_ref
from oracle.codecs import bf16_bits_to_f64
from gen import MoESpec, make_moe_case, make_moe_down
from npcase import raw


def _spec(**kw):
    base = dict(name="l", T=11, K=32, E=5, n_proj=16, top_k=2, chunk=2, group=16, b=8, q_sigma=0.2, seed=21)
    base.update(kw)
    return MoESpec(**base)


def _banks(spec):
    case = make_moe_case(spec)
    down = make_moe_down(spec)
    bank = moe_ref.ExpertBank(raw(case["codes"]), raw(case["scales"]), spec.K, spec.group, spec.n_proj)
    dbank = moe_ref.DownBank(raw(down["down_codes"]), raw(down["down_scales"]), spec.n_proj, spec.group)
    return case, down, bank, dbank


def test_silu_closed_forms():
    x = np.linspace(-40, 40, 2001)
    s = moe_ref.silu(x)
    assert moe_ref.silu(0.0) == 0.0
    np.testing.assert_allclose(s - moe_ref.silu(-x), x, rtol=0, atol=1e-12)   # sigmoid(x) + sigmoid(-x) = 1
    np.testing.assert_allclose(s, x * expit(x), rtol=1e-14, atol=1e-300)
    assert abs(moe_ref.silu(40.0) - 40.0) < 1e-15 and abs(moe_ref.silu(-40.0)) < 1e-15
    assert abs(moe_ref.silu(1.0) - 1.0 / (1.0 + np.exp(-1.0))) < 1e-16


def test_single_expert_layer_is_two_chained_linears():
    spec = _spec(top_k=1)
    case, down, bank, dbank = _banks(spec)
    logits = np.full((spec.T, spec.E), -3.0, dtype=np.float32)
    logits[:, 3] = 3.0
    Y = moe_ref.moe_layer_direct(raw(case["X"]), logits, bank, dbank, raw(case["Q"]), raw(down["Q_down"]),
                                 spec.b, 1)
    X = bf16_bits_to_f64(raw(case["X"]))
    R = oft_ref.rotations(raw(case["Q"])[3], spec.b)
    GU = oft_ref.linear_fwd(X, bank.weight_t(3), (spec.n_proj, spec.n_proj), R)
    n = spec.n_proj
    h = GU[:, :n] * expit(GU[:, :n]) * GU[:, n:]
    Rd = oft_ref.rotations(raw(down["Q_down"])[3][None], spec.b)
    Yl = oft_ref.linear_fwd(h, dbank.weight_t(3), (spec.K,), Rd)
    assert np.abs(Y - Yl).max() <= 1e-12 * np.abs(Yl).max()


def test_layer_is_weighted_sum_of_slot_terms():
    spec = _spec(top_k=3, E=6)
    case, down, bank, dbank = _banks(spec)
    Xb, logits = raw(case["X"]), raw(case["logits"])
    Y = moe_ref.moe_layer_direct(Xb, logits, bank, dbank, raw(case["Q"]), raw(down["Q_down"]), spec.b, spec.top_k)
    idx, w = moe_ref.topk(logits, spec.top_k)
    X = bf16_bits_to_f64(Xb)
    t = 4
    terms = [moe_ref.expert_layer(X[t:t + 1], int(e), bank, dbank, raw(case["Q"])[e], raw(down["Q_down"])[e],
                                  spec.b)[0] for e in idx[t]]
    ref = sum(w[t, k] * terms[k] for k in range(spec.top_k))
    assert np.abs(Y[t] - ref).max() <= 1e-13 * np.abs(ref).max()
    # restricted rows agree with the full computation
    Ys = moe_ref.moe_layer_direct(Xb, logits, bank, dbank, raw(case["Q"]), raw(down["Q_down"]), spec.b,
                                  spec.top_k, tokens=[0, t])
    assert np.array_equal(Ys, Y[[0, t]])
