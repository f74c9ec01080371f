"""Pins of the LoRA layer reference (oracle.lora) against facts other than its
own formulas: the adapter-free limit, the merged-weight identity of a
low-rank update, and central finite differences of the whole layer step
(projections + radial attention + output projection) for every gradient."""

import numpy as np
import pytest

from oracle import lora as LO
from oracle import mask as M


def _params(rng, C, r, s):
    P = {"s": s}
    for p in LO.PROJ:
        P["W_" + p] = rng.standard_normal((C, C)) / np.sqrt(C)
        P["A_" + p] = rng.standard_normal((r, C)) / np.sqrt(C)
        P["B_" + p] = rng.standard_normal((C, r)) / np.sqrt(r)
    return P


def test_zero_adapter_is_the_frozen_projection():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((7, 12))
    W = rng.standard_normal((9, 12))
    A = rng.standard_normal((3, 12))
    np.testing.assert_array_equal(LO.lora_linear(x, W, A, np.zeros((9, 3)), 0.7), x @ W.T)


def test_low_rank_update_equals_merged_weight():
    # a LoRA projection is the frozen one with W replaced by W + s B A
    rng = np.random.default_rng(1)
    x = rng.standard_normal((11, 16))
    W = rng.standard_normal((10, 16))
    A = rng.standard_normal((4, 16))
    B = rng.standard_normal((10, 4))
    np.testing.assert_allclose(LO.lora_linear(x, W, A, B, 0.25), x @ (W + 0.25 * B @ A).T, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("sink", [True, False])
def test_layer_gradients_match_finite_differences(sink):
    rng = np.random.default_rng(2 + sink)
    heads, D, f, s_tok, r = 2, 4, 3, 4, 2
    C, N = heads * D, f * s_tok
    P = _params(rng, C, r, 0.5)
    x = rng.standard_normal((1, N, C))
    dy = rng.standard_normal((1, N, C))
    y, cache = LO.layer_forward(x, P, heads, f, s_tok, sink)
    g = LO.layer_backward(P, cache, dy, heads, f, s_tok, sink)

    def loss(xx, PP):
        return float(np.sum(LO.layer_forward(xx, PP, heads, f, s_tok, sink)[0] * dy))

    eps = 1e-6
    # dx: a handful of coordinates
    for idx in [(0, 0, 0), (0, N - 1, C - 1), (0, 5, 3), (0, 7, 1)]:
        xp, xm = x.copy(), x.copy()
        xp[idx] += eps
        xm[idx] -= eps
        num = (loss(xp, P) - loss(xm, P)) / (2 * eps)
        assert abs(num - g["x"][idx]) <= 1e-6 * max(1.0, abs(num)), ("x", idx, num, g["x"][idx])
    # every adapter gradient, a few entries each
    for key in [k for k in g if k != "x"]:
        shape = P[key].shape
        for idx in [(0, 0), (shape[0] - 1, shape[1] - 1), (shape[0] // 2, shape[1] // 2)]:
            Pp = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in P.items()}
            Pm = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in P.items()}
            Pp[key][idx] += eps
            Pm[key][idx] -= eps
            num = (loss(x, Pp) - loss(x, Pm)) / (2 * eps)
            assert abs(num - g[key][idx]) <= 1e-6 * max(1.0, abs(num)), (key, idx, num, g[key][idx])


def test_layer_attention_is_the_masked_attention_of_the_projections():
    # with identity projections and zero adapters the layer is the attention
    # itself followed by the identity: compare against a direct masked softmax
    rng = np.random.default_rng(5)
    heads, D, f, s_tok = 1, 4, 2, 4
    C, N = heads * D, f * s_tok
    P = {"s": 1.0}
    for p in LO.PROJ:
        P["W_" + p] = np.eye(C)
        P["A_" + p] = np.zeros((1, C))
        P["B_" + p] = np.zeros((C, 1))
    x = rng.standard_normal((1, N, C))
    y, _ = LO.layer_forward(x, P, heads, f, s_tok, True)
    allowed = M.token_mask(f, s_tok, True)
    S = (x[0] @ x[0].T) / np.sqrt(D)
    S = np.where(allowed, S, -np.inf)
    Pm = np.exp(S - S.max(axis=1, keepdims=True))
    Pm /= Pm.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(y[0], Pm @ x[0], rtol=1e-12, atol=1e-12)
