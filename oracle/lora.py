"""LoRA-wrapped Q/K/V/O projections around radial attention -- plain CPU
reference, fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.

The Radial Attention review (§4.3) adapts a pretrained video DiT to longer
videos by fine-tuning LoRA adapters on the Q/K/V/O projections of its
attention layers, with the radial mask in place of dense attention.  The
pages fix nothing else about the adapters.  Readings taken:

- the standard low-rank update of a frozen projection W (d_out x d_in):
  ``y = x W^T + s (x A^T) B^T`` with trainable A (r x d_in), B (d_out x r)
  and a fixed scale s (alpha / r); no biases;
- hidden size C = H * D, heads split from the channel axis as [B, N, H, D];
- the attention between the projections is Eq.2 of the review under the
  radial mask (``oracle.attention``), scale 1/sqrt(D);
- a fine-tuning step needs dx (the layer below) and dA, dB of all four
  projections; W is frozen, so no dW.

Backward of one LoRA projection (plain matrix calculus of the line above):
    h  = x A^T
    dB = s dy^T h
    dh = s dy B
    dA = dh^T x
    dx = dy W + dh A

``rnd`` (optional) is applied where a device implementation stores a tensor
in a narrower type (the attention inputs q, k, v, its output, and dO), so the
reference sees the same values; the arithmetic stays fp64.
"""

from __future__ import annotations

import numpy as np

from . import attention as _att

PROJ = ("q", "k", "v", "o")


def _as64(x):
    return np.asarray(x, dtype=np.float64)


def lora_linear(x, W, A, B, s):
    """y = x W^T + s (x A^T) B^T over the last axis of x."""
    x, W, A, B = (_as64(t) for t in (x, W, A, B))
    return x @ W.T + s * ((x @ A.T) @ B.T)


def lora_linear_backward(x, W, A, B, s, dy):
    """(dx, dA, dB) of lora_linear for upstream gradient dy; x, dy are 2-D."""
    x, W, A, B, dy = (_as64(t) for t in (x, W, A, B, dy))
    h = x @ A.T
    dB = s * (dy.T @ h)
    dh = s * (dy @ B)
    dA = dh.T @ x
    dx = dy @ W + dh @ A
    return dx, dA, dB


def _heads(t, H):
    """[B, N, C] -> [B, H, N, D]."""
    Bn, N, C = t.shape
    return t.reshape(Bn, N, H, C // H).transpose(0, 2, 1, 3)


def _merge(t):
    """[B, H, N, D] -> [B, N, C]."""
    Bn, H, N, D = t.shape
    return t.transpose(0, 2, 1, 3).reshape(Bn, N, H * D)


def layer_forward(x, params, heads, f, s_tok, sink=True, spec=None, rnd=None):
    """One attention layer: LoRA projections q, k, v -> radial attention ->
    LoRA output projection.  x [B, N, C]; params holds W_p, A_p, B_p for p in
    q, k, v, o and the scale "s".  Returns (y [B, N, C], cache)."""
    r = rnd if rnd is not None else (lambda t: t)
    x = _as64(x)
    Bn, N, C = x.shape
    s = params["s"]
    x2 = x.reshape(Bn * N, C)
    qkv = {}
    for p in ("q", "k", "v"):
        t = lora_linear(x2, params["W_" + p], params["A_" + p], params["B_" + p], s).reshape(Bn, N, C)
        qkv[p] = r(_heads(t, heads))
    O, L = _att.radial_forward(qkv["q"], qkv["k"], qkv["v"], f, s_tok, sink, spec=spec)
    O = r(O)
    a = _merge(O).reshape(Bn * N, C)
    y = lora_linear(a, params["W_o"], params["A_o"], params["B_o"], s).reshape(Bn, N, C)
    cache = {"x2": x2, "a": a, "O": O, "L": L, **qkv}
    return y, cache


def layer_backward(params, cache, dy, heads, f, s_tok, sink=True, spec=None, rnd=None):
    """Gradients of one layer step: dx and dA_p, dB_p for p in q, k, v, o."""
    r = rnd if rnd is not None else (lambda t: t)
    s = params["s"]
    dy = _as64(dy)
    Bn, N, C = dy.shape
    grads = {}
    da, grads["A_o"], grads["B_o"] = lora_linear_backward(cache["a"], params["W_o"], params["A_o"],
                                                          params["B_o"], s, dy.reshape(Bn * N, C))
    dO = r(_heads(da.reshape(Bn, N, C), heads))
    dq, dk, dv = _att.radial_backward(cache["q"], cache["k"], cache["v"], cache["O"], dO, cache["L"],
                                      f, s_tok, sink, spec=spec)
    dx = np.zeros((Bn * N, C))
    for p, g in (("q", dq), ("k", dk), ("v", dv)):
        dxp, grads["A_" + p], grads["B_" + p] = lora_linear_backward(
            cache["x2"], params["W_" + p], params["A_" + p], params["B_" + p], s, _merge(g).reshape(Bn * N, C))
        dx += dxp
    grads["x"] = dx.reshape(Bn, N, C)
    return grads
