"""fp64 oracle of the short causal convolution ahead of the GDN recurrence.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Qwen3.8-Flash-Next summary (picx.dev), "Methodology", "1. GDN Hybrid Token Mixing":
the GDN layers use "short causal convolutions" for local inductive bias.  The page
gives neither the width nor the form, so this module takes these readings:

* depthwise: every channel c of q, k and v (each laid out [T, C], C = H * d) has
  its own W taps w[c, 0..W-1]; no bias;
* causal: the output at token t mixes the inputs at t - W + 1 .. t only,

      y[t, c] = act( sum_{i=0}^{W-1} w[c, i] * x[t - (W - 1) + i, c] ),

  so tap W - 1 weighs the current token;
* act is the identity (the page names no activation) or, on request, SiLU
  (x * sigmoid(x), the activation of the published Gated DeltaNet layer);
* documents are independent: inputs before a document's first token come from
  that document's conv state, state[n, j, c] = the input at position
  start_n - (W - 1) + j (zero when no state is given), and the state after the
  document holds its last W - 1 inputs (taken from the initial state where the
  document is shorter than W - 1);
* one decode step is the same with one token per sequence, the state updated.

Each output is the plain sum above, written as a loop over taps.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def silu(x):
    x = _f64(x)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def short_conv_varlen(x, w, cu_seqlens, state=None, activation="none"):
    """x [T, C]; w [C, W]; cu_seqlens [N+1]; state [N, W-1, C] or None (zero).

    Returns (y [T, C], final_state [N, W-1, C]) in float64."""
    x, w = _f64(x), _f64(w)
    T, C = x.shape
    W = w.shape[1]
    assert w.shape == (C, W) and W >= 1
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    N = len(cu) - 1
    assert cu[0] == 0 and cu[-1] == T
    st = np.zeros((N, W - 1, C)) if state is None else _f64(state)
    assert st.shape == (N, W - 1, C)
    y = np.zeros((T, C))
    final = np.zeros((N, W - 1, C))
    for n in range(N):
        a, b = cu[n], cu[n + 1]
        # the document's inputs, preceded by its W - 1 state rows (positions a - W + 1 .. a - 1)
        ext = np.concatenate([st[n], x[a:b]], axis=0)
        for t in range(b - a):
            acc = np.zeros(C)
            for i in range(W):
                acc += w[:, i] * ext[t + i]
            y[a + t] = acc
        final[n] = ext[ext.shape[0] - (W - 1):] if W > 1 else final[n]
    if activation == "silu":
        y = silu(y)
    elif activation != "none":
        raise ValueError(activation)
    return y, final


def short_conv_step(x, w, state, activation="none"):
    """One token per sequence: x [N, C], state [N, W-1, C].  Returns (y [N, C], new_state)."""
    x = _f64(x)
    N = x.shape[0]
    return short_conv_varlen(x, w, np.arange(N + 1), state, activation)
