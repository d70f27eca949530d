"""Attention over the compressed cache (oracle side, float64).

Test infrastructure only; see oracle/__init__.py. The JoLT pages do not describe an attention
kernel; they compress the cache that attention reads (Abstract; news summary, "Two details"
paragraph, for the cache structure). This module states what attention over a JoLT stream
computes, so that a kernel reading the stream directly can be checked:

* the plain definition: with K_hat, V_hat the float64 reconstructions of one layer's K and V
  (G x2 U_T x3 U_D plus the dequantised residual rotated back, no output rounding), query head
  j of Hq reads KV head h = j // (Hq / H) (grouped-query attention; Hq = H is multi-head) and
      O[j, i] = softmax_t(scale * Q[j, i] . K_hat[h, t]) V_hat[h]   over the T tokens;
* the factored form (the reading taken for a kernel that never rebuilds K_hat or V_hat): by
  linearity of the reconstruction,
      Q[j, i] . K_hat[h, t] = U_T[t] (G_h (U_D^T q)) + s_t Y_hat[h, t] (Pi^T q),
      sum_t p_t V_hat[h, t] = ((p^T U_T) G_h) U_D^T + ((p * s)^T Y_hat[h]) Pi^T,
  where s_t is the row scale and Y_hat the unit-scale cell centres (2 c + 1 - 2^b) / 2^b.
The two forms agree up to rounding order; a test pins the second against the first.
"""
from __future__ import annotations

import numpy as np

from .jolt import KINDS, decode_lt, dequantize_rows
from .numerics import rotation_matrix


def kv_head_of(j: int, Hq: int, H: int) -> int:
    """KV head read by query head j (Hq a multiple of H)."""
    return j // (Hq // H)


def softmax_rows(S):
    """Row-wise softmax, max-shifted."""
    S = S - S.max(axis=-1, keepdims=True)
    E = np.exp(S)
    return E / E.sum(axis=-1, keepdims=True)


def attention_dense(Q, K_hat, V_hat, scale: float):
    """The plain definition. Q [Hq][n][D]; K_hat, V_hat [H][T][D] float64. Returns [Hq][n][D]."""
    Hq, H = Q.shape[0], K_hat.shape[0]
    out = np.empty(Q.shape, dtype=np.float64)
    for j in range(Hq):
        h = kv_head_of(j, Hq, H)
        P = softmax_rows(scale * (Q[j] @ K_hat[h].T))
        out[j] = P @ V_hat[h]
    return out


def attention_over_stream(st, layer: int, Q, scale: float, Pi=None):
    """The plain definition on one layer of an oracle stream: K_hat, V_hat rebuilt in float64."""
    if Pi is None:
        Pi = rotation_matrix(st.seed, st.D, st.rotation)
    K_hat = decode_lt(st, layer * KINDS + 0, Pi)
    V_hat = decode_lt(st, layer * KINDS + 1, Pi)
    return attention_dense(np.asarray(Q, dtype=np.float64), K_hat, V_hat, scale)


def _lt_parts(c, H, T, D):
    """(U_T, G, U_D, scales, unit cell centres) of one layer-tensor, zero-sized when absent."""
    if c.b > 0:
        Yh = dequantize_rows(np.ones_like(c.scales), c.codes, c.b)      # unit-scale centres
        s = c.scales
    else:
        Yh = np.zeros((H, T, D))
        s = np.zeros((H, T))
    return c.U_T, c.G, c.U_D, s, Yh


def attention_factored(st, layer: int, Q, scale: float, Pi=None):
    """The factored form on one layer of an oracle stream (no K_hat or V_hat is formed)."""
    if Pi is None:
        Pi = rotation_matrix(st.seed, st.D, st.rotation)
    Q = np.asarray(Q, dtype=np.float64)
    Hq, n, D = Q.shape
    H, T = st.H, st.T
    UTk, Gk, UDk, sk, Yk = _lt_parts(st.lts[layer * KINDS + 0], H, T, D)
    UTv, Gv, UDv, sv, Yv = _lt_parts(st.lts[layer * KINDS + 1], H, T, D)
    out = np.empty(Q.shape, dtype=np.float64)
    for j in range(Hq):
        h = kv_head_of(j, Hq, H)
        q = Q[j]                                             # n x D
        qhat = (q @ UDk) @ Gk[h].T                           # n x r_t: G_h (U_D^T q)
        qpi = q @ Pi                                         # n x D: Pi^T q
        S = qhat @ UTk.T + (qpi @ Yk[h].T) * sk[h][None, :]  # n x T scores
        P = np.exp(scale * S - (scale * S).max(axis=1, keepdims=True))
        P = P / P.sum(axis=1, keepdims=True)
        tucker = ((P @ UTv) @ Gv[h]) @ UDv.T                 # n x D
        resid = ((P * sv[h][None, :]) @ Yv[h]) @ Pi.T        # n x D
        out[j] = tucker + resid
    return out
