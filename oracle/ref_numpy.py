"""Second, independent fp64 oracle in numpy: dense masked matrices, tiny sizes.

TEST INFRASTRUCTURE ONLY (imported by tests, never by the product library).

It is written differently from ``swat_oracle.c`` on purpose, so that the two
can check each other:

* the mask is built the way the "Sliding Window Attention" glossary builds it
  in its PyTorch sample (section "How the window grows with depth"): an
  ``offset = i - j`` matrix and ``(offset >= 0) & (offset < window)``; sinks
  (the SWA(w, s) page: the first s tokens are kept besides the window) are
  OR-ed in as extra columns;
* RoPE is the RoFormer definition in complex form: the pair
  (x[2t], x[2t+1]) is the complex number x[2t] + i x[2t+1], multiplied by
  exp(i * m * theta_t), theta_t = base^(-2t/d);
* scores are one dense matrix product; the activation acts on the whole
  matrix (sigmoid element-wise, softmax per row over the mask).

The backward (``swat_bwd``) is the analytic chain rule on the same dense
matrices, so that it and the C oracle's backward (and finite differences of
either forward) check one another. It takes an optional ``operand_round``
hook applied to the four matrices a bf16 tensor-core backward must hold in
bf16 as matrix-product operands (rotated Q and K, P, dS); with the hook left
out every step is fp64.
"""
from __future__ import annotations

import numpy as np


def mask_matrix(N: int, window: int, n_sink: int = 0) -> np.ndarray:
    pos = np.arange(N)
    offset = pos[:, None] - pos[None, :]
    m = (offset >= 0) & (offset < window)
    if n_sink > 0:
        sink_cols = (pos[None, :] < n_sink) & (offset >= 0)
        m = m | sink_cols
    return m


def rope_complex(x: np.ndarray, positions: np.ndarray, rope_base: float) -> np.ndarray:
    """x [..., N, d] with positions [N]; returns the rotated copy (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    if not rope_base > 0:
        return x.copy()
    d = x.shape[-1]
    t = np.arange(d // 2, dtype=np.float64)
    theta = rope_base ** (-2.0 * t / d)
    ang = positions.astype(np.float64)[:, None] * theta[None, :]
    z = x[..., 0::2] + 1j * x[..., 1::2]
    z = z * np.exp(1j * ang)
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def swat_fwd(q, k, v, *, window: int, n_sink: int = 0, mode: int = 0, slopes=None,
             rope_base: float = 10000.0):
    """q [B,N,H,d], k/v [B,N,Hkv,d] -> o [B,N,H,d], lse [B,H,N] (fp64).

    Inputs are used at full fp64 precision as given (finite-difference checks
    perturb them in fp64); pass fp32 values to compare with the C oracle.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    G = H // Hkv
    pos = np.arange(N)
    mask = mask_matrix(N, window, n_sink)
    dist = (pos[:, None] - pos[None, :]).astype(np.float64)
    o = np.zeros((B, N, H, d))
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            qh = rope_complex(q[b, :, h, :], pos, rope_base)
            kh = rope_complex(k[b, :, h // G, :], pos, rope_base)
            vh = v[b, :, h // G, :]
            slope = 0.0 if slopes is None else float(slopes[h])
            s = qh @ kh.T / np.sqrt(d) + slope * dist
            if mode == 0:
                p = np.where(mask, 1.0 / (1.0 + np.exp(-s)), 0.0)
            else:
                s_m = np.where(mask, s, -np.inf)
                mx = s_m.max(axis=1, keepdims=True)
                e = np.exp(s_m - mx)
                den = e.sum(axis=1, keepdims=True)
                p = e / den
                lse[b, h] = (mx + np.log(den))[:, 0]
            o[b, :, h, :] = p @ vh
    return o, lse


def swat_bwd(q, k, v, dout, *, window: int, n_sink: int = 0, mode: int = 0, slopes=None,
             rope_base: float = 10000.0, operand_round=None):
    """Gradients dq [B,N,H,d], dk/dv [B,N,Hkv,d] (fp64) of sum(o * dout).

    Chain rule of the attention equation ("SWAT: Sliding Window Attention
    Training", section "Balanced ALiBi"; softmax form from the SWA(w, s)
    page): with s = q'k'^T/sqrt(d) + slope*(i-j) and p = act(s) on the mask,
    dv = p^T dout, dp = dout v^T, ds = dp * p(1-p) (sigmoid) or
    p (dp - rowsum(p dp)) (softmax), dq' = ds k'/sqrt(d), dk' = ds^T q'/sqrt(d),
    and dq, dk rotate dq', dk' back by -position.
    """
    rnd = operand_round if operand_round is not None else (lambda x: x)
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    G = H // Hkv
    pos = np.arange(N)
    mask = mask_matrix(N, window, n_sink)
    dist = (pos[:, None] - pos[None, :]).astype(np.float64)
    sc = 1.0 / np.sqrt(d)
    dq = np.zeros((B, N, H, d))
    dk = np.zeros((B, N, Hkv, d))
    dv = np.zeros((B, N, Hkv, d))
    for b in range(B):
        for h in range(H):
            kvh = h // G
            qh = rnd(rope_complex(q[b, :, h, :], pos, rope_base))
            kh = rnd(rope_complex(k[b, :, kvh, :], pos, rope_base))
            vh = v[b, :, kvh, :]
            doh = dout[b, :, h, :]
            slope = 0.0 if slopes is None else float(slopes[h])
            s = qh @ kh.T * sc + slope * dist
            if mode == 0:
                p = np.where(mask, 1.0 / (1.0 + np.exp(-s)), 0.0)
            else:
                s_m = np.where(mask, s, -np.inf)
                e = np.exp(s_m - s_m.max(axis=1, keepdims=True))
                p = e / e.sum(axis=1, keepdims=True)
            dp = doh @ vh.T
            if mode == 0:
                ds = dp * p * (1.0 - p)
            else:
                ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            ds = rnd(ds * sc)
            dv[b, :, kvh, :] += rnd(p).T @ doh
            dq[b, :, h, :] = rope_complex(ds @ kh, -pos, rope_base)
            dk[b, :, kvh, :] += rope_complex(ds.T @ qh, -pos, rope_base)
    return dq, dk, dv
