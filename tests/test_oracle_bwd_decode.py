"""Oracle backward (finite differences) and ring-cache decode pins."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import ref_numpy
from sliding_window_sigmoid_b200 import inputs


def _loss(q, k, v, dout, **kw):
    o, _ = ref_numpy.swat_fwd(q, k, v, **kw)
    return float((o * dout).sum())


# The pages print no backward; it is pinned here by central finite differences
# of the independent numpy forward (fp64, h = 1e-6), for both activations,
# grouped KV heads, sinks and windows 1, 3 and N+2.
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("Hkv", [1, 2])
@pytest.mark.parametrize("w,s", [(1, 0), (3, 2), (12, 0)])
def test_bwd_matches_finite_differences(mode, Hkv, w, s):
    B, N, H, d = 1, 10, 2, 8
    q, k, v, do = [t.numpy().astype(np.float64)
                   for t in inputs.qkv(B, N, H, Hkv, d, seed=21, dtype=torch.float32, with_dout=True)]
    sl = inputs.balanced_alibi_slopes(H).numpy().astype(np.float64)
    kw = dict(window=w, n_sink=s, mode=mode, slopes=sl, rope_base=1e4)
    dq, dk, dv = oracle.swat_bwd(q, k, v, do, **kw)
    h = 1e-6
    rng = np.random.default_rng(0)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        flat = x.reshape(-1)
        idxs = rng.choice(flat.size, size=min(40, flat.size), replace=False)
        for ix in idxs:
            old = flat[ix]
            flat[ix] = old + h
            lp = _loss(q, k, v, do, **kw)
            flat[ix] = old - h
            lm = _loss(q, k, v, do, **kw)
            flat[ix] = old
            fd = (lp - lm) / (2 * h)
            an = g.reshape(-1)[ix]
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (name, ix, fd, an)


def test_bwd_sigmoid_zero_qk_dv_closed_form():
    # Q = K = 0, slopes 0: every p is 1/2, so dV_j = 1/2 * sum_{i : j in keys(i)} dO_i.
    B, N, H, d, w = 1, 15, 2, 4, 4
    q = np.zeros((B, N, H, d), np.float32)
    k = np.zeros((B, N, 1, d), np.float32)
    v = np.ones((B, N, 1, d), np.float32)
    do = inputs.normal((B, N, H, d), 3, dtype=torch.float32).numpy()
    _, _, dv = oracle.swat_bwd(q, k, v, do, window=w, rope_base=1e4)
    for j in range(N):
        ref = 0.5 * sum(do[0, i, h].astype(np.float64) for h in range(H) for i in range(j, min(N, j + w)))
        np.testing.assert_allclose(dv[0, j, 0], ref, atol=1e-12)


def test_bwd_sampled_rows_equal_full():
    B, N, H, Hkv, d = 2, 30, 4, 2, 8
    q, k, v, do = [t.numpy() for t in inputs.qkv(B, N, H, Hkv, d, seed=9, dtype=torch.float32,
                                                 with_dout=True)]
    sl = inputs.balanced_alibi_slopes(H).numpy()
    for mode, s in ((0, 0), (1, 2)):
        kw = dict(window=6, n_sink=s, mode=mode, slopes=sl, rope_base=1e4)
        dq, dk, dv = oracle.swat_bwd(q, k, v, do, **kw)
        qrows = np.array([[0, 0, 0], [1, 3, 29], [0, 2, 11]])
        krows = np.array([[0, 0, 0], [1, 1, 29], [1, 0, 5], [0, 1, 1]])
        dqr, dkr, dvr = oracle.swat_bwd_rows(q, k, v, do, qrows, krows, **kw)
        for r, (b, h, i) in enumerate(qrows):
            np.testing.assert_allclose(dqr[r], dq[b, i, h], atol=1e-13)
        for r, (b, kh, j) in enumerate(krows):
            np.testing.assert_allclose(dkr[r], dk[b, j, kh], atol=1e-13)
            np.testing.assert_allclose(dvr[r], dv[b, j, kh], atol=1e-13)


# ---------------------------------------------------------------------------
# Ring cache: glossary ring-buffer paragraph (slot = i mod w, oldest overwritten)
# ---------------------------------------------------------------------------

def test_ring_state_is_direct_scatter():
    B, Hkv, d, w, s, base = 2, 2, 8, 5, 2, 1e4
    n_tok = 13
    k = inputs.normal((B, n_tok, Hkv, d), 1, dtype=torch.float32).numpy()
    v = inputs.normal((B, n_tok, Hkv, d), 2, dtype=torch.float32).numpy()
    rc = oracle.RingCache(B, Hkv, d, w, s, base)
    rc.fill(k, v, 0)
    for b in range(B):
        for kh in range(Hkv):
            # the last w positions, each in slot pos mod w, rotated at its absolute position
            for p in range(n_tok - w, n_tok):
                slot = p % w
                np.testing.assert_allclose(rc.kc[b, kh, slot], oracle.rope_rotate(k[b, p, kh], p, base),
                                           atol=1e-14)
                np.testing.assert_array_equal(rc.vc[b, kh, slot], v[b, p, kh].astype(np.float64))
            for p in range(s):
                np.testing.assert_allclose(rc.ks[b, kh, p], oracle.rope_rotate(k[b, p, kh], p, base),
                                           atol=1e-14)


@pytest.mark.parametrize("mode,w,s", [(0, 4, 0), (1, 4, 2), (0, 7, 3), (1, 1, 0), (0, 64, 0)])
def test_decode_equals_forward_row(mode, w, s):
    # A decode step at position p over the cache equals row p of the forward
    # over the same tokens: from p = 0 (partial ring) through several wraps.
    B, H, Hkv, d, N, base = 2, 4, 2, 8, 19, 1e4
    q, k, v = [t.numpy() for t in inputs.qkv(B, N, H, Hkv, d, seed=31, dtype=torch.float32)]
    sl = inputs.balanced_alibi_slopes(H).numpy() if mode == 0 else None
    o_ref, _ = oracle.swat_fwd(q, k, v, window=w, n_sink=s, mode=mode, slopes=sl, rope_base=base)
    rc = oracle.RingCache(B, Hkv, d, w, s, base)
    for p in range(N):
        o = rc.step(q[:, p], k[:, p], v[:, p], np.full(B, p), mode=mode, slopes=sl)
        np.testing.assert_allclose(o, o_ref[:, p], atol=1e-12)


def test_decode_after_fill_equals_forward_row():
    # fill positions 0..P-1 from a prefill, then decode P: same as forward row P
    B, H, Hkv, d, N, w, s, base = 1, 2, 1, 8, 24, 6, 2, 5e5
    q, k, v = [t.numpy() for t in inputs.qkv(B, N, H, Hkv, d, seed=41, dtype=torch.float32)]
    o_ref, _ = oracle.swat_fwd(q, k, v, window=w, n_sink=s, mode=1, rope_base=base)
    P = 20
    rc = oracle.RingCache(B, Hkv, d, w, s, base)
    rc.fill(k[:, :P], v[:, :P], 0)
    for p in range(P, N):
        o = rc.step(q[:, p], k[:, p], v[:, p], np.full(B, p), mode=1)
        np.testing.assert_allclose(o, o_ref[:, p], atol=1e-12)


@pytest.mark.parametrize("mode,Hkv,w,s", [(0, 2, 9, 0), (1, 1, 7, 3), (1, 4, 100, 2), (0, 2, 5, 4)])
def test_bwd_c_oracle_equals_dense_numpy_bwd(mode, Hkv, w, s):
    """Two backward derivations written independently (per-row C loops vs
    dense numpy matrices) agree to rounding."""
    from oracle import ref_numpy
    q, k, v, do = [t.numpy().astype(np.float32) for t in
                   inputs.qkv(2, 37, 4, Hkv, 8, seed=11, dtype=torch.float32, with_dout=True)]
    sl = inputs.balanced_alibi_slopes(4).numpy()
    kw = dict(window=w, n_sink=s, mode=mode, slopes=sl, rope_base=1e4)
    for a, b in zip(oracle.swat_bwd(q, k, v, do, **kw), ref_numpy.swat_bwd(q, k, v, do, **kw)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


def test_round_bf16_helper_matches_torch_cast():
    from tests.helpers import round_bf16
    x = np.random.default_rng(0).standard_normal(50000).astype(np.float32) * 7
    x[:4] = [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]   # exact ties
    assert np.array_equal(round_bf16(x), torch.tensor(x).bfloat16().double().numpy())
