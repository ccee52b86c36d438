"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test names the page passage (or the closed form / library routine) it
pins. A plausible mistake in the oracle — a dropped ALiBi term, a flipped
slope sign, an off-by-one window, a transposed rotation, a wrong GQA head
index, a double-counted sink — fails at least one of them.
"""
from __future__ import annotations

import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import ref_numpy
from sliding_window_sigmoid_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kv(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = [x.strip() for x in line.split("=", 1)]
        out[k] = v
    return out


def _oracle_mask(N, window, n_sink=0):
    return np.array([[oracle.in_keyset(i, j, window, n_sink) for j in range(N)] for i in range(N)],
                    dtype=bool)


# ---------------------------------------------------------------------------
# Mask / key set: glossary "How the window grows with depth"
# ---------------------------------------------------------------------------

def test_mask_counts_58_vs_136():
    g = _kv("mask_counts.txt")
    N, w = int(g["seq_len"]), int(g["window"])
    m = _oracle_mask(N, w)
    assert m.sum() == int(g["windowed_scores"])
    causal = _oracle_mask(N, N)
    assert causal.sum() == int(g["causal_scores"])
    # the numpy oracle builds the same mask from the offset matrix
    assert (ref_numpy.mask_matrix(N, w) == m).all()


def test_reach_4_7_10_13():
    g = _kv("mask_counts.txt")
    N, w = int(g["seq_len"]), int(g["window"])
    m = _oracle_mask(N, w).astype(np.int64)
    expected = [int(x) for x in g["reach_layers_1_to_4"].split()]
    reach = m.copy()
    got = []
    for _ in range(4):
        got.append(int(reach[-1].sum()))
        reach = ((m @ reach) > 0).astype(np.int64)
    assert got == expected


def _last_token_reach(N, w, L):
    m = _oracle_mask_fast(N, w)
    r = np.zeros(N, dtype=np.float32)
    r[-1] = 1.0
    for _ in range(L):
        r = ((r @ m) > 0).astype(np.float32)
    return int(r.sum())


def _oracle_mask_fast(N, w):
    # the oracle's key-set predicate evaluated on the band only (it is zero elsewhere)
    m = np.zeros((N, N), dtype=np.float32)
    for i in range(N):
        for j in range(max(0, i - w - 1), i + 1):
            if oracle.in_keyset(i, j, w, 0):
                m[i, j] = 1.0
    return m


def test_receptive_field_255_and_1525():
    g = _kv("receptive_field.txt")
    w = int(g["window_a"])
    assert _last_token_reach(300, w, int(g["layers_a"])) == int(g["field_a"])
    assert _last_token_reach(1600, w, int(g["layers_b"])) == int(g["field_b"])
    # ~131K for 32 layers, window 4096 (printed rounded to thousands)
    wc, Lc = int(g["window_c"]), int(g["layers_c"])
    field_c = 1 + (wc - 1) * Lc
    assert round(field_c / 1000) == int(g["field_c_approx_thousands"])
    # the closed form 1 + (w-1) L agrees with the composed mask on the cases above
    assert 1 + (w - 1) * int(g["layers_a"]) == int(g["field_a"])
    assert 1 + (w - 1) * int(g["layers_b"]) == int(g["field_b"])


def test_keyset_sinks_union_no_double_count():
    # SWA(w, s): the first s tokens plus the recent w; a sink inside the window counts once
    w, s = 4, 2
    for i in range(12):
        keys = [j for j in range(i + 1) if oracle.in_keyset(i, j, w, s)]
        expect = sorted(set(range(max(0, i - w + 1), i + 1)) | set(j for j in range(s) if j <= i))
        assert keys == expect
        assert oracle.keyset_size(i, w, s) == len(expect)


def test_ring_capacity_8x():
    g = _kv("ring_cache.txt")
    assert int(g["seq_tokens"]) // int(g["window"]) == int(g["memory_reduction"])


# ---------------------------------------------------------------------------
# Activations through the full forward
# ---------------------------------------------------------------------------

def _single_score_fwd(x, mode=oracle.MODE_SIGMOID):
    # N=1, d=2, no RoPE: s = q.k / sqrt(2) with q = (sqrt(2) x, 0), k = (1, 0); v = (1, 0)
    q = np.array([[[[math.sqrt(2.0) * x, 0.0]]]], np.float64)
    k = np.array([[[[1.0, 0.0]]]], np.float64)
    v = np.array([[[[1.0, 0.0]]]], np.float64)
    o, _ = oracle.swat_fwd(q, k, v, window=1, mode=mode, rope_base=0.0)
    return o[0, 0, 0, 0]


def test_sigmoid_printed_values():
    for line in open(os.path.join(GOLDEN, "sigmoid_values.txt")):
        if line.startswith("#") or not line.strip():
            continue
        x, val, dec = line.split()
        got = _single_score_fwd(float(x))
        assert round(got, int(dec)) == pytest.approx(float(val), abs=1e-12)
    assert _single_score_fwd(0.0) == pytest.approx(0.5, abs=1e-7)


def test_softmax_printed_example():
    g = _kv("softmax_example.txt")
    scores = [float(x) for x in g["scores"].split()]
    want = [float(x) for x in g["weights_2dp"].split()]
    n, d = len(scores), 6
    q = np.zeros((1, n, 1, d), np.float32)
    k = np.zeros((1, n, 1, d), np.float32)
    v = np.zeros((1, n, 1, d), np.float32)
    # last query's score for key j is scores[j]; v_j is the unit vector e_j
    q[0, n - 1, 0, 0] = 1.0
    for j, s in enumerate(scores):
        k[0, j, 0, 0] = s * math.sqrt(d)
        v[0, j, 0, j] = 1.0
    o, _ = oracle.swat_fwd(q, k, v, window=n, mode=oracle.MODE_SOFTMAX, rope_base=0.0)
    weights = o[0, n - 1, 0, :n]
    assert [round(x, 2) for x in weights] == want
    assert weights.sum() == pytest.approx(1.0, abs=1e-12)
    assert int(np.argmax(weights)) == 1 and weights[1] > 0.85  # "88% mass on one token"


# ---------------------------------------------------------------------------
# Softmax mode == PyTorch SDPA (library routine) with the key-set mask
# ("the same mask can be passed as attn_mask to scaled_dot_product_attention")
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("H,Hkv,N,d,w,s,slopes", [
    (2, 2, 33, 8, 5, 0, None),
    (4, 2, 40, 16, 7, 3, "balanced"),
    (4, 1, 29, 8, 64, 2, "balanced"),   # window >= N: full causal
    (2, 2, 50, 8, 1, 4, None),          # window 1: self (+ sinks) only
])
def test_softmax_matches_sdpa(H, Hkv, N, d, w, s, slopes):
    B = 2
    q, k, v = [t.float().numpy() for t in inputs.qkv(B, N, H, Hkv, d, seed=7, dtype=torch.float32)]
    sl = None if slopes is None else inputs.balanced_alibi_slopes(H).numpy()
    base = 10000.0
    o, lse = oracle.swat_fwd(q, k, v, window=w, n_sink=s, mode=oracle.MODE_SOFTMAX,
                             slopes=sl, rope_base=base)
    pos = np.arange(N)
    G = H // Hkv
    qt = torch.tensor(ref_numpy.rope_complex(q.transpose(0, 2, 1, 3), pos, base))  # [B,H,N,d]
    kt = torch.tensor(ref_numpy.rope_complex(k.transpose(0, 2, 1, 3), pos, base))
    vt = torch.tensor(v.transpose(0, 2, 1, 3).astype(np.float64))
    kt = kt.repeat_interleave(G, dim=1)
    vt = vt.repeat_interleave(G, dim=1)
    allowed = torch.tensor(_oracle_mask(N, w, s))
    bias = torch.zeros(H, N, N, dtype=torch.float64)
    if sl is not None:
        dist = torch.tensor((pos[:, None] - pos[None, :]).astype(np.float64))
        bias = torch.tensor(sl.astype(np.float64))[:, None, None] * dist[None]
    attn_mask = torch.where(allowed[None], bias, torch.tensor(float("-inf"), dtype=torch.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=attn_mask[None])
    ref = ref.permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    if w >= N and s == 0 and sl is None:
        causal = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
        np.testing.assert_allclose(o, causal.permute(0, 2, 1, 3).numpy(), atol=1e-12)


# ---------------------------------------------------------------------------
# Sigmoid-mode closed forms
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("w,s", [(4, 0), (5, 2), (100, 0), (1, 3)])
def test_sigmoid_zero_qk_counts_keys(w, s):
    # Q = K = 0, slopes 0 -> every weight is sigma(0) = 1/2, so with V = 1 the
    # output is half the size of the key set: |window part| + |sinks before it|.
    N, d = 23, 4
    q = np.zeros((1, N, 1, d), np.float32)
    k = np.zeros((1, N, 1, d), np.float32)
    v = np.ones((1, N, 1, d), np.float32)
    o, _ = oracle.swat_fwd(q, k, v, window=w, n_sink=s, rope_base=1e4)
    for i in range(N):
        n_keys = min(i + 1, w) + min(s, max(0, i - w + 1))
        assert o[0, i, 0, 0] == pytest.approx(0.5 * n_keys, abs=1e-12)


@pytest.mark.parametrize("slope", [-0.25, 0.125, -2.0 ** -6, 0.5])
def test_sigmoid_zero_qk_alibi_closed_form(slope):
    # Q = K = 0: the score is slope * (i - j). With V = 1,
    # o_i = sum_{delta=0}^{min(i, w-1)} sigma(slope * delta).
    N, d, w = 40, 4, 9
    q = np.zeros((1, N, 1, d), np.float32)
    k = np.zeros((1, N, 1, d), np.float32)
    v = np.ones((1, N, 1, d), np.float32)
    o, _ = oracle.swat_fwd(q, k, v, window=w, slopes=np.array([slope], np.float32), rope_base=0.0)
    sl = float(np.float32(slope))
    for i in range(N):
        ref = sum(1.0 / (1.0 + math.exp(-sl * dl)) for dl in range(min(i, w - 1) + 1))
        assert o[0, i, 0, 0] == pytest.approx(ref, abs=1e-12)


def test_alibi_sign_semantics():
    # "Negative slopes favor small (m-n) (recent tokens); positive slopes favor
    # large (m-n) (distant tokens within the window)" — Balanced ALiBi section.
    N, d, w = 12, 12, 12
    q = np.zeros((1, N, 2, d), np.float32)
    k = np.zeros((1, N, 1, d), np.float32)
    v = np.zeros((1, N, 1, d), np.float32)
    for j in range(N):
        v[0, j, 0, j] = 1.0          # output column j = weight of key j
    sl = np.array([-0.5, 0.5], np.float32)
    o, _ = oracle.swat_fwd(q, k, v, window=w, slopes=sl, rope_base=0.0)
    i = N - 1
    fwd_w = o[0, i, 0, :N]           # forward-looking head, weight by key j
    bwd_w = o[0, i, 1, :N]
    # weight as a function of distance delta = i - j
    fwd_by_delta = fwd_w[::-1]
    bwd_by_delta = bwd_w[::-1]
    assert np.all(np.diff(fwd_by_delta) < 0)   # decreasing with distance
    assert np.all(np.diff(bwd_by_delta) > 0)   # increasing with distance


def test_window_at_least_n_is_full_causal():
    # "short-sequence (window > sequence, global attention)": any window >= N
    # gives the same output as the full causal (lower-triangular) mask.
    B, N, H, d = 1, 30, 2, 8
    q, k, v = [t.numpy() for t in inputs.qkv(B, N, H, H, d, seed=3, dtype=torch.float32)]
    sl = inputs.balanced_alibi_slopes(H).numpy()
    o1, _ = oracle.swat_fwd(q, k, v, window=N, slopes=sl)
    o2, _ = oracle.swat_fwd(q, k, v, window=N + 37, slopes=sl)
    o3, _ = ref_numpy.swat_fwd(q, k, v, window=10 ** 6, slopes=sl)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_allclose(o1, o3, atol=1e-12)


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

def test_rope_matches_complex_form_and_is_rotation():
    rng = np.random.default_rng(0)
    d = 16
    for pos in [0, 1, 7, 4095, 65535]:
        x = rng.standard_normal(d)
        y = oracle.rope_rotate(x, pos, 1e4)
        z = ref_numpy.rope_complex(x[None, :], np.array([pos]), 1e4)[0]
        np.testing.assert_allclose(y, z, atol=1e-12)
        assert np.linalg.norm(y) == pytest.approx(np.linalg.norm(x), rel=1e-14)
        back = oracle.rope_rotate(y, pos, 1e4, inverse=True)
        np.testing.assert_allclose(back, x, atol=1e-12)
    # position 0 is the identity; base <= 0 disables the rotation
    x = rng.standard_normal(d)
    np.testing.assert_array_equal(oracle.rope_rotate(x, 0, 1e4), x)
    np.testing.assert_array_equal(oracle.rope_rotate(x, 123, 0.0), x)


def test_rope_depends_only_on_relative_position():
    # "The rotation encodes relative position (m-n) directly in the inner product"
    rng = np.random.default_rng(1)
    d = 32
    qv, kv = rng.standard_normal(d), rng.standard_normal(d)
    for (m, n) in [(10, 3), (100, 99), (5000, 1000)]:
        ref = oracle.rope_rotate(qv, m, 1e4) @ oracle.rope_rotate(kv, n, 1e4)
        for c in [1, 17, 30000]:
            got = oracle.rope_rotate(qv, m + c, 1e4) @ oracle.rope_rotate(kv, n + c, 1e4)
            assert got == pytest.approx(ref, abs=1e-9)


# ---------------------------------------------------------------------------
# The two oracles agree (independent formulations)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("H,Hkv,N,d,w,s,slopes,base", [
    (2, 2, 37, 8, 6, 0, "geometric", 1e4),
    (4, 2, 41, 16, 9, 3, "balanced", 5e5),
    (4, 4, 20, 8, 30, 2, "balanced", 1e4),
    (6, 3, 26, 4, 1, 0, None, 1e4),
    (2, 1, 33, 8, 5, 4, "balanced", 0.0),
])
def test_c_oracle_matches_numpy_oracle(mode, H, Hkv, N, d, w, s, slopes, base):
    B = 2
    q, k, v = [t.numpy() for t in inputs.qkv(B, N, H, Hkv, d, seed=11, dtype=torch.float32)]
    sl = None
    if slopes == "balanced":
        sl = inputs.balanced_alibi_slopes(H).numpy()
    elif slopes == "geometric":
        sl = inputs.geometric_alibi_slopes(H).numpy()
    o1, l1 = oracle.swat_fwd(q, k, v, window=w, n_sink=s, mode=mode, slopes=sl, rope_base=base)
    o2, l2 = ref_numpy.swat_fwd(q, k, v, window=w, n_sink=s, mode=mode, slopes=sl, rope_base=base)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    if mode == 1:
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_sampled_rows_equal_full_forward():
    B, N, H, Hkv, d = 2, 50, 4, 2, 8
    q, k, v = [t.numpy() for t in inputs.qkv(B, N, H, Hkv, d, seed=5, dtype=torch.float32)]
    sl = inputs.balanced_alibi_slopes(H).numpy()
    for mode in (0, 1):
        o, lse = oracle.swat_fwd(q, k, v, window=7, n_sink=2, mode=mode, slopes=sl)
        rows = np.array([[0, 0, 0], [1, 3, 49], [0, 2, 17], [1, 1, 8]])
        orow, lrow = oracle.swat_fwd_rows(q, k, v, rows, window=7, n_sink=2, mode=mode, slopes=sl)
        for r, (b, h, i) in enumerate(rows):
            np.testing.assert_array_equal(orow[r], o[b, i, h])
            if mode == 1:
                assert lrow[r] == lse[b, h, i]


# ---------------------------------------------------------------------------
# Slope generators ("Balanced ALiBi": half the heads -2^-k, half +2^-k)
# ---------------------------------------------------------------------------

def test_balanced_slopes():
    s = inputs.balanced_alibi_slopes(16).numpy()
    assert (s[:8] < 0).all() and (s[8:] > 0).all()
    np.testing.assert_array_equal(-s[:8], s[8:])
    np.testing.assert_array_equal(s[8:], [2.0 ** -k for k in range(1, 9)])
    # for 16 heads each half equals standard ALiBi's geometric 2^(-8k/n) with n = 8
    np.testing.assert_allclose(s[8:], [2.0 ** (-8.0 * k / 8) for k in range(1, 9)])
    g = inputs.geometric_alibi_slopes(2).numpy()
    np.testing.assert_array_equal(g, [-1.0 / 16, 1.0 / 256])
    with pytest.raises(ValueError):
        inputs.balanced_alibi_slopes(3)
