"""GPU forward parity against the CPU oracle, through the C ABI."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from sliding_window_sigmoid_b200 import binding, inputs
from tests.helpers import assert_bf16_close, assert_f32_close, sample_rows, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _run_fwd(q, k, v, **kw):
    o, lse = binding.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), **kw)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    return o, lse


# ---------------------------------------------------------------------------
# fp32 path: the tiny SWAT config at 1e-5, plus the 16-token window-4 probe
# ---------------------------------------------------------------------------

def test_tiny_f32_config_matches_oracle():
    w = inputs.TINY_F32
    q, k, v = inputs.qkv(w.B, w.N, w.H, w.Hkv, w.d, seed=0, dtype=torch.float32)
    sl = w.slope_tensor()
    o, _ = _run_fwd(q, k, v, window=w.window, mode=0, slopes=sl, rope_base=w.rope_base)
    ref, _ = oracle.swat_fwd(q.numpy(), k.numpy(), v.numpy(), window=w.window, slopes=sl.numpy(),
                             rope_base=w.rope_base)
    assert_f32_close(o, ref, "tiny fp32")


@pytest.mark.parametrize("mode,H,Hkv,N,d,w,s,base", [
    (0, 4, 2, 97, 32, 9, 0, 1e4),
    (1, 4, 2, 97, 32, 9, 3, 1e4),
    (1, 2, 1, 70, 6, 100, 2, 5e5),   # odd-ish small head size, window > N
    (0, 2, 2, 50, 128, 1, 0, 0.0),   # window 1, RoPE off
])
def test_f32_variants_match_oracle(mode, H, Hkv, N, d, w, s, base):
    B = 2
    q, k, v = inputs.qkv(B, N, H, Hkv, d, seed=4, dtype=torch.float32)
    sl = inputs.balanced_alibi_slopes(H)
    o, lse = _run_fwd(q, k, v, window=w, n_sink=s, mode=mode, slopes=sl, rope_base=base)
    ref, lref = oracle.swat_fwd(q.numpy(), k.numpy(), v.numpy(), window=w, n_sink=s, mode=mode,
                                slopes=sl.numpy(), rope_base=base)
    assert_f32_close(o, ref, "fp32 o")
    if mode == 1:
        assert_f32_close(lse, lref, "fp32 lse")


def _index_probe(N, window, n_sink, dtype, d=64):
    # Q = K = 0 and slopes 0 make every weight sigma(0) = 1/2 exactly. V_j holds
    # the bits of j in channels 0..16 and a 1 in channel 17, so 2*o_i recovers
    # |keys(i)| and, per bit, how many keys have that bit: exact integers.
    q = torch.zeros(1, N, 1, d, dtype=dtype)
    k = torch.zeros(1, N, 1, d, dtype=dtype)
    v = torch.zeros(1, N, 1, d, dtype=torch.float32)
    for j in range(N):
        for c in range(17):
            v[0, j, 0, c] = (j >> c) & 1
        v[0, j, 0, 17] = 1.0
    v = v.to(dtype)
    o, _ = _run_fwd(q, k, v, window=window, n_sink=n_sink, mode=0, slopes=None, rope_base=1e4)
    got = (2.0 * to_np(o)[0, :, 0, :18])
    for i in range(N):
        keys = [j for j in range(i + 1) if oracle.in_keyset(i, j, window, n_sink)]
        want = [sum((j >> c) & 1 for j in keys) for c in range(17)] + [len(keys)]
        np.testing.assert_array_equal(got[i], np.array(want, dtype=np.float64), err_msg=f"row {i}")


def test_index_probe_16_tokens_window_4_fp32():
    _index_probe(16, 4, 0, torch.float32)
    # the probe's key count over all rows is the page's 58
    q = torch.zeros(1, 16, 1, 64)
    v = torch.zeros(1, 16, 1, 64)
    v[..., 0] = 1.0
    o, _ = _run_fwd(q, q.clone(), v, window=4, mode=0)
    assert int(round(2.0 * float(o[0, :, 0, 0].sum()))) == 58


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
# (257, 256): a 128 x 128 tile whose farthest pair sits at distance 255 is
# entirely in the window (unmasked pass); (400, 255): at distance 255 it is
# not, so the same tiles take the masked pass.
@pytest.mark.parametrize("N,w,s", [(300, 64, 0), (300, 100, 5), (257, 256, 0), (400, 255, 0), (400, 129, 2),
                                   (130, 1, 3), (200, 500, 0)])
def test_index_probe_bit_exact(dtype, N, w, s):
    _index_probe(N, w, s, dtype)


# ---------------------------------------------------------------------------
# bf16 tensor-core path
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode,B,H,Hkv,N,d,w,s,base,slopes", [
    (0, 2, 4, 4, 300, 64, 64, 0, 1e4, "balanced"),
    (0, 1, 4, 2, 777, 128, 200, 0, 1e4, "balanced"),
    (0, 2, 2, 2, 129, 64, 16, 0, 1e4, "geometric"),
    (0, 1, 2, 1, 1000, 64, 1000, 0, 1e4, "balanced"),   # window >= N: full causal
    (0, 1, 2, 2, 65, 128, 1, 0, 0.0, None),             # window 1, no RoPE
    (1, 1, 8, 2, 700, 128, 64, 4, 5e5, None),           # SWA(64,4) shape, GQA
    (1, 2, 4, 4, 333, 64, 100, 0, 1e4, "balanced"),     # softmax with ALiBi
    (1, 1, 4, 1, 450, 64, 30, 64, 1e4, None),           # many sinks
    (0, 1, 4, 2, 300, 128, 50, 7, 1e4, "balanced"),     # sinks in sigmoid mode
])
@pytest.mark.parametrize("ws", ["rotated copies", "in-kernel rotation"])
def test_bf16_matches_oracle(mode, B, H, Hkv, N, d, w, s, base, slopes, ws):
    """Both entry points: swat_attn_fwd_ws (rotated Q/K copies in a workspace)
    and swat_attn_fwd (tiles rotated in shared memory)."""
    scale = 1.0 / np.sqrt(d) if mode == 0 else 1.0
    q, k, v = inputs.qkv(B, N, H, Hkv, d, seed=2, scale=scale, dtype=torch.bfloat16)
    sl = None
    if slopes == "balanced":
        sl = inputs.balanced_alibi_slopes(H)
    elif slopes == "geometric":
        sl = inputs.geometric_alibi_slopes(H)
    o, lse = _run_fwd(q, k, v, window=w, n_sink=s, mode=mode, slopes=sl, rope_base=base,
                      workspace=None if ws == "rotated copies" else False)
    ref, lref = oracle.swat_fwd(q.float().numpy(), k.float().numpy(), v.float().numpy(), window=w,
                                n_sink=s, mode=mode, slopes=None if sl is None else sl.numpy(),
                                rope_base=base)
    assert_bf16_close(o, ref, "bf16 o")
    if mode == 1:
        np.testing.assert_allclose(to_np(lse), lref, atol=2e-2, rtol=0)


def _full_size_rows(wl, seed, n_random=300):
    q, k, v = inputs.qkv(wl.B, wl.N, wl.H, wl.Hkv, wl.d, seed=seed, scale=wl.scale,
                         dtype=torch.bfloat16)
    sl = wl.slope_tensor()
    o, lse = _run_fwd(q, k, v, window=wl.window, n_sink=wl.n_sink, mode=wl.mode, slopes=sl,
                      rope_base=wl.rope_base)
    rows = sample_rows(wl.B, wl.H, wl.N, wl.window, n_random=n_random, seed=seed)
    ref, lref = oracle.swat_fwd_rows(q.float().numpy(), k.float().numpy(), v.float().numpy(), rows,
                                     window=wl.window, n_sink=wl.n_sink, mode=wl.mode,
                                     slopes=None if sl is None else sl.numpy(),
                                     rope_base=wl.rope_base)
    o_np = o.float().cpu().numpy()
    got = np.stack([o_np[b, i, h] for b, h, i in rows])
    assert_bf16_close(got, ref, wl.name)
    if wl.mode == 1:
        l_np = lse.cpu().numpy()
        lgot = np.array([l_np[b, h, i] for b, h, i in rows])
        np.testing.assert_allclose(lgot, lref, atol=2e-2, rtol=0)
    assert np.isfinite(o_np).all()


def test_full_size_swat_340m_layer_sampled_rows():
    _full_size_rows(inputs.SWAT_340M, seed=0)


def test_full_size_long_sequence_sampled_rows():
    _full_size_rows(inputs.SWAT_LONG, seed=0, n_random=120)


def test_full_size_swa_sink_gqa_sampled_rows():
    _full_size_rows(inputs.SWA_SINK, seed=0)


def test_translation_of_rope_positions_only_matters_relatively():
    # Shifting all tokens by whole tiles changes absolute RoPE angles but the
    # outputs of a shifted copy of a sequence stay within tolerance of each
    # other wherever the windows see the same tokens (window fully inside).
    B, N, H, d, w = 1, 512, 2, 64, 64
    q, k, v = inputs.qkv(B, N, H, H, d, seed=13, scale=0.125, dtype=torch.bfloat16)
    o1, _ = _run_fwd(q, k, v, window=w, mode=0, slopes=inputs.balanced_alibi_slopes(H))
    pad = 128
    qp = torch.cat([torch.zeros(B, pad, H, d, dtype=q.dtype), q], 1)
    kp = torch.cat([torch.zeros(B, pad, H, d, dtype=q.dtype), k], 1)
    vp = torch.cat([torch.zeros(B, pad, H, d, dtype=q.dtype), v], 1)
    o2, _ = _run_fwd(qp, kp, vp, window=w, mode=0, slopes=inputs.balanced_alibi_slopes(H))
    assert_bf16_close(o2[:, pad + w:], o1[:, w:], "shifted")
