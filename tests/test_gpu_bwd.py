"""GPU backward parity against the CPU oracle, through the C ABI."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from sliding_window_sigmoid_b200 import binding, inputs
from tests.helpers import assert_bf16_close, assert_f32_close, quantized_operand_bwd

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _fwd_bwd(q, k, v, do, **kw):
    q, k, v, do = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    o, lse = binding.attn_fwd(q, k, v, **kw)
    dq, dk, dv = binding.attn_bwd(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    return dq, dk, dv


@pytest.mark.parametrize("mode,H,Hkv,N,d,w,s", [
    (0, 2, 2, 70, 16, 9, 0),
    (1, 4, 2, 70, 16, 9, 3),
    (0, 4, 1, 45, 8, 64, 2),
    (1, 2, 2, 33, 64, 1, 0),
])
def test_f32_bwd_matches_oracle(mode, H, Hkv, N, d, w, s):
    B = 1
    q, k, v, do = inputs.qkv(B, N, H, Hkv, d, seed=5, dtype=torch.float32, with_dout=True)
    sl = inputs.balanced_alibi_slopes(H)
    kw = dict(window=w, n_sink=s, mode=mode, slopes=sl, rope_base=1e4)
    dq, dk, dv = _fwd_bwd(q, k, v, do, **kw)
    rq, rk, rv = oracle.swat_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), window=w, n_sink=s,
                                 mode=mode, slopes=sl.numpy(), rope_base=1e4)
    # gradients sum many more terms than the forward; 1e-5 relative to their scale
    for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        scale = max(1.0, float(np.abs(r).max()))
        assert_f32_close(g, r, name, tol=1e-5 * scale)


@pytest.mark.parametrize("mode,B,H,Hkv,N,d,w,s,slopes", [
    (0, 1, 4, 4, 300, 64, 64, 0, "balanced"),
    (0, 1, 4, 2, 400, 128, 100, 0, "balanced"),
    (1, 1, 8, 2, 300, 128, 64, 4, None),
    (1, 2, 2, 2, 260, 64, 50, 0, "balanced"),
    (0, 1, 2, 1, 200, 64, 300, 3, "balanced"),
])
def test_bf16_bwd_matches_oracle(mode, B, H, Hkv, N, d, w, s, slopes):
    scale = 1.0 / np.sqrt(d) if mode == 0 else 1.0
    q, k, v, do = inputs.qkv(B, N, H, Hkv, d, seed=6, scale=scale, dtype=torch.bfloat16,
                             with_dout=True)
    sl = inputs.balanced_alibi_slopes(H) if slopes == "balanced" else None
    kw = dict(window=w, n_sink=s, mode=mode, slopes=sl, rope_base=1e4)
    dq, dk, dv = _fwd_bwd(q, k, v, do, **kw)
    f = lambda t: t.float().numpy()
    sl_np = None if sl is None else sl.numpy()
    rq, rk, rv = oracle.swat_bwd(f(q), f(k), f(v), f(do), window=w, n_sink=s, mode=mode,
                                 slopes=sl_np, rope_base=1e4)
    aq, ak, av = quantized_operand_bwd(f(q), f(k), f(v), f(do), window=w, n_sink=s, mode=mode,
                                       slopes=sl_np, rope_base=1e4, exact=(rq, rk, rv))
    assert_bf16_close(dq, rq, "dq", allowance=aq)
    assert_bf16_close(dk, rk, "dk", allowance=ak)
    assert_bf16_close(dv, rv, "dv", allowance=av)


def test_full_size_swat_340m_bwd_sampled_rows():
    wl = inputs.SWAT_340M
    q, k, v, do = inputs.qkv(wl.B, wl.N, wl.H, wl.Hkv, wl.d, seed=0, scale=wl.scale,
                             dtype=torch.bfloat16, with_dout=True)
    sl = wl.slope_tensor()
    kw = dict(window=wl.window, n_sink=0, mode=0, slopes=sl, rope_base=wl.rope_base)
    dq, dk, dv = _fwd_bwd(q, k, v, do, **kw)
    rng = np.random.default_rng(1)
    qrows = np.array([[rng.integers(wl.B), rng.integers(wl.H), i] for i in
                      [0, 1, 511, 512, 2047, 4095] + list(rng.integers(0, wl.N, 90))])
    krows = np.array([[rng.integers(wl.B), rng.integers(wl.Hkv), j] for j in
                      [0, 1, 127, 128, 3583, 3584, 4095] + list(rng.integers(0, wl.N, 60))])
    f = lambda t: t.float().numpy()
    rq, rk, rv = oracle.swat_bwd_rows(f(q), f(k), f(v), f(do), qrows, krows, window=wl.window,
                                      n_sink=0, mode=0, slopes=sl.numpy(), rope_base=wl.rope_base)
    dq_np, dk_np, dv_np = f(dq.cpu()), f(dk.cpu()), f(dv.cpu())
    assert_bf16_close(np.stack([dq_np[b, i, h] for b, h, i in qrows]), rq, "dq rows")
    assert_bf16_close(np.stack([dk_np[b, j, h] for b, h, j in krows]), rk, "dk rows")
    assert_bf16_close(np.stack([dv_np[b, j, h] for b, h, j in krows]), rv, "dv rows")
    for g in (dq_np, dk_np, dv_np):
        assert np.isfinite(g).all()


@pytest.mark.parametrize("mode,H,Hkv,d", [(0, 4, 4, 64), (1, 8, 2, 128)])
def test_bwd_reusing_forward_rotated_copies_is_identical(mode, H, Hkv, d):
    """swat_attn_bwd_rotated with the forward workspace gives bit-identical
    gradients to swat_attn_bwd (same rotation, same kernels)."""
    B, N, w, s = 2, 333, 96, (4 if mode == 1 else 0)
    scale = 1.0 / np.sqrt(d) if mode == 0 else 1.0
    q, k, v, do = [t.to(DEV) for t in inputs.qkv(B, N, H, Hkv, d, seed=9, scale=scale, dtype=torch.bfloat16,
                                                  with_dout=True)]
    sl = inputs.balanced_alibi_slopes(H).to(DEV) if mode == 0 else None
    kw = dict(window=w, n_sink=s, mode=mode, slopes=sl, rope_base=1e4)
    fws = torch.empty(binding.fwd_workspace_bytes(B, H, Hkv, N, d), dtype=torch.uint8, device=DEV)
    o, lse = binding.attn_fwd(q, k, v, workspace=fws, **kw)
    g_ref = binding.attn_bwd(q, k, v, o, lse, do, **kw)
    g_rot = binding.attn_bwd(q, k, v, o, lse, do, qk_rot=fws, **kw)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    for a, b in zip(g_ref, g_rot):
        assert torch.equal(a, b)
