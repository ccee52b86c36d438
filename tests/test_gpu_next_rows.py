"""Next rows of the hot path, through the GPU kernels.

* decode after a prefill equals the prefill's own last row (ring fill at
  scale: slot = pos mod w, sinks), "Sliding Window Attention" glossary,
  ring-buffer paragraph;
* SWAT(-) forward-only slopes ("SWAT" page, section "Balanced ALiBi");
* stacked layers: the last token's reach over a 4-layer, window-4 stack
  grows 4, 7, 10, 13 ("Sliding Window Attention" glossary, the 16-token
  example), and a local (w < N) then global (w >= N) pair of layers matches
  the oracle composed the same way.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from sliding_window_sigmoid_b200 import binding, inputs
from tests.helpers import assert_bf16_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("mode,H,Hkv,d,w,s,base", [
    (0, 32, 8, 128, 1024, 0, 1e4),      # sigmoid, balanced ALiBi, GQA
    (1, 32, 8, 128, 1024, 4, 5e5),      # softmax with 4 sinks
])
def test_decode_after_prefill_equals_prefill_last_row(mode, H, Hkv, d, w, s, base):
    """Prefill N tokens with swat_attn_fwd; fill the ring with the first N-1
    and decode token N-1: the decode output equals the forward's last row."""
    B, N = 4, 3001
    q, k, v = [t.to(DEV) for t in inputs.qkv(B, N, H, Hkv, d, seed=21, dtype=torch.bfloat16)]
    sl = inputs.balanced_alibi_slopes(H) if mode == 0 else None
    o, _ = binding.attn_fwd(q, k, v, window=w, n_sink=s, mode=mode, slopes=sl, rope_base=base)
    cache = binding.RingCache(B, H, Hkv, d, w, s, mode=mode, slopes=sl, rope_base=base, device=DEV)
    if s > 0:
        cache.fill(k[:, :s].contiguous(), v[:, :s].contiguous(), 0)
    cache.fill(k[:, :N - 1].contiguous(), v[:, :N - 1].contiguous(), 0)
    pos = torch.full((B,), N - 1, dtype=torch.int64, device=DEV)
    od = cache.step(q[:, N - 1].contiguous(), k[:, N - 1].contiguous(), v[:, N - 1].contiguous(), pos)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    # both sides are rounded to bf16: allow the second rounding (half an ulp of |o|)
    ref = o[:, N - 1].float().cpu().numpy()
    assert_bf16_close(od, ref, "decode vs prefill last row", allowance=2.0 ** -8 * np.abs(ref))


def test_forward_only_slopes_match_oracle():
    B, N, H, Hkv, d, w = 2, 400, 8, 8, 64, 128
    q, k, v = inputs.qkv(B, N, H, Hkv, d, seed=22, scale=0.125, dtype=torch.bfloat16)
    sl = inputs.forward_only_slopes(H)
    assert (sl < 0).all()
    o, _ = binding.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), window=w, slopes=sl, rope_base=1e4)
    ref, _ = oracle.swat_fwd(q.float().numpy(), k.float().numpy(), v.float().numpy(), window=w,
                             slopes=sl.numpy(), rope_base=1e4)
    assert_bf16_close(o, ref, "SWAT(-) forward")


def _stack_reach(n_layers, w=4, N=16, d=64):
    """Row-nonzero pattern of d(out_L[N-1]) / d(x_0) through an L-layer stack
    of SWAT layers with q = k = v = x (GPU forward and backward)."""
    x0 = inputs.qkv(1, N, 1, 1, d, seed=23, scale=1.0, dtype=torch.bfloat16)[0].to(DEV)
    kw = dict(window=w, mode=0, slopes=None, rope_base=1e4)
    xs = [x0]
    for _ in range(n_layers):
        o, _ = binding.attn_fwd(xs[-1], xs[-1], xs[-1], **kw)
        xs.append(o)
    g = torch.zeros_like(x0)
    g[0, N - 1, 0, :] = 1.0
    for layer in range(n_layers, 0, -1):
        x = xs[layer - 1]
        dq, dk, dv = binding.attn_bwd(x, x, x, xs[layer], None, g, **kw)
        g = (dq.float() + dk.float() + dv.float()).to(torch.bfloat16)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    return (g[0, :, 0, :].float().abs().sum(dim=1) != 0).cpu().numpy()


@pytest.mark.parametrize("n_layers,reach", [(1, 4), (2, 7), (3, 10), (4, 13)])
def test_last_token_reach_through_stacked_layers(n_layers, reach):
    nz = _stack_reach(n_layers)
    N = nz.size
    expect = np.zeros(N, dtype=bool)
    expect[N - reach:] = True
    assert np.array_equal(nz, expect), f"nonzero rows {np.nonzero(nz)[0].tolist()}"


def test_local_then_global_layer_pair_matches_oracle():
    B, N, H, d = 1, 300, 4, 64
    x = inputs.qkv(B, N, H, H, d, seed=24, scale=0.5, dtype=torch.bfloat16)[0]
    sl = inputs.balanced_alibi_slopes(H)
    kw1 = dict(window=32, slopes=sl, rope_base=1e4)
    kw2 = dict(window=N, slopes=sl, rope_base=1e4)          # w >= N: full causal
    xd = x.to(DEV)
    o1, _ = binding.attn_fwd(xd, xd, xd, **kw1)
    o2, _ = binding.attn_fwd(o1, o1, o1, **kw2)
    xf = x.float().numpy()
    r1, _ = oracle.swat_fwd(xf, xf, xf, window=32, slopes=sl.numpy(), rope_base=1e4)
    # the second layer takes the first layer's bf16 output, as the GPU stack does
    r1b = torch.tensor(r1, dtype=torch.float32).to(torch.bfloat16).float().numpy()
    r2, _ = oracle.swat_fwd(r1b, r1b, r1b, window=N, slopes=sl.numpy(), rope_base=1e4)
    assert_bf16_close(o1, r1, "local layer")
    assert_bf16_close(o2, r2, "global layer")
