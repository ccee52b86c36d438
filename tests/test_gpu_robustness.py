"""Guard bands, run-to-run determinism and decode resume, through the C ABI.

* Every output and workspace of the forward, backward and decode calls sits
  inside a larger buffer whose margins hold a sentinel; after the call the
  margins must be untouched (ragged N, so the last 128-row tiles are partial).
* Two runs of the same call give bit-identical outputs: the kernels have no
  atomics and a fixed reduction order.
* A decode that is stopped, whose caller-owned ring state (cache, sinks,
  positions) is copied into a fresh cache object, and resumed gives the same
  outputs, bit for bit, as one that ran straight through.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from sliding_window_sigmoid_b200 import binding, inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
PAD = 4096            # elements of margin on each side (keeps 16-byte alignment)
SENTINEL = -7.0


def _guarded(shape, dtype):
    """(buffer, view): view = the tensor of `shape` inside `buffer`, whose
    PAD-element margins hold SENTINEL."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * PAD,), SENTINEL, dtype=dtype, device=DEV)
    return buf, buf[PAD:PAD + n].view(*shape)


def _guarded_bytes(nbytes):
    buf = torch.full((nbytes + 2 * PAD,), 0xA5, dtype=torch.uint8, device=DEV)
    return buf, buf[PAD:PAD + nbytes]


def _margins_intact(buf, what):
    head, tail = buf[:PAD], buf[-PAD:]
    if buf.dtype == torch.uint8:
        ok = bool((head == 0xA5).all()) and bool((tail == 0xA5).all())
    else:
        ok = bool((head == SENTINEL).all()) and bool((tail == SENTINEL).all())
    assert ok, f"{what}: a write landed outside the tensor"


def _sync_ok():
    torch.cuda.synchronize()
    assert binding.device_status() == 0


@pytest.mark.parametrize("mode,H,Hkv,N,d,w,s", [
    (0, 4, 2, 300, 64, 64, 0),       # sigmoid, GQA, d 64
    (0, 4, 2, 333, 128, 200, 0),     # sigmoid, GQA, d 128
    (1, 8, 2, 300, 128, 64, 4),      # SWA(64, 4) shape: softmax with sinks, GQA
])
def test_forward_backward_write_only_their_tensors(mode, H, Hkv, N, d, w, s):
    B = 2
    scale = 1.0 / np.sqrt(d) if mode == 0 else 1.0
    q, k, v, do = [t.to(DEV) for t in inputs.qkv(B, N, H, Hkv, d, seed=31, scale=scale, dtype=torch.bfloat16,
                                                  with_dout=True)]
    sl = inputs.balanced_alibi_slopes(H) if mode == 0 else None
    kw = dict(window=w, n_sink=s, mode=mode, slopes=sl, rope_base=1e4)
    ob, o = _guarded((B, N, H, d), torch.bfloat16)
    lb, lse = _guarded((B, H, N), torch.float32)
    wb, ws = _guarded_bytes(max(16, binding.fwd_workspace_bytes(B, H, Hkv, N, d)))
    binding.attn_fwd(q, k, v, out=o, lse=lse if mode == 1 else None, workspace=ws, **kw)
    _sync_ok()
    _margins_intact(ob, "o")
    _margins_intact(wb, "forward workspace")
    if mode == 1:
        _margins_intact(lb, "lse")
    lse_in = lse if mode == 1 else None
    grads = [_guarded(t.shape, torch.bfloat16) for t in (q, k, v)]
    bb, bws = _guarded_bytes(max(16, binding.bwd_workspace_bytes(B, H, Hkv, N, d)))
    binding.attn_bwd(q, k, v, o, lse_in, do, dq=grads[0][1], dk=grads[1][1], dv=grads[2][1], workspace=bws, **kw)
    _sync_ok()
    for (buf, _), name in zip(grads, ("dq", "dk", "dv")):
        _margins_intact(buf, name)
    _margins_intact(bb, "backward workspace")
    assert torch.isfinite(o.float()).all()
    for _, g in grads:
        assert torch.isfinite(g.float()).all()


def test_decode_writes_only_its_output():
    B, H, Hkv, d, w, s = 4, 8, 2, 128, 300, 2
    cache = binding.RingCache(B, H, Hkv, d, w, s, mode=1, slopes=None, rope_base=5e5, device=DEV)
    kf = inputs.normal((B, 250, Hkv, d), 621).to(DEV)
    vf = inputs.normal((B, 250, Hkv, d), 622).to(DEV)
    cache.fill(kf, vf, 0)
    q, kn, vn = [t.to(DEV) for t in inputs.decode_step_inputs(B, H, Hkv, d, 0)]
    ob, o = _guarded((B, H, d), torch.bfloat16)
    cache.step(q, kn, vn, torch.full((B,), 250, dtype=torch.int64, device=DEV), out=o)
    _sync_ok()
    _margins_intact(ob, "decode o")


@pytest.mark.parametrize("mode", [0, 1])
def test_forward_backward_deterministic(mode):
    B, H, Hkv, N, d, w = 2, 4, 4, 700, 64, 256
    q, k, v, do = [t.to(DEV) for t in inputs.qkv(B, N, H, Hkv, d, seed=32, scale=0.125, dtype=torch.bfloat16,
                                                  with_dout=True)]
    kw = dict(window=w, n_sink=0, mode=mode,
              slopes=inputs.balanced_alibi_slopes(H) if mode == 0 else None, rope_base=1e4)
    runs = []
    for _ in range(2):
        o, lse = binding.attn_fwd(q, k, v, **kw)
        dq, dk, dv = binding.attn_bwd(q, k, v, o, lse, do, **kw)
        _sync_ok()
        runs.append([t.clone() for t in (o, dq, dk, dv)] + ([lse.clone()] if lse is not None else []))
    for a, b, name in zip(runs[0], runs[1], ("o", "dq", "dk", "dv", "lse")):
        assert torch.equal(a, b), f"{name} differs between two identical runs"


def test_decode_resume_from_copied_state_is_bit_identical():
    B, H, Hkv, d, w, s, steps = 3, 8, 2, 128, 200, 2, 8
    kw = dict(mode=1, slopes=None, rope_base=5e5, device=DEV)
    kf = inputs.normal((B, 180, Hkv, d), 631).to(DEV)
    vf = inputs.normal((B, 180, Hkv, d), 632).to(DEV)
    step_in = [[t.to(DEV) for t in inputs.decode_step_inputs(B, H, Hkv, d, t)] for t in range(steps)]
    pos = [torch.full((B,), 180 + t, dtype=torch.int64, device=DEV) for t in range(steps)]

    straight = binding.RingCache(B, H, Hkv, d, w, s, **kw)
    straight.fill(kf, vf, 0)
    want = [straight.step(*step_in[t], pos[t]).clone() for t in range(steps)]

    first = binding.RingCache(B, H, Hkv, d, w, s, **kw)
    first.fill(kf, vf, 0)
    got = [first.step(*step_in[t], pos[t]).clone() for t in range(steps // 2)]
    _sync_ok()
    resumed = binding.RingCache(B, H, Hkv, d, w, s, **kw)
    for name in ("k_cache", "v_cache", "k_sink", "v_sink"):
        getattr(resumed, name).copy_(getattr(first, name))
    del first
    got += [resumed.step(*step_in[t], pos[t]).clone() for t in range(steps // 2, steps)]
    _sync_ok()
    for t in range(steps):
        assert torch.equal(got[t], want[t]), f"step {t}"
