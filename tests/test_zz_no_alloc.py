"""swa_decode_step_noalloc (decode step with the library's own static scratch
buffer, no workspace argument) against swa_decode_step, through the C ABI.

Collected last on purpose: it must also pass after every other test has run
in the same process (the scratch buffer is then set up after other work)."""
from __future__ import annotations

import ctypes

import pytest
import torch

from sliding_window_sigmoid_b200 import binding, inputs
from tests.helpers import assert_bf16_close, assert_f32_close

DEV = "cuda"
FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: rejected before any launch


def test_noalloc_rejects_too_large_before_any_launch():
    L = binding.lib()
    B, H, Hkv, d, w = 2048, 32, 8, 128, 4096
    assert L.swa_decode_workspace_bytes(B, H, Hkv, d, w) > binding.NOALLOC_SCRATCH_BYTES
    n0 = binding.launch_count()
    st = L.swa_decode_step_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE,
                                   B, H, Hkv, d, w, 0, 0, None, 1e4, binding.BF16, None)
    assert st == binding.SCRATCH_LIMIT
    assert binding.status_string(st) == "SWAT_ERR_SCRATCH_LIMIT"
    assert binding.launch_count() == n0


def _pair(B, H, Hkv, d, w, s, mode, dtype, p0, seed):
    sl = inputs.balanced_alibi_slopes(H) if mode == 0 else None
    caches = [binding.RingCache(B, H, Hkv, d, w, s, mode=mode, slopes=sl, rope_base=1e4,
                                dtype=dtype, device=DEV) for _ in range(2)]
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, p0, Hkv, d, generator=g).to(dtype).to(DEV)
    v = torch.randn(B, p0, Hkv, d, generator=g).to(dtype).to(DEV)
    for c in caches:
        c.fill(k, v, 0)
    return caches


@pytest.mark.gpu
@pytest.mark.parametrize("mode,s,dtype,shape", [
    (0, 0, torch.bfloat16, (4, 32, 8, 128, 1024)),
    (1, 4, torch.bfloat16, (4, 32, 8, 128, 1024)),
    (0, 0, torch.bfloat16, (3, 16, 16, 64, 700)),
    (1, 2, torch.float32, (2, 4, 2, 32, 7)),
])
def test_noalloc_equals_workspace_entry_two_calls_in_a_row(mode, s, dtype, shape):
    B, H, Hkv, d, w = shape
    p0 = w + w // 2 + 3                      # the ring has wrapped
    ws_cache, na_cache = _pair(B, H, Hkv, d, w, s, mode, dtype, p0, seed=7)
    for t in range(2):
        q, kn, vn = inputs.decode_step_inputs(B, H, Hkv, d, t, dtype=dtype)
        q, kn, vn = q.to(DEV), kn.to(DEV), vn.to(DEV)
        pos = torch.full((B,), p0 + t, dtype=torch.int64, device=DEV)
        n0 = binding.launch_count()
        o_ref = ws_cache.step(q, kn, vn, pos)
        o_na = na_cache.step_noalloc(q, kn, vn, pos)
        torch.cuda.synchronize()
        assert binding.device_status() == 0
        assert binding.launch_count() > n0
        if dtype == torch.bfloat16:
            assert_bf16_close(o_na, o_ref, f"call {t}")
        else:
            assert_f32_close(o_na, o_ref, f"call {t}")
        assert torch.equal(o_na, o_ref), f"call {t}: the two entry points run the same kernels"
    assert torch.equal(ws_cache.k_cache, na_cache.k_cache)
    assert torch.equal(ws_cache.v_cache, na_cache.v_cache)
