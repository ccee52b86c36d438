"""Host-only checks of the C ABI: the library loads, exports every symbol the
header declares, sizes its workspaces, names its status codes and rejects
invalid arguments before launching anything (no GPU needed)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from sliding_window_sigmoid_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"SWAT_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


@pytest.fixture(scope="module")
def L():
    from sliding_window_sigmoid_b200 import build
    build.build()
    return binding.lib()


def test_header_declares_the_boundary():
    names = _declared()
    for fn in ("swat_attn_fwd", "swat_attn_bwd", "swa_decode_step"):
        assert fn in names
    assert set(binding.EXPORTED) <= set(names)


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_status_strings(L):
    assert binding.status_string(0) == "SWAT_OK"
    assert binding.status_string(-1) == "SWAT_ERR_INVALID_ARG"
    assert binding.status_string(-2) == "SWAT_ERR_UNSUPPORTED"
    assert binding.status_string(-3) == "SWAT_ERR_CUDA"
    assert binding.status_string(-4) == "SWAT_ERR_TIMEOUT"
    assert binding.status_string(12345) == "SWAT_ERR_UNKNOWN"


def test_workspace_sizes(L):
    # decode: partial sums (d floats) plus max and denominator per (b, h, split)
    B, H, Hkv, d, w = 64, 32, 8, 128, 4096
    n = binding.lib().swa_decode_workspace_bytes(B, H, Hkv, d, w)
    nsplit = (w + 2047) // 2048          # the decode kernel streams 2048 ring slots per CTA
    assert n >= B * H * nsplit * (d + 2) * 4
    assert n < 2 * B * H * nsplit * (d + 2) * 4 + 4096
    assert binding.lib().swa_decode_workspace_bytes(0, H, Hkv, d, w) == 0
    # backward: at least the per-row D_i buffer of the softmax mode
    m = binding.bwd_workspace_bytes(8, 16, 16, 4096, 64, binding.BF16)
    assert m >= 8 * 16 * 4096 * 4


FAKE = ctypes.c_void_p(0x10000)   # 16-byte aligned, never dereferenced: validation fails first


def _fwd(L, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=2, Hkv=2, N=16, d=64, window=4,
             n_sink=0, mode=0, slopes=None, rope_base=1e4, dtype=0, stream=None)
    a.update(kw)
    return L.swat_attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Hkv"],
                           a["N"], a["d"], a["window"], a["n_sink"], a["mode"], a["slopes"],
                           a["rope_base"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), -1),
    (dict(window=0), -1),
    (dict(n_sink=-1), -1),
    (dict(n_sink=65), -1),
    (dict(H=3, Hkv=2), -1),
    (dict(d=7), -1),
    (dict(d=130), -1),
    (dict(d=96), -2),               # valid fp32 head size, not on the bf16 tensor-core path
    (dict(mode=2), -1),
    (dict(mode=1, lse=None), -1),
    (dict(dtype=5), -1),
    (dict(N=0), -1),
    (dict(B=0), -1),
    (dict(q=ctypes.c_void_p(0x10008)), -1),   # misaligned
])
def test_fwd_rejects_invalid_arguments(L, kw, expect):
    before = binding.launch_count()
    assert _fwd(L, **kw) == expect
    assert binding.launch_count() == before   # nothing launched


def test_bwd_and_decode_reject_invalid_arguments(L):
    before = binding.launch_count()
    st = L.swat_attn_bwd(FAKE, FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, FAKE,
                         1, 2, 2, 16, 64, 4, 0, 1, None, 1e4, 0, None)   # softmax needs o, lse
    assert st == -1
    st = L.swat_attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                         1, 2, 2, 16, 64, 4, 0, 0, None, 1e4, 0, None)   # no workspace
    assert st == -1
    st = L.swa_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, FAKE,
                           2, 4, 2, 64, 16, 2, 1, None, 1e4, 0, None)    # sinks but no sink buffers
    assert st == -1
    st = L.swa_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, FAKE,
                           2, 36, 2, 64, 16, 0, 1, None, 1e4, 0, None)   # group of 18 heads
    assert st == -2
    st = L.swa_cache_fill(FAKE, FAKE, FAKE, FAKE, None, None, 1, 2, 8, 64, 0, 0, 0, 1e4, 0, None)
    assert st == -1                                                      # window 0
    assert binding.launch_count() == before


def test_check_wait_timeout_rejects_bad_limits_before_launch(L):
    n0 = binding.launch_count()
    for bad in (0, 999, 2_000_000_001, -5):
        assert L.swat_check_wait_timeout(bad, None) == -1
    assert binding.launch_count() == n0
