"""ctypes binding of libswat.so — argument marshalling only.

Every function here checks tensor shapes/dtypes/devices, allocates outputs
with torch when the caller did not pass them, and forwards raw device
pointers and the current CUDA stream to the C ABI of ``include/swat.h``.
All arithmetic happens in the library's CUDA kernels. If the library is
missing, the first call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libswat.so")

MODE_SIGMOID = 0
MODE_SOFTMAX = 1
BF16 = 0
F32 = 1

_STATUS = {0: "SWAT_OK", -1: "SWAT_ERR_INVALID_ARG", -2: "SWAT_ERR_UNSUPPORTED",
           -3: "SWAT_ERR_CUDA", -4: "SWAT_ERR_TIMEOUT", -5: "SWAT_ERR_SCRATCH_LIMIT"}
SCRATCH_LIMIT = -5
NOALLOC_SCRATCH_BYTES = 16 << 20   # SWA_DECODE_NOALLOC_SCRATCH_BYTES

EXPORTED = ["swat_attn_fwd", "swat_attn_fwd_workspace_bytes", "swat_attn_fwd_ws", "swat_attn_bwd_workspace_bytes", "swat_attn_bwd", "swat_attn_bwd_rotated",
            "swa_cache_fill",
            "swa_decode_step", "swa_decode_workspace_bytes", "swa_decode_step_noalloc", "swat_status_string",
            "swat_get_device_status", "swat_launch_count", "swat_check_wait_timeout"]


class SwatError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {status} ({_STATUS.get(status, 'unknown')})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libswat.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libswat.so not found at {LIB_PATH}; build it with "
                           "`python -m sliding_window_sigmoid_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, LL, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong, ctypes.c_size_t
    L.swat_attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, P, F, I, P]
    L.swat_attn_fwd.restype = I
    L.swat_attn_fwd_workspace_bytes.argtypes = [I, I, I, I, I, I]
    L.swat_attn_fwd_workspace_bytes.restype = SZ
    L.swat_attn_fwd_ws.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, F, I, P]
    L.swat_attn_fwd_ws.restype = I
    L.swat_attn_bwd_workspace_bytes.argtypes = [I, I, I, I, I, I]
    L.swat_attn_bwd_workspace_bytes.restype = SZ
    L.swat_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, F, I, P]
    L.swat_attn_bwd.restype = I
    L.swat_attn_bwd_rotated.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, F, I, P]
    L.swat_attn_bwd_rotated.restype = I
    L.swa_cache_fill.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, LL, F, I, P]
    L.swa_cache_fill.restype = I
    L.swa_decode_step.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, F, I, P]
    L.swa_decode_step.restype = I
    L.swa_decode_step_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, F, I, P]
    L.swa_decode_step_noalloc.restype = I
    L.swa_decode_workspace_bytes.argtypes = [I, I, I, I, I]
    L.swa_decode_workspace_bytes.restype = SZ
    L.swat_status_string.argtypes = [I]
    L.swat_status_string.restype = ctypes.c_char_p
    L.swat_get_device_status.argtypes = [P]
    L.swat_get_device_status.restype = I
    L.swat_check_wait_timeout.argtypes = [LL, P]
    L.swat_check_wait_timeout.restype = I
    L.swat_launch_count.argtypes = []
    L.swat_launch_count.restype = LL
    _lib = L
    return L


def _check(fn: str, st: int):
    if st != 0:
        raise SwatError(fn, st)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, shape, dtype, device):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _slopes(slopes, H, device):
    if slopes is None:
        return None
    s = torch.as_tensor(slopes, dtype=torch.float32)
    if s.device != device:
        s = s.to(device)
    s = s.contiguous()
    if s.numel() != H:
        raise ValueError(f"slopes: {s.numel()} values for {H} heads")
    return s


def fwd_workspace_bytes(B, H, Hkv, N, d, dtype=BF16) -> int:
    return int(lib().swat_attn_fwd_workspace_bytes(B, H, Hkv, N, d, dtype))


def attn_fwd(q, k, v, *, window: int, n_sink: int = 0, mode: int = MODE_SIGMOID, slopes=None,
             rope_base: float = 10000.0, out=None, lse=None, workspace=None, stream=None):
    """SWAT forward. q [B,N,H,d], k/v [B,N,Hkv,d] (bf16 or fp32, CUDA).
    Returns (o [B,N,H,d], lse [B,H,N] fp32 or None in sigmoid mode).

    workspace: None allocates one and calls swat_attn_fwd_ws (rotated Q/K
    copies); a uint8 CUDA tensor of fwd_workspace_bytes() is used as given;
    False calls swat_attn_fwd (tiles rotated in shared memory)."""
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    dev = q.device
    _need(k, "k", (B, N, Hkv, d), q.dtype, dev)
    _need(v, "v", (B, N, Hkv, d), q.dtype, dev)
    if out is None:
        out = torch.empty_like(q)
    if mode == MODE_SOFTMAX and lse is None:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    sl = _slopes(slopes, H, dev)
    args = (B, H, Hkv, N, d, window, n_sink, mode, _ptr(sl), float(rope_base), _dtype_code(q),
            _stream(stream))
    if workspace is False:
        st = lib().swat_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), *args)
        _check("swat_attn_fwd", st)
        return out, lse
    if workspace is None:
        nbytes = fwd_workspace_bytes(B, H, Hkv, N, d, _dtype_code(q))
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    st = lib().swat_attn_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(workspace), *args)
    _check("swat_attn_fwd_ws", st)
    return out, lse


def bwd_workspace_bytes(B, H, Hkv, N, d, dtype=BF16) -> int:
    return int(lib().swat_attn_bwd_workspace_bytes(B, H, Hkv, N, d, dtype))


def attn_bwd(q, k, v, o, lse, dout, *, window: int, n_sink: int = 0, mode: int = MODE_SIGMOID,
             slopes=None, rope_base: float = 10000.0, dq=None, dk=None, dv=None, workspace=None,
             qk_rot=None, stream=None):
    """Backward of attn_fwd. Returns (dq, dk, dv).

    qk_rot: the workspace given to attn_fwd for the same q and k (its rotated
    copies are reused: swat_attn_bwd_rotated), or None (swat_attn_bwd)."""
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    dev = q.device
    _need(dout, "dout", (B, N, H, d), q.dtype, dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        nbytes = bwd_workspace_bytes(B, H, Hkv, N, d, _dtype_code(q))
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    sl = _slopes(slopes, H, dev)
    rest = (B, H, Hkv, N, d, window, n_sink, mode, _ptr(sl), float(rope_base), _dtype_code(q),
            _stream(stream))
    if qk_rot is not None:
        st = lib().swat_attn_bwd_rotated(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                         _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), _ptr(qk_rot), *rest)
        _check("swat_attn_bwd_rotated", st)
        return dq, dk, dv
    st = lib().swat_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                             _ptr(dk), _ptr(dv), _ptr(workspace), *rest)
    _check("swat_attn_bwd", st)
    return dq, dk, dv


class RingCache:
    """Device ring-buffer KV cache ([B, Hkv, window, d]) plus sink slots, and the
    decode step over it. Buffers are torch tensors owned by this object."""

    def __init__(self, B, H, Hkv, d, window, n_sink=0, *, mode=MODE_SIGMOID, slopes=None,
                 rope_base=10000.0, dtype=torch.bfloat16, device="cuda"):
        self.B, self.H, self.Hkv, self.d, self.window, self.n_sink = B, H, Hkv, d, window, n_sink
        self.mode, self.rope_base, self.dtype = mode, float(rope_base), dtype
        self.device = torch.device(device)
        if self.device.type == "cuda" and self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        self.k_cache = torch.zeros(B, Hkv, window, d, dtype=dtype, device=self.device)
        self.v_cache = torch.zeros_like(self.k_cache)
        ns = max(n_sink, 1)
        self.k_sink = torch.zeros(B, Hkv, ns, d, dtype=dtype, device=self.device)
        self.v_sink = torch.zeros_like(self.k_sink)
        self.slopes = _slopes(slopes, H, self.device)
        nbytes = int(lib().swa_decode_workspace_bytes(B, H, Hkv, d, window))
        self.workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=self.device)
        self._code = BF16 if dtype == torch.bfloat16 else F32

    def fill(self, k, v, p0: int = 0, stream=None):
        """k, v [B, n_tok, Hkv, d]: raw tokens at positions p0 .. p0+n_tok-1."""
        n_tok = k.shape[1]
        _need(k, "k", (self.B, n_tok, self.Hkv, self.d), self.dtype, self.device)
        _need(v, "v", (self.B, n_tok, self.Hkv, self.d), self.dtype, self.device)
        st = lib().swa_cache_fill(_ptr(k), _ptr(v), _ptr(self.k_cache), _ptr(self.v_cache),
                                  _ptr(self.k_sink), _ptr(self.v_sink), self.B, self.Hkv, n_tok,
                                  self.d, self.window, self.n_sink, int(p0), self.rope_base,
                                  self._code, _stream(stream))
        _check("swa_cache_fill", st)

    def step(self, q, k_new, v_new, pos, out=None, stream=None):
        """q [B,H,d], k_new/v_new [B,Hkv,d], pos [B] int64 (device). Returns o [B,H,d]."""
        _need(q, "q", (self.B, self.H, self.d), self.dtype, self.device)
        _need(k_new, "k_new", (self.B, self.Hkv, self.d), self.dtype, self.device)
        _need(v_new, "v_new", (self.B, self.Hkv, self.d), self.dtype, self.device)
        _need(pos, "pos", (self.B,), torch.int64, self.device)
        out = torch.empty_like(q) if out is None else out
        st = lib().swa_decode_step(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(self.k_cache),
                                   _ptr(self.v_cache), _ptr(self.k_sink), _ptr(self.v_sink),
                                   _ptr(pos), _ptr(out), _ptr(self.workspace), self.B, self.H,
                                   self.Hkv, self.d, self.window, self.n_sink, self.mode,
                                   _ptr(self.slopes), self.rope_base, self._code, _stream(stream))
        _check("swa_decode_step", st)
        return out

    def step_noalloc(self, q, k_new, v_new, pos, out=None, stream=None):
        """The same step through swa_decode_step_noalloc: the library's own
        static scratch buffer instead of this object's workspace (calls that
        can overlap on the device must not use it concurrently)."""
        _need(q, "q", (self.B, self.H, self.d), self.dtype, self.device)
        _need(k_new, "k_new", (self.B, self.Hkv, self.d), self.dtype, self.device)
        _need(v_new, "v_new", (self.B, self.Hkv, self.d), self.dtype, self.device)
        _need(pos, "pos", (self.B,), torch.int64, self.device)
        out = torch.empty_like(q) if out is None else out
        st = lib().swa_decode_step_noalloc(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(self.k_cache),
                                           _ptr(self.v_cache), _ptr(self.k_sink), _ptr(self.v_sink),
                                           _ptr(pos), _ptr(out), self.B, self.H, self.Hkv, self.d,
                                           self.window, self.n_sink, self.mode, _ptr(self.slopes),
                                           self.rope_base, self._code, _stream(stream))
        _check("swa_decode_step_noalloc", st)
        return out


def status_string(code: int) -> str:
    return lib().swat_status_string(int(code)).decode()


def device_status(stream=None) -> int:
    return int(lib().swat_get_device_status(_stream(stream)))


def check_wait_timeout(limit_ns: int, stream=None) -> None:
    """Runs the bounded-wait failure path once (see swat_check_wait_timeout)."""
    _check("swat_check_wait_timeout", lib().swat_check_wait_timeout(int(limit_ns), _stream(stream)))


def launch_count() -> int:
    return int(lib().swat_launch_count())
