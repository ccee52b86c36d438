"""CPU oracle for SWAT sliding-window attention — test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library never does.

Two independent implementations live here:

* ``swat_oracle.c`` (loaded through ctypes): plain fp64 loops with OpenMP over
  rows; the full-size and sampled-row reference.
* ``ref_numpy.py``: dense masked fp64 matrices for tiny sizes, written from
  the pages' mask construction and the complex-number form of RoPE.

Both compute the SWAT attention equation of "SWAT: Sliding Window Attention
Training" (section "Balanced ALiBi"), the softmax-with-sinks SWA(w, s) of
"Sliding-window beats linear attention" and the ring cache of the
"Sliding Window Attention" glossary (ring-buffer paragraph).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swat_oracle.c")
_LIB = os.path.join(_HERE, "libswat_oracle.so")

MODE_SIGMOID = 0
MODE_SOFTMAX = 1


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libswat_oracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        LL = ctypes.c_longlong
        D = ctypes.c_double
        L.oracle_in_keyset.argtypes = [LL, LL, LL, LL]
        L.oracle_in_keyset.restype = I
        L.oracle_keyset_size.argtypes = [LL, LL, LL]
        L.oracle_keyset_size.restype = LL
        L.oracle_rope_rotate.argtypes = [P, I, LL, D]
        L.oracle_rope_rotate_inv.argtypes = [P, I, LL, D]
        L.oracle_sigmoid.argtypes = [D]
        L.oracle_sigmoid.restype = D
        L.oracle_swat_fwd_rows.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P, D, LL, P, P, P]
        L.oracle_swat_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, P, D]
        L.oracle_swat_bwd.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, D]
        L.oracle_swat_bwd_rows.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, P, D,
                                           LL, P, P, LL, P, P, P]
        L.oracle_cache_fill.argtypes = [P, P, P, P, P, P, I, I, I, I, I, LL, LL, D]
        L.oracle_decode_step.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, D]
        L.oracle_num_threads.restype = I
        _lib = L
    return _lib


def _f32(a) -> np.ndarray:
    a = np.asarray(a, dtype=np.float32)
    return np.ascontiguousarray(a)


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def in_keyset(i: int, j: int, window: int, n_sink: int = 0) -> bool:
    return bool(lib().oracle_in_keyset(i, j, window, n_sink))


def keyset_size(i: int, window: int, n_sink: int = 0) -> int:
    return int(lib().oracle_keyset_size(i, window, n_sink))


def sigmoid(x: float) -> float:
    return float(lib().oracle_sigmoid(float(x)))


def rope_rotate(x, pos: int, rope_base: float, inverse: bool = False) -> np.ndarray:
    y = np.array(x, dtype=np.float64, copy=True)
    fn = lib().oracle_rope_rotate_inv if inverse else lib().oracle_rope_rotate
    fn(_ptr(y), y.shape[-1], int(pos), float(rope_base))
    return y


def swat_fwd(q, k, v, *, window: int, n_sink: int = 0, mode: int = MODE_SIGMOID,
             slopes=None, rope_base: float = 10000.0):
    """Full forward. q [B,N,H,d], k/v [B,N,Hkv,d] -> (o [B,N,H,d] f64, lse [B,H,N] f64)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    sl = None if slopes is None else _f32(slopes)
    o = np.zeros((B, N, H, d), np.float64)
    lse = np.zeros((B, H, N), np.float64)
    lib().oracle_swat_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, N, d,
                          window, n_sink, mode, _ptr(sl), float(rope_base))
    return o, lse


def swat_fwd_rows(q, k, v, rows, *, window: int, n_sink: int = 0, mode: int = MODE_SIGMOID,
                  slopes=None, rope_base: float = 10000.0):
    """Forward for sampled rows; rows is an int array [n, 3] of (b, h, i)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    sl = None if slopes is None else _f32(slopes)
    o = np.zeros((rows.shape[0], d), np.float64)
    lse = np.zeros((rows.shape[0],), np.float64)
    lib().oracle_swat_fwd_rows(_ptr(q), _ptr(k), _ptr(v), B, H, Hkv, N, d, window, n_sink, mode,
                               _ptr(sl), float(rope_base), rows.shape[0], _ptr(rows), _ptr(o),
                               _ptr(lse))
    return o, lse


def swat_bwd(q, k, v, dout, *, window: int, n_sink: int = 0, mode: int = MODE_SIGMOID,
             slopes=None, rope_base: float = 10000.0):
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    sl = None if slopes is None else _f32(slopes)
    dq = np.zeros(q.shape, np.float64)
    dk = np.zeros(k.shape, np.float64)
    dv = np.zeros(v.shape, np.float64)
    lib().oracle_swat_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                          B, H, Hkv, N, d, window, n_sink, mode, _ptr(sl), float(rope_base))
    return dq, dk, dv


def swat_bwd_rows(q, k, v, dout, qrows, krows, *, window: int, n_sink: int = 0,
                  mode: int = MODE_SIGMOID, slopes=None, rope_base: float = 10000.0):
    """Backward on sampled rows: qrows [n,3] of (b,h,i) -> dq rows; krows [m,3] of
    (b,kvh,j) -> dk, dv rows."""
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    qrows = np.ascontiguousarray(np.asarray(qrows, dtype=np.int64).reshape(-1, 3))
    krows = np.ascontiguousarray(np.asarray(krows, dtype=np.int64).reshape(-1, 3))
    sl = None if slopes is None else _f32(slopes)
    dq = np.zeros((qrows.shape[0], d), np.float64)
    dk = np.zeros((krows.shape[0], d), np.float64)
    dv = np.zeros((krows.shape[0], d), np.float64)
    lib().oracle_swat_bwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, H, Hkv, N, d, window,
                               n_sink, mode, _ptr(sl), float(rope_base), qrows.shape[0],
                               _ptr(qrows), _ptr(dq), krows.shape[0], _ptr(krows), _ptr(dk),
                               _ptr(dv))
    return dq, dk, dv


class RingCache:
    """fp64 ring-buffer KV cache with sink slots, one per (b, kv head)."""

    def __init__(self, B: int, Hkv: int, d: int, window: int, n_sink: int, rope_base: float):
        self.B, self.Hkv, self.d, self.window, self.n_sink = B, Hkv, d, window, n_sink
        self.rope_base = float(rope_base)
        self.kc = np.zeros((B, Hkv, window, d), np.float64)
        self.vc = np.zeros((B, Hkv, window, d), np.float64)
        self.ks = np.zeros((B, Hkv, max(n_sink, 1), d), np.float64)
        self.vs = np.zeros((B, Hkv, max(n_sink, 1), d), np.float64)

    def fill(self, k, v, p0: int):
        """k, v [B, n_tok, Hkv, d] raw (unrotated) tokens at positions p0 .. p0+n_tok-1."""
        k, v = _f32(k), _f32(v)
        n_tok = k.shape[1]
        lib().oracle_cache_fill(_ptr(self.kc), _ptr(self.vc), _ptr(self.ks), _ptr(self.vs),
                                _ptr(k), _ptr(v), self.B, self.Hkv, self.d, self.window,
                                self.n_sink, int(p0), int(n_tok), self.rope_base)

    def step(self, q, k_new, v_new, pos, *, mode: int = MODE_SIGMOID, slopes=None):
        q, k_new, v_new = _f32(q), _f32(k_new), _f32(v_new)
        B, H, d = q.shape
        pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(B))
        sl = None if slopes is None else _f32(slopes)
        o = np.zeros((B, H, d), np.float64)
        lib().oracle_decode_step(_ptr(self.kc), _ptr(self.vc), _ptr(self.ks), _ptr(self.vs),
                                 _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(pos), _ptr(o), B, H,
                                 self.Hkv, d, self.window, self.n_sink, mode, _ptr(sl),
                                 self.rope_base)
        return o
