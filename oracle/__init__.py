"""fp64 CPU oracle for LLaMA self-attention (prefill and KV-cache decode).

TEST INFRASTRUCTURE.  Only the tests, the package smoke check and the
benchmark's CPU-baseline / reference leg may import this package.  The product
library (``llama_gqa_causal_b200``) never imports, links or calls it, and it
imports nothing from the product.

The arithmetic lives in ``llama_attn_oracle.c`` (plain loops in double,
OpenMP only across independent output rows); this module builds it with gcc
and wraps it with numpy.  ``brute.py`` is a second, independent pure-Python
restatement used to cross-check it on tiny shapes.

Parity status of each function (what pins it, see tests/test_oracle_pins.py):
  rope_cos_sin / rope_rotate : pinned (2-D textbook rotation, norm
      preservation, relative-position property, HF LLaMA rotary embedding and
      apply_rotary_pos_emb as library routines, linear-scaling identity)
  prefill                    : pinned (torch SDPA and HF eager attention as
      library routines, closed forms in tests/golden, GQA/MHA/MQA and
      head-concat invariants, causal invariants, brute force)
  decode                     : pinned (equals the last row of causal prefill,
      row i of prefill equals decode with i+1 cached keys, brute force)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "llama_attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

MAX_HEAD_DIM = 512


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _bind(path: str):
    """Open a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    D = ctypes.c_double
    L = ctypes.c_long
    lib.oracle_rope_cos_sin.argtypes = [P, L, I, D, D, P, P]
    lib.oracle_rope_cos_sin.restype = None
    lib.oracle_rope_ntk_theta.argtypes = [D, D, I]
    lib.oracle_rope_ntk_theta.restype = D
    lib.oracle_rope_rotate.argtypes = [P, L, I, P, P, P]
    lib.oracle_rope_rotate.restype = None
    lib.oracle_prefill.argtypes = [P, P, P, P, I, I, I, I, I, D, D, D, I, P,
                                   I, I, I, I, P, P, I]
    lib.oracle_prefill.restype = I
    lib.oracle_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, D, D, D, P, P, I]
    lib.oracle_decode.restype = I
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = I
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(_LIB)
    return _lib


def _f32(a) -> np.ndarray:
    """Same values as float32 (exact for bf16 and fp32 inputs)."""
    if hasattr(a, "detach"):  # torch tensor
        import torch

        a = a.detach().to("cpu")
        if a.dtype not in (torch.float32,):
            a = a.to(torch.float32)
        a = a.numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data) if a is not None else ctypes.c_void_p(0)


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def rope_cos_sin(pos, head_dim: int, theta: float = 10000.0, factor: float = 1.0):
    """cos, sin [n, head_dim] float64 for int positions ``pos`` (any shape, flattened)."""
    lib = _load()
    p = np.ascontiguousarray(np.asarray(pos).reshape(-1), dtype=np.int64)
    n = p.shape[0]
    c = np.empty((n, head_dim), np.float64)
    s = np.empty((n, head_dim), np.float64)
    lib.oracle_rope_cos_sin(_ptr(p), n, head_dim, float(theta), float(factor), _ptr(c), _ptr(s))
    return c, s


def rope_ntk_theta(theta: float, alpha: float, head_dim: int) -> float:
    """Base of the NTK-aware scaled table: theta * alpha^(D / (D - 2))."""
    lib = _load()
    return float(lib.oracle_rope_ntk_theta(float(theta), float(alpha), int(head_dim)))


def rope_cos_sin_ntk(pos, head_dim: int, theta: float = 10000.0, alpha: float = 1.0):
    """cos, sin [n, head_dim] float64 of the NTK-aware scaled table."""
    return rope_cos_sin(pos, head_dim, rope_ntk_theta(theta, alpha, head_dim), 1.0)


def rope_rotate(x, cos, sin):
    """x * cos + rotate_half(x) * sin for rows of x ([n, D], float64)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    D = x.shape[-1]
    xs = x.reshape(-1, D)
    c = np.ascontiguousarray(np.broadcast_to(cos, x.shape), dtype=np.float64).reshape(-1, D)
    s = np.ascontiguousarray(np.broadcast_to(sin, x.shape), dtype=np.float64).reshape(-1, D)
    y = np.empty_like(xs)
    lib.oracle_rope_rotate(_ptr(xs), xs.shape[0], D, _ptr(c), _ptr(s), _ptr(y))
    return y.reshape(x.shape)


def prefill(q, k, v, pos=None, *, theta=10000.0, factor=1.0, scale=None, causal=True,
            mask=None, heads=None, rows=None, return_probs=False, nthreads=0):
    """Full-sequence attention.  q [b,S,H,D], k/v [b,S,Hkv,D] (torch or numpy).

    pos: [b,S] int positions or None (no RoPE).  mask: [b,1,S,S] additive or None.
    heads / rows: optional (lo, hi) ranges to compute; other outputs are NaN.
    Returns out [b, S, H*D] float64 (and probs [b,H,S,S] when requested).
    """
    lib = _load()
    qf, kf, vf = _f32(q), _f32(k), _f32(v)
    b, S, H, D = qf.shape
    Hkv = kf.shape[2]
    if D > MAX_HEAD_DIM:
        raise ValueError("head_dim too large for the oracle")
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    p = None if pos is None else np.ascontiguousarray(np.asarray(pos).reshape(b, S), dtype=np.int64)
    m = None if mask is None else _f32(mask).reshape(b, 1, S, S)
    h_lo, h_hi = heads if heads is not None else (0, H)
    i_lo, i_hi = rows if rows is not None else (0, S)
    out = np.full((b, S, H * D), np.nan, np.float64)
    probs = np.zeros((b, H, S, S), np.float64) if return_probs else None
    rc = lib.oracle_prefill(_ptr(qf), _ptr(kf), _ptr(vf), _ptr(p), b, H, Hkv, S, D,
                            float(theta), float(factor), float(scale), int(bool(causal)),
                            _ptr(m), h_lo, h_hi, i_lo, i_hi, _ptr(out), _ptr(probs),
                            int(nthreads))
    if rc != 0:
        raise ValueError("oracle_prefill rejected its arguments")
    return (out, probs) if return_probs else out


def decode(q, k_cache, v_cache, lens, qpos=None, *, theta=10000.0, factor=1.0, scale=None,
           return_probs=False, nthreads=0):
    """Single-token decode.  q [b,H,D] un-rotated, caches [b,Hkv,L,D] (rotated keys).

    lens: [b] cached lengths; qpos: [b] query positions or None (no RoPE).
    Returns out [b, H*D] float64 (and probs [b,H,L]).
    """
    lib = _load()
    qf, kf, vf = _f32(q), _f32(k_cache), _f32(v_cache)
    b, H, D = qf.shape
    Hkv, L = kf.shape[1], kf.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    ln = np.ascontiguousarray(np.asarray(lens).reshape(b), dtype=np.int32)
    qp = None if qpos is None else np.ascontiguousarray(np.asarray(qpos).reshape(b), dtype=np.int64)
    out = np.empty((b, H * D), np.float64)
    probs = np.zeros((b, H, L), np.float64) if return_probs else None
    rc = lib.oracle_decode(_ptr(qf), _ptr(kf), _ptr(vf), _ptr(ln), _ptr(qp), b, H, Hkv, L, D,
                           float(theta), float(factor), float(scale), _ptr(out), _ptr(probs),
                           int(nthreads))
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    return (out, probs) if return_probs else out
