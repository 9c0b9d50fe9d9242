"""ctypes binding of libllama_attn.so: the same entry points, torch tensors in.

Argument marshalling only: tensors become device pointers, the current torch
CUDA stream becomes ``cuda_stream``, outputs and workspaces are allocated by
torch when the caller does not pass them, and a non-zero status raises.  Every
step of the computation runs in the library's kernels.  There is no CPU
fallback: without the built library, or on a tensor that is not on a CUDA
device, the call raises.

cos/sin arguments are LLaMA RoPE tables as ``rope_table`` returns them: the
second half of every row repeats the first (the frequencies concatenated with
themselves).  The kernels may read either copy; a table whose halves differ
is not supported (include/llama_attn.h states the same for the C ABI).
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

from . import build as _build

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libllama_attn.so")

LLAMA_DT_F32 = 0
LLAMA_DT_BF16 = 1
LLAMA_OK = 0
LLAMA_ERR_INVALID_ARG = 1
LLAMA_ERR_UNSUPPORTED = 2
LLAMA_ERR_CUDA = 3
LLAMA_ERR_DEVICE_TIMEOUT = 4

# Every symbol include/llama_attn.h declares.
EXPORTED = (
    "llama_rope_table",
    "llama_rope_table_ntk",
    "llama_attn_qkv_rope",
    "llama_attn_out_proj",
    "llama_attn_prefill_workspace_bytes",
    "llama_attn_prefill",
    "llama_attn_prefill_window",
    "llama_attn_prefill_varlen",
    "llama_attn_prefill_packed",
    "llama_attn_decode_workspace_bytes",
    "llama_attn_decode",
    "llama_attn_decode_append",
    "llama_attn_decode_noalloc",
    "llama_attn_device_status",
    "llama_attn_selftest_wait_timeout",
    "llama_attn_selftest_launch_error",
    "llama_attn_status_string",
    "llama_attn_abi_version",
)

_lib = None


class LlamaAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def load() -> ctypes.CDLL:
    """Load the in-tree library.

    Raises if it has not been built, or if it was built from sources other
    than the ones now in the tree (a stale library would silently run old
    kernels).
    """
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m llama_gqa_causal_b200.build`")
    if os.path.abspath(LIB_PATH) == os.path.abspath(_build.LIB) and \
            _build.built_hash() != _build.source_hash():
        raise RuntimeError(
            f"{LIB_PATH} was built from other sources than the ones in the tree: "
            "rebuild it with `python -m llama_gqa_causal_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, D, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_size_t, ctypes.c_float
    lib.llama_rope_table.argtypes = [P, I, I, I, D, D, P, P, P]
    lib.llama_rope_table.restype = I
    lib.llama_rope_table_ntk.argtypes = [P, I, I, I, D, D, P, P, P]
    lib.llama_rope_table_ntk.restype = I
    lib.llama_attn_qkv_rope.argtypes = [P, P, P, P, I, I, I, I, I, P, P, P, I, P]
    lib.llama_attn_qkv_rope.restype = I
    lib.llama_attn_out_proj.argtypes = [P, P, I, I, I, P, I, P]
    lib.llama_attn_out_proj.restype = I
    lib.llama_attn_prefill_workspace_bytes.argtypes = [I, I, I, I, I, I, I]
    lib.llama_attn_prefill_workspace_bytes.restype = Z
    lib.llama_attn_prefill.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, P, P, I, P, Z, P]
    lib.llama_attn_prefill.restype = I
    lib.llama_attn_prefill_window.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, P, I, P, Z, P]
    lib.llama_attn_prefill_window.restype = I
    lib.llama_attn_prefill_varlen.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, P, I, P, Z, P]
    lib.llama_attn_prefill_varlen.restype = I
    lib.llama_attn_prefill_packed.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, I, P, I, P, Z, P]
    lib.llama_attn_prefill_packed.restype = I
    lib.llama_attn_decode_workspace_bytes.argtypes = [I, I, I, I]
    lib.llama_attn_decode_workspace_bytes.restype = Z
    lib.llama_attn_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, P, P, Z, I, P]
    lib.llama_attn_decode.restype = I
    lib.llama_attn_decode_append.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, F, P, P, Z, I, P]
    lib.llama_attn_decode_append.restype = I
    lib.llama_attn_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, P, I, P]
    lib.llama_attn_decode_noalloc.restype = I
    lib.llama_attn_device_status.argtypes = [P]
    lib.llama_attn_device_status.restype = I
    lib.llama_attn_selftest_wait_timeout.argtypes = [ctypes.c_uint, P]
    lib.llama_attn_selftest_wait_timeout.restype = I
    lib.llama_attn_selftest_launch_error.argtypes = [P]
    lib.llama_attn_selftest_launch_error.restype = I
    lib.llama_attn_status_string.argtypes = [I]
    lib.llama_attn_status_string.restype = ctypes.c_char_p
    lib.llama_attn_abi_version.argtypes = []
    lib.llama_attn_abi_version.restype = I
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().llama_attn_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != LLAMA_OK:
        raise LlamaAttnError(status, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("llama_attn: tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("llama_attn: tensors must be contiguous")
    return t.data_ptr()


def _need(t: Optional[torch.Tensor], where: str, name: str, dtype: torch.dtype,
          device: torch.device, shape=None, numel: Optional[int] = None) -> None:
    """Reject a tensor whose dtype, device or size disagrees with the sizes the
    entry point is given (the C ABI sees only pointers: a short buffer would be
    read or written past its end)."""
    if t is None:
        return
    if t.dtype != dtype:
        raise ValueError(f"{where}: {name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{where}: {name} is on {t.device}, expected {device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{where}: {name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{where}: {name} must hold {numel} elements, got {t.numel()}")


def _tables(cos, sin, where, device, rows, D) -> None:
    if (cos is None) != (sin is None):
        raise ValueError(f"{where}: pass both cos and sin, or neither")
    _need(cos, where, "cos", torch.float32, device, numel=rows * D)
    _need(sin, where, "sin", torch.float32, device, numel=rows * D)


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return LLAMA_DT_BF16
    if dt == torch.float32:
        return LLAMA_DT_F32
    raise ValueError(f"llama_attn: unsupported dtype {dt}")


def rope_table(pos: torch.Tensor, head_dim: int, theta: float = 10000.0,
               factor: float = 1.0, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """cos, sin [*pos.shape, head_dim] fp32 from int64 positions (llama_rope_table)."""
    lib = load()
    pos = pos.to(torch.int64).contiguous()
    n = pos.numel()
    cos = torch.empty(*pos.shape, head_dim, device=pos.device, dtype=torch.float32)
    sin = torch.empty_like(cos)
    bsz = pos.shape[0] if pos.dim() > 1 else 1
    seq = n // bsz
    _check(lib.llama_rope_table(_ptr(pos), bsz, seq, head_dim, float(theta), float(factor),
                                _ptr(cos), _ptr(sin), _stream(stream)), "llama_rope_table")
    return cos, sin


def rope_table_ntk(pos: torch.Tensor, head_dim: int, theta: float = 10000.0, alpha: float = 1.0,
                   stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """cos, sin of the NTK-aware scaled table (llama_rope_table_ntk)."""
    lib = load()
    pos = pos.to(torch.int64).contiguous()
    n = pos.numel()
    cos = torch.empty(*pos.shape, head_dim, device=pos.device, dtype=torch.float32)
    sin = torch.empty_like(cos)
    bsz = pos.shape[0] if pos.dim() > 1 else 1
    seq = n // bsz
    _check(lib.llama_rope_table_ntk(_ptr(pos), bsz, seq, head_dim, float(theta), float(alpha),
                                    _ptr(cos), _ptr(sin), _stream(stream)), "llama_rope_table_ntk")
    return cos, sin


def qkv_rope(x: torch.Tensor, w_qkv: torch.Tensor, n_heads: int, n_kv_heads: int, head_dim: int,
             cos: Optional[torch.Tensor] = None, sin: Optional[torch.Tensor] = None, *,
             out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None,
             stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """llama_attn_qkv_rope.  x [T, hidden], w_qkv [(H+2Hkv)D, hidden] -> q [T,H,D], k, v [T,Hkv,D]."""
    lib = load()
    T, hidden = x.shape
    w = "llama_attn_qkv_rope"
    _need(w_qkv, w, "w_qkv", x.dtype, x.device, shape=((n_heads + 2 * n_kv_heads) * head_dim, hidden))
    _tables(cos, sin, w, x.device, T, head_dim)
    if out is None:
        q = torch.empty(T, n_heads, head_dim, device=x.device, dtype=x.dtype)
        k = torch.empty(T, n_kv_heads, head_dim, device=x.device, dtype=x.dtype)
        v = torch.empty_like(k)
    else:
        q, k, v = out
        _need(q, w, "q", x.dtype, x.device, numel=T * n_heads * head_dim)
        _need(k, w, "k", x.dtype, x.device, numel=T * n_kv_heads * head_dim)
        _need(v, w, "v", x.dtype, x.device, numel=T * n_kv_heads * head_dim)
    _check(lib.llama_attn_qkv_rope(_ptr(x), _ptr(w_qkv), _ptr(cos), _ptr(sin), T, hidden, n_heads,
                                   n_kv_heads, head_dim, _ptr(q), _ptr(k), _ptr(v),
                                   _dtype_code(x.dtype), _stream(stream)), "llama_attn_qkv_rope")
    return q, k, v


def out_proj(attn: torch.Tensor, w_o: torch.Tensor, *, out: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    """llama_attn_out_proj.  attn [T, in], w_o [out, in] -> y [T, out]."""
    lib = load()
    attn2 = attn.reshape(attn.shape[0], -1)
    T, d_in = attn2.shape
    d_out = w_o.shape[0]
    _need(w_o, "llama_attn_out_proj", "w_o", attn.dtype, attn.device, shape=(d_out, d_in))
    if out is None:
        out = torch.empty(T, d_out, device=attn.device, dtype=attn.dtype)
    _need(out, "llama_attn_out_proj", "out", attn.dtype, attn.device, numel=T * d_out)
    _check(lib.llama_attn_out_proj(_ptr(attn2), _ptr(w_o), T, d_in, d_out, _ptr(out),
                                   _dtype_code(attn.dtype), _stream(stream)), "llama_attn_out_proj")
    return out


def prefill_workspace_bytes(bsz, n_heads, n_kv_heads, seq, head_dim, dtype, has_rope) -> int:
    return int(load().llama_attn_prefill_workspace_bytes(
        bsz, n_heads, n_kv_heads, seq, head_dim, _dtype_code(dtype), int(bool(has_rope))))


def decode_workspace_bytes(bsz, n_heads, max_cache_len, head_dim) -> int:
    return int(load().llama_attn_decode_workspace_bytes(bsz, n_heads, max_cache_len, head_dim))


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
            cos: Optional[torch.Tensor] = None, sin: Optional[torch.Tensor] = None, *,
            causal: bool = True, scale: Optional[float] = None,
            mask: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
            workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """llama_attn_prefill.  q [b,S,H,D], k/v [b,S,Hkv,D] -> out [b, S, H*D]."""
    lib = load()
    b, S, H, D = q.shape
    Hkv = k.shape[2]
    _need(k, "llama_attn_prefill", "k", q.dtype, q.device, shape=(b, S, Hkv, D))
    _need(v, "llama_attn_prefill", "v", q.dtype, q.device, shape=(b, S, Hkv, D))
    _tables(cos, sin, "llama_attn_prefill", q.device, b * S, D)
    _need(out, "llama_attn_prefill", "out", q.dtype, q.device, numel=b * S * H * D)
    _need(mask, "llama_attn_prefill", "mask", torch.float32, q.device, numel=b * S * S)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(b, S, H * D, device=q.device, dtype=q.dtype)
    need = prefill_workspace_bytes(b, H, Hkv, S, D, q.dtype, cos is not None)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.llama_attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(cos), _ptr(sin), b, H, Hkv, S,
                                  D, float(scale), int(bool(causal)), _ptr(out), _ptr(mask),
                                  _dtype_code(q.dtype), _ptr(workspace), ws_bytes,
                                  _stream(stream)), "llama_attn_prefill")
    return out


def prefill_window(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                   cos: Optional[torch.Tensor] = None, sin: Optional[torch.Tensor] = None, *,
                   window: int, scale: Optional[float] = None,
                   out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """llama_attn_prefill_window.  Causal; query i sees keys i - window < j <= i."""
    lib = load()
    b, S, H, D = q.shape
    Hkv = k.shape[2]
    _need(k, "llama_attn_prefill_window", "k", q.dtype, q.device, shape=(b, S, Hkv, D))
    _need(v, "llama_attn_prefill_window", "v", q.dtype, q.device, shape=(b, S, Hkv, D))
    _tables(cos, sin, "llama_attn_prefill_window", q.device, b * S, D)
    _need(out, "llama_attn_prefill_window", "out", q.dtype, q.device, numel=b * S * H * D)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(b, S, H * D, device=q.device, dtype=q.dtype)
    need = prefill_workspace_bytes(b, H, Hkv, S, D, q.dtype, cos is not None)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.llama_attn_prefill_window(_ptr(q), _ptr(k), _ptr(v), _ptr(cos), _ptr(sin), b, H,
                                         Hkv, S, D, float(scale), int(window), _ptr(out),
                                         _dtype_code(q.dtype), _ptr(workspace), ws_bytes,
                                         _stream(stream)), "llama_attn_prefill_window")
    return out


def prefill_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, seq_lens: torch.Tensor,
                   cos: Optional[torch.Tensor] = None, sin: Optional[torch.Tensor] = None, *,
                   causal: bool = True, scale: Optional[float] = None,
                   out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """llama_attn_prefill_varlen.  Right-padded batch; seq_lens int32 [b] valid rows."""
    lib = load()
    b, S, H, D = q.shape
    Hkv = k.shape[2]
    _need(k, "llama_attn_prefill_varlen", "k", q.dtype, q.device, shape=(b, S, Hkv, D))
    _need(v, "llama_attn_prefill_varlen", "v", q.dtype, q.device, shape=(b, S, Hkv, D))
    _tables(cos, sin, "llama_attn_prefill_varlen", q.device, b * S, D)
    _need(out, "llama_attn_prefill_varlen", "out", q.dtype, q.device, numel=b * S * H * D)
    _need(seq_lens, "llama_attn_prefill_varlen", "seq_lens", torch.int32, q.device, numel=b)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if seq_lens.dtype != torch.int32:
        raise ValueError("llama_attn_prefill_varlen: seq_lens must be int32")
    if out is None:
        out = torch.empty(b, S, H * D, device=q.device, dtype=q.dtype)
    need = prefill_workspace_bytes(b, H, Hkv, S, D, q.dtype, cos is not None)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.llama_attn_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(cos), _ptr(sin),
                                         _ptr(seq_lens), b, H, Hkv, S, D, float(scale),
                                         int(bool(causal)), _ptr(out), _dtype_code(q.dtype),
                                         _ptr(workspace), ws_bytes, _stream(stream)),
           "llama_attn_prefill_varlen")
    return out


def prefill_packed(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                   max_seqlen: int, cos: Optional[torch.Tensor] = None,
                   sin: Optional[torch.Tensor] = None, *, causal: bool = True,
                   scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """llama_attn_prefill_packed.  q [T,H,D], k/v [T,Hkv,D], cu_seqlens int32 [n+1] -> out [T, H*D]."""
    lib = load()
    T, H, D = q.shape
    Hkv = k.shape[1]
    n = cu_seqlens.numel() - 1
    w = "llama_attn_prefill_packed"
    _need(k, w, "k", q.dtype, q.device, shape=(T, Hkv, D))
    _need(v, w, "v", q.dtype, q.device, shape=(T, Hkv, D))
    _tables(cos, sin, w, q.device, T, D)
    _need(out, w, "out", q.dtype, q.device, numel=T * H * D)
    _need(cu_seqlens, w, "cu_seqlens", torch.int32, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("llama_attn_prefill_packed: cu_seqlens must be int32")
    if out is None:
        out = torch.empty(T, H * D, device=q.device, dtype=q.dtype)
    need = prefill_workspace_bytes(1, H, Hkv, T, D, q.dtype, cos is not None)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.llama_attn_prefill_packed(_ptr(q), _ptr(k), _ptr(v), _ptr(cos), _ptr(sin),
                                         _ptr(cu_seqlens), n, T, int(max_seqlen), H, Hkv, D,
                                         float(scale), int(bool(causal)), _ptr(out),
                                         _dtype_code(q.dtype), _ptr(workspace), ws_bytes,
                                         _stream(stream)), "llama_attn_prefill_packed")
    return out


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
           cache_lens: torch.Tensor, cos: Optional[torch.Tensor] = None,
           sin: Optional[torch.Tensor] = None, *, scale: Optional[float] = None,
           out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
           stream=None) -> torch.Tensor:
    """llama_attn_decode.  q [b,H,D], caches [b,Hkv,L,D], cache_lens int32 [b] -> out [b, H*D]."""
    lib = load()
    b, H, D = q.shape
    Hkv, L = k_cache.shape[1], k_cache.shape[2]
    _need(k_cache, "llama_attn_decode", "k_cache", q.dtype, q.device, shape=(b, Hkv, L, D))
    _need(v_cache, "llama_attn_decode", "v_cache", q.dtype, q.device, shape=(b, Hkv, L, D))
    _need(cache_lens, "llama_attn_decode", "cache_lens", torch.int32, q.device, numel=b)
    _tables(cos, sin, "llama_attn_decode", q.device, b, D)
    _need(out, "llama_attn_decode", "out", q.dtype, q.device, numel=b * H * D)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(b, H * D, device=q.device, dtype=q.dtype)
    if workspace is None:
        workspace = torch.empty(decode_workspace_bytes(b, H, L, D), device=q.device,
                                dtype=torch.uint8)
    ws_bytes = workspace.numel() * workspace.element_size()
    if cache_lens.dtype != torch.int32:
        raise ValueError("llama_attn_decode: cache_lens must be int32")
    _check(lib.llama_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens),
                                 _ptr(cos), _ptr(sin), b, H, Hkv, L, D, float(scale), _ptr(out),
                                 _ptr(workspace), ws_bytes, _dtype_code(q.dtype),
                                 _stream(stream)), "llama_attn_decode")
    return out


def decode_append(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                  k_cache: torch.Tensor, v_cache: torch.Tensor, cache_lens: torch.Tensor,
                  cos: Optional[torch.Tensor] = None, sin: Optional[torch.Tensor] = None, *,
                  scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """llama_attn_decode_append.  q [b,H,D], k_new/v_new [b,Hkv,D] (k_new not rotated),
    caches [b,Hkv,L,D] (written at row min(cache_lens[b], L-1)), cache_lens int32 [b]
    (read only) -> out [b, H*D]."""
    lib = load()
    b, H, D = q.shape
    Hkv, L = k_cache.shape[1], k_cache.shape[2]
    _need(k_cache, "llama_attn_decode_append", "k_cache", q.dtype, q.device, shape=(b, Hkv, L, D))
    _need(v_cache, "llama_attn_decode_append", "v_cache", q.dtype, q.device, shape=(b, Hkv, L, D))
    _need(cache_lens, "llama_attn_decode_append", "cache_lens", torch.int32, q.device, numel=b)
    _tables(cos, sin, "llama_attn_decode_append", q.device, b, D)
    _need(out, "llama_attn_decode_append", "out", q.dtype, q.device, numel=b * H * D)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(b, H * D, device=q.device, dtype=q.dtype)
    if workspace is None:
        workspace = torch.empty(decode_workspace_bytes(b, H, L, D), device=q.device,
                                dtype=torch.uint8)
    ws_bytes = workspace.numel() * workspace.element_size()
    if cache_lens.dtype != torch.int32:
        raise ValueError("llama_attn_decode_append: cache_lens must be int32")
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        if tuple(t.shape) != (b, Hkv, D) or not t.is_contiguous():
            raise ValueError(f"llama_attn_decode_append: {name} must be contiguous [b, Hkv, D]")
    _check(lib.llama_attn_decode_append(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                        _ptr(v_cache), _ptr(cache_lens), _ptr(cos), _ptr(sin), b, H,
                                        Hkv, L, D, float(scale), _ptr(out), _ptr(workspace),
                                        ws_bytes, _dtype_code(q.dtype), _stream(stream)),
           "llama_attn_decode_append")
    return out


def decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   cache_lens: torch.Tensor, cos: Optional[torch.Tensor] = None,
                   sin: Optional[torch.Tensor] = None, *, scale: Optional[float] = None,
                   out: torch.Tensor, stream=None) -> torch.Tensor:
    """llama_attn_decode_noalloc: decode with the library's static scratch.

    For callers that must not allocate device memory: ``out`` is required
    (shape [b, H*D], same dtype as q) and nothing is allocated here either.
    """
    lib = load()
    b, H, D = q.shape
    Hkv, L = k_cache.shape[1], k_cache.shape[2]
    _need(k_cache, "llama_attn_decode_noalloc", "k_cache", q.dtype, q.device, shape=(b, Hkv, L, D))
    _need(v_cache, "llama_attn_decode_noalloc", "v_cache", q.dtype, q.device, shape=(b, Hkv, L, D))
    _need(cache_lens, "llama_attn_decode_noalloc", "cache_lens", torch.int32, q.device, numel=b)
    _tables(cos, sin, "llama_attn_decode_noalloc", q.device, b, D)
    _need(out, "llama_attn_decode_noalloc", "out", q.dtype, q.device, numel=b * H * D)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if cache_lens.dtype != torch.int32:
        raise ValueError("llama_attn_decode_noalloc: cache_lens must be int32")
    _check(lib.llama_attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens),
                                         _ptr(cos), _ptr(sin), b, H, Hkv, L, D, float(scale),
                                         _ptr(out), _dtype_code(q.dtype), _stream(stream)),
           "llama_attn_decode_noalloc")
    return out


def device_status(stream=None) -> int:
    """llama_attn_device_status: sync the stream, read and clear the device status word."""
    return int(load().llama_attn_device_status(_stream(stream)))


def selftest_wait_timeout(limit_us: int, stream=None) -> int:
    """llama_attn_selftest_wait_timeout: a bounded device wait that runs out (status code)."""
    return int(load().llama_attn_selftest_wait_timeout(int(limit_us), _stream(stream)))


def selftest_launch_error(stream=None) -> int:
    """llama_attn_selftest_launch_error: a launch the runtime refuses (status code)."""
    return int(load().llama_attn_selftest_launch_error(_stream(stream)))
