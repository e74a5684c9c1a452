"""Thin ctypes binding of libarkattn (``include/arkattn.h``).

Each ``ark_attn_*`` function here has the name and the meaning of the C entry
point it forwards to; it only derives sizes from tensor shapes, checks dtype /
device / contiguity, and passes ``data_ptr()`` and the current CUDA stream.
All compute happens in the library's CUDA kernels.  There is no fallback: if
``libarkattn.so`` is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libarkattn.so")

ARK_OK = 0
ARK_ERR_INVALID_ARG = 1
ARK_ERR_UNSUPPORTED = 2
ARK_ERR_WORKSPACE = 3
ARK_ERR_CUDA = 4
ARK_ERR_TIMEOUT = 5

ARK_LENGTH_AWARE = 0
ARK_MASKED_STATIC = 1

ARK_DEV_BAD_POS = 1
ARK_DEV_BAD_KVLEN = 2
ARK_DEV_TIMEOUT = 4

ARK_MAX_LAYERS = 64

# every symbol include/arkattn.h declares
EXPORTS = (
    "ark_attn_status_string",
    "ark_attn_rope_table_bytes",
    "ark_attn_rope_table_init",
    "ark_attn_append_rope",
    "ark_attn_decode_workspace_size",
    "ark_attn_decode",
    "ark_attn_combine",
    "ark_attn_prefill",
    "ark_attn_append_rope_layers",
    "ark_attn_decode_layers_workspace_size",
    "ark_attn_decode_layers",
    "ark_attn_decode_noalloc_scratch_bytes",
    "ark_attn_decode_noalloc",
    "ark_attn_append_rope_fp8",
    "ark_attn_append_rope_fp8_layers",
    "ark_attn_decode_fp8",
    "ark_attn_decode_fp8_layers",
    "ark_attn_prefill_layers",
    "ark_attn_append_rope_kv",
    "ark_attn_append_rope_kv_layers",
    "ark_attn_prefill_rope",
    "ark_attn_prefill_rope_layers",
    "ark_attn_encoder",
    "ark_attn_qkv_proj",
    "ark_attn_qkv_rope_append",
)


class ArkError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


_lib = None


def load() -> ctypes.CDLL:
    """Load libarkattn.so (built in-tree by ``gqa_attention_static_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libarkattn.so is not built ({LIB_PATH}); run "
                           "`python -m gqa_attention_static_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.ark_attn_status_string.argtypes = [I]
    lib.ark_attn_status_string.restype = ctypes.c_char_p
    lib.ark_attn_rope_table_bytes.argtypes = [I, I]
    lib.ark_attn_rope_table_bytes.restype = Z
    lib.ark_attn_rope_table_init.argtypes = [P, I, I, ctypes.c_double, P]
    lib.ark_attn_rope_table_init.restype = I
    lib.ark_attn_append_rope.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P]
    lib.ark_attn_append_rope.restype = I
    lib.ark_attn_decode_workspace_size.argtypes = [I, I, I, I, I]
    lib.ark_attn_decode_workspace_size.restype = Z
    lib.ark_attn_decode.argtypes = [P, P, P, P, I, I, I, I, I, ctypes.c_float, I, I, P, Z, P, P, P, P]
    lib.ark_attn_decode.restype = I
    lib.ark_attn_combine.argtypes = [P, P, I, I, I, I, P, P, P]
    lib.ark_attn_combine.restype = I
    lib.ark_attn_prefill.argtypes = [P, P, P, P, P, I, I, I, I, I, I, ctypes.c_float, P, P, P, P]
    lib.ark_attn_prefill.restype = I
    PP = ctypes.POINTER(ctypes.c_void_p)
    lib.ark_attn_append_rope_layers.argtypes = [I, PP, PP, PP, PP, PP, P, P, I, I, I, I, I, I, P, P, P]
    lib.ark_attn_append_rope_layers.restype = I
    lib.ark_attn_decode_layers_workspace_size.argtypes = [I, I, I, I, I, I]
    lib.ark_attn_decode_layers_workspace_size.restype = Z
    lib.ark_attn_decode_layers.argtypes = [I, PP, PP, PP, P, I, I, I, I, I, ctypes.c_float, I, I, P, Z,
                                           PP, PP, P, P]
    lib.ark_attn_decode_layers.restype = I
    lib.ark_attn_decode_noalloc_scratch_bytes.argtypes = []
    lib.ark_attn_decode_noalloc_scratch_bytes.restype = Z
    lib.ark_attn_decode_noalloc.argtypes = [P, P, P, P, I, I, I, I, I, ctypes.c_float, I, I, P, P, P, P]
    lib.ark_attn_decode_noalloc.restype = I
    lib.ark_attn_append_rope_fp8.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P]
    lib.ark_attn_append_rope_fp8.restype = I
    lib.ark_attn_append_rope_fp8_layers.argtypes = [I, PP, PP, PP, PP, PP, PP, PP, P, P, I, I, I, I, I, I, P, P,
                                                    P]
    lib.ark_attn_append_rope_fp8_layers.restype = I
    lib.ark_attn_decode_fp8.argtypes = [P, P, P, P, P, P, I, I, I, I, I, ctypes.c_float, I, I, P, Z, P, P, P, P]
    lib.ark_attn_decode_fp8.restype = I
    lib.ark_attn_decode_fp8_layers.argtypes = [I, PP, PP, PP, PP, PP, P, I, I, I, I, I, ctypes.c_float, I, I, P,
                                               Z, PP, PP, P, P]
    lib.ark_attn_decode_fp8_layers.restype = I
    lib.ark_attn_prefill_layers.argtypes = [I, PP, PP, PP, P, P, I, I, I, I, I, I, ctypes.c_float, PP, PP, P, P]
    lib.ark_attn_prefill_layers.restype = I
    lib.ark_attn_append_rope_kv.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, P, P]
    lib.ark_attn_append_rope_kv.restype = I
    lib.ark_attn_append_rope_kv_layers.argtypes = [I, PP, PP, PP, PP, P, P, I, I, I, I, I, I, P, P, P]
    lib.ark_attn_append_rope_kv_layers.restype = I
    lib.ark_attn_prefill_rope.argtypes = [P, P, P, P, P, I, I, I, I, I, I, ctypes.c_float, P, P, P, P, P]
    lib.ark_attn_prefill_rope.restype = I
    lib.ark_attn_prefill_rope_layers.argtypes = [I, PP, PP, PP, P, P, I, I, I, I, I, I, ctypes.c_float, P, PP, PP,
                                                 P, P]
    lib.ark_attn_prefill_rope_layers.restype = I
    lib.ark_attn_encoder.argtypes = [P, P, P, P, I, I, I, I, ctypes.c_float, P, P, P, P]
    lib.ark_attn_encoder.restype = I
    lib.ark_attn_qkv_proj.argtypes = [P, P, P, I, I, I, P, P, P]
    lib.ark_attn_qkv_proj.restype = I
    lib.ark_attn_qkv_rope_append.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P, P]
    lib.ark_attn_qkv_rope_append.restype = I
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().ark_attn_status_string(int(code)).decode()


def _raise(code: int, what: str) -> None:
    if code != ARK_OK:
        raise ArkError(code, what)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype, ndim: Optional[int] = None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")


# ------------------------------------------------------------------ RoPE ----

def ark_attn_rope_table_bytes(T: int, D: int = 128) -> int:
    return int(load().ark_attn_rope_table_bytes(T, D))


def ark_attn_rope_table_init(table: torch.Tensor, T: int, D: int = 128, rope_theta: float = 1e6,
                             stream=None) -> None:
    _need(table, "table", torch.float32)
    if table.numel() * 4 < ark_attn_rope_table_bytes(T, D):
        raise ValueError("table too small")
    _raise(load().ark_attn_rope_table_init(_ptr(table), T, D, float(rope_theta), _stream(stream)),
           "ark_attn_rope_table_init")


def rope_table(T: int, D: int = 128, rope_theta: float = 1e6, device="cuda") -> torch.Tensor:
    """Allocate and fill a rotary table [T, D/2, 2] (fp32 cos, sin)."""
    t = torch.empty((T, D // 2, 2), dtype=torch.float32, device=device)
    ark_attn_rope_table_init(t, T, D, rope_theta)
    return t


# --------------------------------------------------------- RoPE + append ----

def ark_attn_append_rope(q, k_new, v_new, cache_k, cache_v, pos0, n_new, table,
                         status: Optional[torch.Tensor] = None, stream=None) -> None:
    """q [B,S,Hq,D] (rotated in place), k_new/v_new [B,S,Hkv,D] -> rows
    pos0[b] + t of cache_k/cache_v [B,T,Hkv,D]."""
    for name, t in (("q", q), ("k_new", k_new), ("v_new", v_new), ("cache_k", cache_k),
                    ("cache_v", cache_v)):
        _need(t, name, torch.bfloat16, 4)
    _need(pos0, "pos0", torch.int32, 1)
    _need(n_new, "n_new", torch.int32, 1)
    _need(table, "table", torch.float32)
    if status is not None:
        _need(status, "status", torch.int32)
    B, S, Hq, D = q.shape
    T, Hkv = cache_k.shape[1], cache_k.shape[2]
    if tuple(k_new.shape) != (B, S, Hkv, D) or tuple(v_new.shape) != (B, S, Hkv, D):
        raise ValueError("k_new/v_new shape")
    if tuple(cache_v.shape) != tuple(cache_k.shape) or cache_k.shape[0] != B or cache_k.shape[3] != D:
        raise ValueError("cache shape")
    if table.numel() < T * (D // 2) * 2:
        raise ValueError("rotary table has fewer than T rows")
    _raise(load().ark_attn_append_rope(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(cache_k), _ptr(cache_v),
                                       _ptr(pos0), _ptr(n_new), B, S, T, Hq, Hkv, D, _ptr(table),
                                       _ptr(status), _stream(stream)),
           "ark_attn_append_rope")


# ---------------------------------------------------------------- decode ----

def ark_attn_decode_workspace_size(B: int, Hq: int, D: int, T: int, max_splits: int) -> int:
    return int(load().ark_attn_decode_workspace_size(B, Hq, D, T, max_splits))


def ark_attn_decode(q, cache_k, cache_v, kv_len, o, lse, scale: float, mode: int = ARK_LENGTH_AWARE,
                    max_splits: int = 8, workspace: Optional[torch.Tensor] = None,
                    status: Optional[torch.Tensor] = None, stream=None) -> None:
    """q [B,1,Hq,D] -> o [B,1,Hq,D] bf16, lse [B,Hq] fp32 over kv_len[b] rows."""
    _need(q, "q", torch.bfloat16, 4)
    _need(cache_k, "cache_k", torch.bfloat16, 4)
    _need(cache_v, "cache_v", torch.bfloat16, 4)
    _need(kv_len, "kv_len", torch.int32, 1)
    _need(o, "o", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32)
    B, S, Hq, D = q.shape
    if S != 1:
        raise ValueError("decode takes one query row per request")
    T, Hkv = cache_k.shape[1], cache_k.shape[2]
    if tuple(o.shape) != tuple(q.shape) or lse.numel() != B * Hq:
        raise ValueError("o/lse shape")
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", workspace.dtype)
        ws_bytes = workspace.numel() * workspace.element_size()
    if status is not None:
        _need(status, "status", torch.int32)
    _raise(load().ark_attn_decode(_ptr(q), _ptr(cache_k), _ptr(cache_v), _ptr(kv_len), B, T, Hq, Hkv, D,
                                  float(scale), int(mode), int(max_splits), _ptr(workspace), ws_bytes,
                                  _ptr(o), _ptr(lse), _ptr(status), _stream(stream)),
           "ark_attn_decode")


def decode_workspace(B: int, Hq: int, D: int, T: int, max_splits: int, device="cuda", layers: int = 1):
    """Decode workspace (it needs no initialisation), or None when the call
    needs none."""
    n = ark_attn_decode_layers_workspace_size(layers, B, Hq, D, T, max_splits)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device) if n else None


# --------------------------------------------------------------- combine ----

def ark_attn_combine(o_part, lse_part, o, lse, stream=None) -> None:
    """o_part [B,Hq,nsplit,D] fp32, lse_part [B,Hq,nsplit] fp32 -> o [B,Hq,D]
    bf16 (any shape with that many elements), lse [B,Hq] fp32."""
    _need(o_part, "o_part", torch.float32, 4)
    _need(lse_part, "lse_part", torch.float32, 3)
    _need(o, "o", torch.bfloat16)
    _need(lse, "lse", torch.float32)
    B, Hq, nsplit, D = o_part.shape
    if tuple(lse_part.shape) != (B, Hq, nsplit) or o.numel() != B * Hq * D or lse.numel() != B * Hq:
        raise ValueError("combine shapes")
    _raise(load().ark_attn_combine(_ptr(o_part), _ptr(lse_part), B, Hq, nsplit, D, _ptr(o), _ptr(lse),
                                   _stream(stream)),
           "ark_attn_combine")


# --------------------------------------------------------------- prefill ----

def ark_attn_prefill(q, cache_k, cache_v, pos0, n_new, o, lse, scale: float,
                     status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Causal prefill: q [B,S,Hq,D] (rotated) over the cache -> o [B,S,Hq,D]
    bf16 (rows t >= n_new[b] untouched), lse [B,Hq,S] fp32."""
    _need(q, "q", torch.bfloat16, 4)
    _need(cache_k, "cache_k", torch.bfloat16, 4)
    _need(cache_v, "cache_v", torch.bfloat16, 4)
    _need(pos0, "pos0", torch.int32, 1)
    _need(n_new, "n_new", torch.int32, 1)
    _need(o, "o", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32)
    if status is not None:
        _need(status, "status", torch.int32)
    B, S, Hq, D = q.shape
    T, Hkv = cache_k.shape[1], cache_k.shape[2]
    if tuple(o.shape) != tuple(q.shape) or lse.numel() != B * Hq * S:
        raise ValueError("o/lse shape")
    if tuple(cache_v.shape) != tuple(cache_k.shape) or cache_k.shape[0] != B:
        raise ValueError("cache shape")
    _raise(load().ark_attn_prefill(_ptr(q), _ptr(cache_k), _ptr(cache_v), _ptr(pos0), _ptr(n_new), B, S, T, Hq,
                                   Hkv, D, float(scale), _ptr(o), _ptr(lse), _ptr(status), _stream(stream)),
           "ark_attn_prefill")


# ------------------------------------------------- layer-batched variants ----

def _ptr_array(ts: Sequence[torch.Tensor]):
    arr = (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])
    return arr


def ark_attn_append_rope_layers(q: Sequence[torch.Tensor], k_new, v_new, cache_k, cache_v, pos0, n_new, table,
                                status: Optional[torch.Tensor] = None, stream=None) -> None:
    """ark_attn_append_rope over L independent layers in one launch (lists of
    per-layer tensors, same shapes as the single-layer call)."""
    L = len(q)
    if not (len(k_new) == len(v_new) == len(cache_k) == len(cache_v) == L) or L == 0:
        raise ValueError("per-layer lists must have the same non-zero length")
    for i in range(L):
        for name, t in (("q", q[i]), ("k_new", k_new[i]), ("v_new", v_new[i]), ("cache_k", cache_k[i]),
                        ("cache_v", cache_v[i])):
            _need(t, name, torch.bfloat16, 4)
        if q[i].shape != q[0].shape or cache_k[i].shape != cache_k[0].shape or \
                k_new[i].shape != k_new[0].shape or v_new[i].shape != k_new[0].shape or \
                cache_v[i].shape != cache_k[0].shape:
            raise ValueError("all layers must have the same shapes")
    _need(pos0, "pos0", torch.int32, 1)
    _need(n_new, "n_new", torch.int32, 1)
    _need(table, "table", torch.float32)
    if status is not None:
        _need(status, "status", torch.int32)
    B, S, Hq, D = q[0].shape
    T, Hkv = cache_k[0].shape[1], cache_k[0].shape[2]
    if tuple(k_new[0].shape) != (B, S, Hkv, D) or cache_k[0].shape[0] != B:
        raise ValueError("shapes")
    if table.numel() < T * (D // 2) * 2:
        raise ValueError("rotary table has fewer than T rows")
    _raise(load().ark_attn_append_rope_layers(L, _ptr_array(q), _ptr_array(k_new), _ptr_array(v_new),
                                              _ptr_array(cache_k), _ptr_array(cache_v), _ptr(pos0),
                                              _ptr(n_new), B, S, T, Hq, Hkv, D, _ptr(table), _ptr(status),
                                              _stream(stream)),
           "ark_attn_append_rope_layers")


def ark_attn_decode_layers_workspace_size(L: int, B: int, Hq: int, D: int, T: int, max_splits: int) -> int:
    return int(load().ark_attn_decode_layers_workspace_size(L, B, Hq, D, T, max_splits))


def ark_attn_decode_layers(q: Sequence[torch.Tensor], cache_k, cache_v, kv_len, o, lse, scale: float,
                           mode: int = ARK_LENGTH_AWARE, max_splits: int = 8,
                           workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                           stream=None) -> None:
    """ark_attn_decode over L independent layers in one launch."""
    L = len(q)
    if not (len(cache_k) == len(cache_v) == len(o) == len(lse) == L) or L == 0:
        raise ValueError("per-layer lists must have the same non-zero length")
    for i in range(L):
        _need(q[i], "q", torch.bfloat16, 4)
        _need(cache_k[i], "cache_k", torch.bfloat16, 4)
        _need(cache_v[i], "cache_v", torch.bfloat16, 4)
        _need(o[i], "o", torch.bfloat16, 4)
        _need(lse[i], "lse", torch.float32)
        if q[i].shape != q[0].shape or cache_k[i].shape != cache_k[0].shape or \
                cache_v[i].shape != cache_k[0].shape or o[i].shape != q[0].shape or \
                lse[i].numel() != q[0].shape[0] * q[0].shape[2]:
            raise ValueError("all layers must have the same shapes")
    _need(kv_len, "kv_len", torch.int32, 1)
    B, S, Hq, D = q[0].shape
    if S != 1:
        raise ValueError("decode takes one query row per request")
    T, Hkv = cache_k[0].shape[1], cache_k[0].shape[2]
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", workspace.dtype)
        ws_bytes = workspace.numel() * workspace.element_size()
    if status is not None:
        _need(status, "status", torch.int32)
    _raise(load().ark_attn_decode_layers(L, _ptr_array(q), _ptr_array(cache_k), _ptr_array(cache_v), _ptr(kv_len),
                                         B, T, Hq, Hkv, D, float(scale), int(mode), int(max_splits),
                                         _ptr(workspace), ws_bytes, _ptr_array(o), _ptr_array(lse), _ptr(status),
                                         _stream(stream)),
           "ark_attn_decode_layers")


# ------------------------------------------------ decode, no allocation ----

def ark_attn_decode_noalloc(q, cache_k, cache_v, kv_len, o, lse, scale: float, mode: int = ARK_LENGTH_AWARE,
                            max_splits: int = 8, status: Optional[torch.Tensor] = None, stream=None) -> None:
    """ark_attn_decode without a workspace: the library's own fixed scratch is
    used (see include/arkattn.h for its limits and the one-stream rule)."""
    _need(q, "q", torch.bfloat16, 4)
    _need(cache_k, "cache_k", torch.bfloat16, 4)
    _need(cache_v, "cache_v", torch.bfloat16, 4)
    _need(kv_len, "kv_len", torch.int32, 1)
    _need(o, "o", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32)
    B, S, Hq, D = q.shape
    if S != 1:
        raise ValueError("decode takes one query row per request")
    T, Hkv = cache_k.shape[1], cache_k.shape[2]
    if tuple(o.shape) != tuple(q.shape) or lse.numel() != B * Hq:
        raise ValueError("o/lse shape")
    if status is not None:
        _need(status, "status", torch.int32)
    _raise(load().ark_attn_decode_noalloc(_ptr(q), _ptr(cache_k), _ptr(cache_v), _ptr(kv_len), B, T, Hq, Hkv, D,
                                          float(scale), int(mode), int(max_splits), _ptr(o), _ptr(lse), _ptr(status),
                                          _stream(stream)),
           "ark_attn_decode_noalloc")


# --------------------------------------------------------- fp8 KV cache ----
# Caches of e4m3 codes (torch.uint8, head-major [B,Hkv,T,D], unlike the bf16
# cache) with fp32 scales per KV head (torch.float32 [Hkv] per layer); see the
# header for the format.

def _fp8_cache_checks(cache_k, cache_v, k_scale, v_scale, Hkv_expected=None):
    _need(cache_k, "cache_k", torch.uint8, 4)
    _need(cache_v, "cache_v", torch.uint8, 4)
    _need(k_scale, "k_scale", torch.float32, 1)
    _need(v_scale, "v_scale", torch.float32, 1)
    if cache_v.shape != cache_k.shape:
        raise ValueError("cache_k and cache_v must have the same shape")
    Hkv = cache_k.shape[1]
    if k_scale.numel() != Hkv or v_scale.numel() != Hkv:
        raise ValueError("one K scale and one V scale per KV head")


def ark_attn_append_rope_fp8_layers(q: Sequence[torch.Tensor], k_new, v_new, cache_k, cache_v, k_scale, v_scale,
                                    pos0, n_new, table, status: Optional[torch.Tensor] = None, stream=None) -> None:
    """ark_attn_append_rope into fp8 caches, L layers in one launch."""
    L = len(q)
    if not (len(k_new) == len(v_new) == len(cache_k) == len(cache_v) == len(k_scale) == len(v_scale) == L) \
            or L == 0:
        raise ValueError("per-layer lists must have the same non-zero length")
    for i in range(L):
        for name, t in (("q", q[i]), ("k_new", k_new[i]), ("v_new", v_new[i])):
            _need(t, name, torch.bfloat16, 4)
        _fp8_cache_checks(cache_k[i], cache_v[i], k_scale[i], v_scale[i])
        if q[i].shape != q[0].shape or cache_k[i].shape != cache_k[0].shape or \
                k_new[i].shape != k_new[0].shape or v_new[i].shape != k_new[0].shape:
            raise ValueError("all layers must have the same shapes")
    _need(pos0, "pos0", torch.int32, 1)
    _need(n_new, "n_new", torch.int32, 1)
    _need(table, "table", torch.float32)
    if status is not None:
        _need(status, "status", torch.int32)
    B, S, Hq, D = q[0].shape
    Hkv, T = cache_k[0].shape[1], cache_k[0].shape[2]
    if tuple(k_new[0].shape) != (B, S, Hkv, D) or cache_k[0].shape[0] != B or cache_k[0].shape[3] != D:
        raise ValueError("shapes")
    if table.numel() < T * (D // 2) * 2:
        raise ValueError("rotary table has fewer than T rows")
    _raise(load().ark_attn_append_rope_fp8_layers(L, _ptr_array(q), _ptr_array(k_new), _ptr_array(v_new),
                                                  _ptr_array(cache_k), _ptr_array(cache_v), _ptr_array(k_scale),
                                                  _ptr_array(v_scale), _ptr(pos0), _ptr(n_new), B, S, T, Hq, Hkv,
                                                  D, _ptr(table), _ptr(status), _stream(stream)),
           "ark_attn_append_rope_fp8_layers")


def ark_attn_append_rope_fp8(q, k_new, v_new, cache_k, cache_v, k_scale, v_scale, pos0, n_new, table,
                             status: Optional[torch.Tensor] = None, stream=None) -> None:
    """RoPE + delta write into one layer's fp8 cache."""
    for name, t in (("q", q), ("k_new", k_new), ("v_new", v_new)):
        _need(t, name, torch.bfloat16, 4)
    _fp8_cache_checks(cache_k, cache_v, k_scale, v_scale)
    _need(pos0, "pos0", torch.int32, 1)
    _need(n_new, "n_new", torch.int32, 1)
    _need(table, "table", torch.float32)
    if status is not None:
        _need(status, "status", torch.int32)
    B, S, Hq, D = q.shape
    Hkv, T = cache_k.shape[1], cache_k.shape[2]
    if tuple(k_new.shape) != (B, S, Hkv, D) or tuple(v_new.shape) != (B, S, Hkv, D) or cache_k.shape[0] != B:
        raise ValueError("shapes")
    if table.numel() < T * (D // 2) * 2:
        raise ValueError("rotary table has fewer than T rows")
    _raise(load().ark_attn_append_rope_fp8(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(cache_k), _ptr(cache_v),
                                           _ptr(k_scale), _ptr(v_scale), _ptr(pos0), _ptr(n_new), B, S, T, Hq,
                                           Hkv, D, _ptr(table), _ptr(status), _stream(stream)),
           "ark_attn_append_rope_fp8")


def ark_attn_decode_fp8(q, cache_k, cache_v, k_scale, v_scale, kv_len, o, lse, scale: float,
                        mode: int = ARK_LENGTH_AWARE, max_splits: int = 8, workspace: Optional[torch.Tensor] = None,
                        status: Optional[torch.Tensor] = None, stream=None) -> None:
    """ark_attn_decode over one layer's fp8 cache."""
    _need(q, "q", torch.bfloat16, 4)
    _fp8_cache_checks(cache_k, cache_v, k_scale, v_scale)
    _need(kv_len, "kv_len", torch.int32, 1)
    _need(o, "o", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32)
    B, S, Hq, D = q.shape
    if S != 1:
        raise ValueError("decode takes one query row per request")
    Hkv, T = cache_k.shape[1], cache_k.shape[2]
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", workspace.dtype)
        ws_bytes = workspace.numel() * workspace.element_size()
    if status is not None:
        _need(status, "status", torch.int32)
    _raise(load().ark_attn_decode_fp8(_ptr(q), _ptr(cache_k), _ptr(cache_v), _ptr(k_scale), _ptr(v_scale),
                                      _ptr(kv_len), B, T, Hq, Hkv, D, float(scale), int(mode), int(max_splits),
                                      _ptr(workspace), ws_bytes, _ptr(o), _ptr(lse), _ptr(status),
                                      _stream(stream)),
           "ark_attn_decode_fp8")


def ark_attn_decode_fp8_layers(q: Sequence[torch.Tensor], cache_k, cache_v, k_scale, v_scale, kv_len, o, lse,
                               scale: float, mode: int = ARK_LENGTH_AWARE, max_splits: int = 8,
                               workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                               stream=None) -> None:
    """ark_attn_decode_fp8 over L independent layers in one launch."""
    L = len(q)
    if not (len(cache_k) == len(cache_v) == len(k_scale) == len(v_scale) == len(o) == len(lse) == L) or L == 0:
        raise ValueError("per-layer lists must have the same non-zero length")
    for i in range(L):
        _need(q[i], "q", torch.bfloat16, 4)
        _fp8_cache_checks(cache_k[i], cache_v[i], k_scale[i], v_scale[i])
        _need(o[i], "o", torch.bfloat16, 4)
        _need(lse[i], "lse", torch.float32)
        if q[i].shape != q[0].shape or cache_k[i].shape != cache_k[0].shape or o[i].shape != q[0].shape or \
                lse[i].numel() != q[0].shape[0] * q[0].shape[2]:
            raise ValueError("all layers must have the same shapes")
    _need(kv_len, "kv_len", torch.int32, 1)
    B, S, Hq, D = q[0].shape
    if S != 1:
        raise ValueError("decode takes one query row per request")
    Hkv, T = cache_k[0].shape[1], cache_k[0].shape[2]
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", workspace.dtype)
        ws_bytes = workspace.numel() * workspace.element_size()
    if status is not None:
        _need(status, "status", torch.int32)
    _raise(load().ark_attn_decode_fp8_layers(L, _ptr_array(q), _ptr_array(cache_k), _ptr_array(cache_v),
                                             _ptr_array(k_scale), _ptr_array(v_scale), _ptr(kv_len), B, T, Hq, Hkv,
                                             D, float(scale), int(mode), int(max_splits), _ptr(workspace), ws_bytes,
                                             _ptr_array(o), _ptr_array(lse), _ptr(status), _stream(stream)),
           "ark_attn_decode_fp8_layers")


def ark_attn_prefill_layers(q: Sequence[torch.Tensor], cache_k, cache_v, pos0, n_new, o, lse, scale: float,
                            status: Optional[torch.Tensor] = None, stream=None) -> None:
    """ark_attn_prefill over L independent layers (up to 36 layers per launch)."""
    L = len(q)
    if not (len(cache_k) == len(cache_v) == len(o) == len(lse) == L) or L == 0:
        raise ValueError("per-layer lists must have the same non-zero length")
    for i in range(L):
        _need(q[i], "q", torch.bfloat16, 4)
        _need(cache_k[i], "cache_k", torch.bfloat16, 4)
        _need(cache_v[i], "cache_v", torch.bfloat16, 4)
        _need(o[i], "o", torch.bfloat16, 4)
        _need(lse[i], "lse", torch.float32, 3)
        if q[i].shape != q[0].shape or cache_k[i].shape != cache_k[0].shape or cache_v[i].shape != cache_k[0].shape \
                or o[i].shape != q[0].shape or lse[i].shape != lse[0].shape:
            raise ValueError("all layers must have the same shapes")
    _need(pos0, "pos0", torch.int32, 1)
    _need(n_new, "n_new", torch.int32, 1)
    if status is not None:
        _need(status, "status", torch.int32)
    B, S, Hq, D = q[0].shape
    T, Hkv = cache_k[0].shape[1], cache_k[0].shape[2]
    if tuple(lse[0].shape) != (B, Hq, S):
        raise ValueError("lse must be [B, Hq, S]")
    _raise(load().ark_attn_prefill_layers(L, _ptr_array(q), _ptr_array(cache_k), _ptr_array(cache_v), _ptr(pos0),
                                          _ptr(n_new), B, S, T, Hq, Hkv, D, float(scale), _ptr_array(o),
                                          _ptr_array(lse), _ptr(status), _stream(stream)),
           "ark_attn_prefill_layers")


# -------------------------------------------- prefill with RoPE on load ----
# The prefill rotates q itself as it loads each tile (the same bf16 values the
# append writes), so the append only has to write the K/V rows.

def ark_attn_append_rope_kv_layers(k_new: Sequence[torch.Tensor], v_new, cache_k, cache_v, pos0, n_new, table,
                                   Hq: int = 16, status: Optional[torch.Tensor] = None, stream=None) -> None:
    """ark_attn_append_rope without the query rows: rotated keys and the
    values written into the cache at cache_position, L layers in one launch."""
    L = len(k_new)
    if not (len(v_new) == len(cache_k) == len(cache_v) == L) or L == 0:
        raise ValueError("per-layer lists must have the same non-zero length")
    for i in range(L):
        for name, t in (("k_new", k_new[i]), ("v_new", v_new[i]), ("cache_k", cache_k[i]), ("cache_v", cache_v[i])):
            _need(t, name, torch.bfloat16, 4)
        if k_new[i].shape != k_new[0].shape or v_new[i].shape != k_new[0].shape or \
                cache_k[i].shape != cache_k[0].shape or cache_v[i].shape != cache_k[0].shape:
            raise ValueError("all layers must have the same shapes")
    _need(pos0, "pos0", torch.int32, 1)
    _need(n_new, "n_new", torch.int32, 1)
    _need(table, "table", torch.float32)
    if status is not None:
        _need(status, "status", torch.int32)
    B, S, Hkv, D = k_new[0].shape
    T = cache_k[0].shape[1]
    if table.numel() < T * (D // 2) * 2:
        raise ValueError("rotary table has fewer than T rows")
    _raise(load().ark_attn_append_rope_kv_layers(L, _ptr_array(k_new), _ptr_array(v_new), _ptr_array(cache_k),
                                                 _ptr_array(cache_v), _ptr(pos0), _ptr(n_new), B, S, T, int(Hq),
                                                 Hkv, D, _ptr(table), _ptr(status), _stream(stream)),
           "ark_attn_append_rope_kv_layers")


def ark_attn_prefill_rope_layers(q: Sequence[torch.Tensor], cache_k, cache_v, pos0, n_new, o, lse, scale: float,
                                 table: torch.Tensor, status: Optional[torch.Tensor] = None, stream=None) -> None:
    """ark_attn_prefill with q given unrotated: each tile is rotated as it is
    loaded, with the append's arithmetic (q itself is not modified)."""
    L = len(q)
    if not (len(cache_k) == len(cache_v) == len(o) == len(lse) == L) or L == 0:
        raise ValueError("per-layer lists must have the same non-zero length")
    for i in range(L):
        _need(q[i], "q", torch.bfloat16, 4)
        _need(cache_k[i], "cache_k", torch.bfloat16, 4)
        _need(cache_v[i], "cache_v", torch.bfloat16, 4)
        _need(o[i], "o", torch.bfloat16, 4)
        _need(lse[i], "lse", torch.float32, 3)
        if q[i].shape != q[0].shape or cache_k[i].shape != cache_k[0].shape or cache_v[i].shape != cache_k[0].shape \
                or o[i].shape != q[0].shape or lse[i].shape != lse[0].shape:
            raise ValueError("all layers must have the same shapes")
    _need(pos0, "pos0", torch.int32, 1)
    _need(n_new, "n_new", torch.int32, 1)
    _need(table, "table", torch.float32)
    if status is not None:
        _need(status, "status", torch.int32)
    B, S, Hq, D = q[0].shape
    T, Hkv = cache_k[0].shape[1], cache_k[0].shape[2]
    if tuple(lse[0].shape) != (B, Hq, S):
        raise ValueError("lse must be [B, Hq, S]")
    if table.numel() < T * (D // 2) * 2:
        raise ValueError("rotary table has fewer than T rows")
    _raise(load().ark_attn_prefill_rope_layers(L, _ptr_array(q), _ptr_array(cache_k), _ptr_array(cache_v),
                                               _ptr(pos0), _ptr(n_new), B, S, T, Hq, Hkv, D, float(scale),
                                               _ptr(table), _ptr_array(o), _ptr_array(lse), _ptr(status),
                                               _stream(stream)),
           "ark_attn_prefill_rope_layers")


# ------------------------------------------------------ encoder attention ----

def ark_attn_encoder(q, k, v, length, o, lse, scale: float, status: Optional[torch.Tensor] = None,
                     stream=None) -> None:
    """Bidirectional multi-head attention of the audio encoder: q, k, v, o
    [B,S,H,64] bf16, length int32[B], lse [B,H,S] fp32."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _need(t, name, torch.bfloat16, 4)
    _need(length, "len", torch.int32, 1)
    _need(lse, "lse", torch.float32, 3)
    if status is not None:
        _need(status, "status", torch.int32)
    B, S, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape or o.shape != q.shape or tuple(lse.shape) != (B, H, S):
        raise ValueError("shapes")
    _raise(load().ark_attn_encoder(_ptr(q), _ptr(k), _ptr(v), _ptr(length), B, S, H, D, float(scale), _ptr(o),
                                   _ptr(lse), _ptr(status), _stream(stream)),
           "ark_attn_encoder")


# ------------------------------------------------------ Q/K/V projection ----

def ark_attn_qkv_proj(x, w, bias, out, status: Optional[torch.Tensor] = None, stream=None) -> None:
    """out [M, N] = bf16(x [M, K] @ w [N, K]^T + bias [N]); bias may be None."""
    _need(x, "x", torch.bfloat16, 2)
    _need(w, "w", torch.bfloat16, 2)
    _need(out, "out", torch.bfloat16, 2)
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
    if status is not None:
        _need(status, "status", torch.int32)
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] != K or tuple(out.shape) != (M, N) or (bias is not None and bias.shape[0] != N):
        raise ValueError("shapes")
    _raise(load().ark_attn_qkv_proj(_ptr(x), _ptr(w), _ptr(bias), M, K, N, _ptr(out), _ptr(status),
                                    _stream(stream)), "ark_attn_qkv_proj")


def ark_attn_qkv_rope_append(x, w, bias, pos0, n_new, table, q, cache_k, cache_v,
                             status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Projection of x [B, S, K] by w [(Hq + 2 Hkv) * 128, K] (+ bias), then RoPE
    and the delta write: q [B, S, Hq, 128], caches [B, T, Hkv, 128]."""
    _need(x, "x", torch.bfloat16, 3)
    _need(w, "w", torch.bfloat16, 2)
    for name, t in (("q", q), ("cache_k", cache_k), ("cache_v", cache_v)):
        _need(t, name, torch.bfloat16, 4)
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
    _need(pos0, "pos0", torch.int32, 1)
    _need(n_new, "n_new", torch.int32, 1)
    _need(table, "table", torch.float32)
    if status is not None:
        _need(status, "status", torch.int32)
    B, S, K = x.shape
    Hq, D = q.shape[2], q.shape[3]
    T, Hkv = cache_k.shape[1], cache_k.shape[2]
    if tuple(q.shape[:2]) != (B, S) or w.shape != ((Hq + 2 * Hkv) * D, K) or cache_v.shape != cache_k.shape:
        raise ValueError("shapes")
    _raise(load().ark_attn_qkv_rope_append(_ptr(x), _ptr(w), _ptr(bias), _ptr(pos0), _ptr(n_new), B, S, T, Hq,
                                           Hkv, D, K, _ptr(table), _ptr(q), _ptr(cache_k), _ptr(cache_v),
                                           _ptr(status), _stream(stream)),
           "ark_attn_qkv_rope_append")
