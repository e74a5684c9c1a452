"""fp64 CPU oracle for GQA attention over a static, sequence-major KV cache.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library (``gqa_attention_static_b200``) never imports it and
shares no code with it: the arithmetic lives in ``arkattn_oracle.c`` (plain C,
double precision) and this module only moves numpy arrays across ctypes.

bf16 tensors are passed as ``numpy.uint16`` arrays holding the bf16 bit
patterns.  Each wrapper names the passage of the pages its C function follows;
the C file's header gives the full list and the readings taken where the pages
are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "arkattn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (double precision, no fast-math, no
    contraction, OpenMP over independent query rows)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.ora_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.ora_bf16_to_f64.restype = ctypes.c_double
        lib.ora_f64_to_bf16_rne.argtypes = [ctypes.c_double]
        lib.ora_f64_to_bf16_rne.restype = ctypes.c_uint16
        lib.ora_rope_table.argtypes = [I, I, ctypes.c_double, P, P]
        lib.ora_rope_table.restype = None
        lib.ora_rope_rotate.argtypes = [P, P, P, I, P]
        lib.ora_rope_rotate.restype = None
        lib.ora_append_rope.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P, P]
        lib.ora_append_rope.restype = I
        lib.ora_attend_one.argtypes = [P, P, P, ctypes.c_long, I, I, I, ctypes.c_double, P, P]
        lib.ora_attend_one.restype = None
        lib.ora_attend_one_static.argtypes = [P, P, P, ctypes.c_long, I, I, I, ctypes.c_double, P, P]
        lib.ora_attend_one_static.restype = None
        lib.ora_attention.argtypes = [P, P, P, P, P, I, I, I, I, I, I, ctypes.c_double, I, P, P]
        lib.ora_attention.restype = None
        lib.ora_combine.argtypes = [P, P, I, I, P, P]
        lib.ora_combine.restype = None
        lib.ora_num_threads.argtypes = []
        lib.ora_num_threads.restype = I
        lib.ora_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.ora_e4m3_to_f64.restype = ctypes.c_double
        lib.ora_f32_to_e4m3.argtypes = [ctypes.c_float]
        lib.ora_f32_to_e4m3.restype = ctypes.c_uint8
        lib.ora_quantize_e4m3.argtypes = [ctypes.c_double, ctypes.c_float]
        lib.ora_quantize_e4m3.restype = ctypes.c_uint8
        lib.ora_append_rope_fp8.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, P, P]
        lib.ora_append_rope_fp8.restype = I
        lib.ora_attention_fp8.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, ctypes.c_double, I, P, P]
        lib.ora_attention_fp8.restype = None
        lib.ora_attention_bidir.argtypes = [P, P, P, P, I, I, I, I, ctypes.c_double, P, P]
        lib.ora_qkv_proj.argtypes = [P, P, P, I, I, I, P]
        lib.ora_qkv_proj.restype = None
        lib.ora_attention_bidir.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _c(a, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def num_threads() -> int:
    """OpenMP threads the oracle's attention loop uses."""
    return int(_load().ora_num_threads())


# ------------------------------------------------------------------ bf16 ----

def bf16_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns to double."""
    lib = _load()
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    out = np.array([lib.ora_bf16_to_f64(int(b)) for b in flat], dtype=np.float64)
    return out.reshape(np.shape(bits))


def bf16_array_to_f64(bits: np.ndarray) -> np.ndarray:
    """Vectorised exact widening (bf16 is the top half of binary32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    with np.errstate(invalid="ignore"):
        return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(x) -> np.ndarray:
    """Round doubles to bf16 bit patterns, nearest-even (IEEE definition)."""
    lib = _load()
    flat = np.asarray(x, dtype=np.float64).ravel()
    out = np.array([lib.ora_f64_to_bf16_rne(float(v)) for v in flat], dtype=np.uint16)
    return out.reshape(np.shape(x))


# ------------------------------------------------------------------ RoPE ----

def rope_table(T: int, D: int = 128, theta: float = 1e6):
    """fp32 cos/sin tables [T, D/2] of the Qwen2 rotary embedding
    ("ARK-ASR-3B" SGLang-Omni cookbook, introduction: Qwen2 decoder)."""
    lib = _load()
    c = np.zeros((T, D // 2), dtype=np.float32)
    s = np.zeros((T, D // 2), dtype=np.float32)
    lib.ora_rope_table(T, D, float(theta), _ptr(c), _ptr(s))
    return c, s


def rope_rotate(x: np.ndarray, c: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE of one fp64 row with fp64 cos/sin (no rounding)."""
    lib = _load()
    x = _c(x, np.float64)
    c = _c(c, np.float64)
    s = _c(s, np.float64)
    D = x.shape[0]
    out = np.zeros(D, dtype=np.float64)
    lib.ora_rope_rotate(_ptr(x), _ptr(c), _ptr(s), D, _ptr(out))
    return out


def append_rope(q, k_new, v_new, cache_k, cache_v, pos0, n_new, theta: float = 1e6):
    """RoPE on the new q/k rows and the delta write into the static cache
    ("ARK-ASR-3B -- INT8 ONNX", section Shapes: key_delta/value_delta rows are
    copied into the cache at cache_position).

    Works on copies; returns (q_rot, cache_k_new, cache_v_new, skipped).
    Shapes: q [B,S,Hq,D], k_new/v_new [B,S,Hkv,D], caches [B,T,Hkv,D] (uint16).
    """
    lib = _load()
    q = np.array(q, dtype=np.uint16, copy=True, order="C")
    ck = np.array(cache_k, dtype=np.uint16, copy=True, order="C")
    cv = np.array(cache_v, dtype=np.uint16, copy=True, order="C")
    kn = _c(k_new, np.uint16)
    vn = _c(v_new, np.uint16)
    p0 = _c(pos0, np.int32)
    nn = _c(n_new, np.int32)
    B, S, Hq, D = q.shape
    T, Hkv = ck.shape[1], ck.shape[2]
    cos_t, sin_t = rope_table(T, D, theta)
    skipped = lib.ora_append_rope(_ptr(q), _ptr(kn), _ptr(vn), _ptr(ck), _ptr(cv),
                                  _ptr(p0), _ptr(nn), B, S, T, Hq, Hkv, D,
                                  _ptr(cos_t), _ptr(sin_t))
    return q, ck, cv, int(skipped)


# ------------------------------------------------------------- attention ----

def attend_one(qrow, krows, vrows, j0: int, j1: int, scale: float):
    """Softmax attention of one query over rows [j0, j1) of K/V ([n, D] uint16)."""
    lib = _load()
    qrow = _c(qrow, np.uint16)
    krows = _c(krows, np.uint16)
    vrows = _c(vrows, np.uint16)
    D = qrow.shape[-1]
    o = np.zeros(D, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    lib.ora_attend_one(_ptr(qrow), _ptr(krows), _ptr(vrows), D, j0, j1, D, float(scale),
                       _ptr(o), _ptr(lse))
    return o, float(lse[0])


def attend_one_static(qrow, krows, vrows, n_valid: int, scale: float):
    """Static-cache form: all T rows scored, rows >= n_valid masked to -inf."""
    lib = _load()
    qrow = _c(qrow, np.uint16)
    krows = _c(krows, np.uint16)
    vrows = _c(vrows, np.uint16)
    D = qrow.shape[-1]
    T = krows.shape[0]
    o = np.zeros(D, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    lib.ora_attend_one_static(_ptr(qrow), _ptr(krows), _ptr(vrows), D, T, n_valid, D,
                              float(scale), _ptr(o), _ptr(lse))
    return o, float(lse[0])


def attention(q, cache_k, cache_v, first_vis, n_rows, scale: float, static_mode: bool = False):
    """Causal GQA attention over the cache ("ARK-ASR-3B -- INT8 ONNX", section
    Shapes: 16 heads, 2 KV heads, head dim 128, static cache).

    q [B,S,Hq,D] uint16; caches [B,T,Hkv,D] uint16; query row t of request b
    sees keys j < first_vis[b] + t.  Returns o [B,S,Hq,D] float64 (rows t >=
    n_rows[b] are NaN) and lse [B,Hq,S] float64 (same rows NaN).
    """
    lib = _load()
    q = _c(q, np.uint16)
    ck = _c(cache_k, np.uint16)
    cv = _c(cache_v, np.uint16)
    fv = _c(first_vis, np.int32)
    nr = _c(n_rows, np.int32)
    B, S, Hq, D = q.shape
    T, Hkv = ck.shape[1], ck.shape[2]
    o = np.full((B, S, Hq, D), np.nan, dtype=np.float64)
    lse = np.full((B, Hq, S), np.nan, dtype=np.float64)
    lib.ora_attention(_ptr(q), _ptr(ck), _ptr(cv), _ptr(fv), _ptr(nr), B, S, T, Hq, Hkv, D,
                      float(scale), 1 if static_mode else 0, _ptr(o), _ptr(lse))
    return o, lse


def decode(q, cache_k, cache_v, kv_len, scale: float, static_mode: bool = False):
    """Single-token decode: q [B,1,Hq,D] attends to keys j < kv_len[b].
    Returns o [B,1,Hq,D], lse [B,Hq]."""
    B = q.shape[0]
    o, lse = attention(q, cache_k, cache_v, kv_len, np.ones(B, dtype=np.int32), scale,
                       static_mode)
    return o, lse[:, :, 0]


def prefill(q, cache_k, cache_v, pos0, n_new, scale: float):
    """Causal prefill: row t of request b (position pos0[b]+t) sees keys
    j <= pos0[b]+t.  Returns o [B,S,Hq,D], lse [B,Hq,S]."""
    fv = np.asarray(pos0, dtype=np.int32) + 1
    return attention(q, cache_k, cache_v, fv, n_new, scale)


def combine(o_part, lse_part):
    """Log-sum-exp merge of partial results over disjoint key ranges.
    o_part [n, D] (normalised partial outputs), lse_part [n]."""
    lib = _load()
    op = _c(o_part, np.float64)
    lp = _c(lse_part, np.float64)
    n, D = op.shape
    o = np.zeros(D, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    lib.ora_combine(_ptr(op), _ptr(lp), n, D, _ptr(o), _ptr(lse))
    return o, float(lse[0])


# ---------------------------------------------------------- fp8 KV cache ----
# An 8-bit cache format that is not on the pages (they quantise weights only);
# the reading is stated in arkattn_oracle.c: OCP E4M3 codes, one fp32 scale per
# (layer, KV head) for K and for V, code = e4m3(fp32(x / scale)).

def e4m3_to_f64(codes) -> np.ndarray:
    """Exact values of e4m3 codes (uint8); NaN for the NaN codes."""
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.ora_e4m3_to_f64(int(x)) for x in c.reshape(-1)], dtype=np.float64).reshape(c.shape)


def f32_to_e4m3(x) -> np.ndarray:
    """fp32 values -> e4m3 codes (nearest even, saturating to +-448)."""
    lib = _load()
    a = np.asarray(x, dtype=np.float32)
    return np.array([lib.ora_f32_to_e4m3(float(v)) for v in a.reshape(-1)], dtype=np.uint8).reshape(a.shape)


def quantize_e4m3(x, scale: float) -> np.ndarray:
    """e4m3(fp32(x / scale)) for fp64 values x."""
    lib = _load()
    a = np.asarray(x, dtype=np.float64)
    return np.array([lib.ora_quantize_e4m3(float(v), float(scale)) for v in a.reshape(-1)],
                    dtype=np.uint8).reshape(a.shape)


def append_rope_fp8(q, k_new, v_new, cache_k, cache_v, k_scale, v_scale, pos0, n_new, theta: float = 1e6):
    """RoPE + delta write into an fp8 cache of one layer: q rotated to bf16 in
    place, rotated keys and values quantised with the per-KV-head scales.
    Works on copies; returns (q_rot, cache_k_new, cache_v_new, skipped)."""
    lib = _load()
    q = np.array(q, dtype=np.uint16, copy=True, order="C")
    ck = np.array(cache_k, dtype=np.uint8, copy=True, order="C")
    cv = np.array(cache_v, dtype=np.uint8, copy=True, order="C")
    kn = _c(k_new, np.uint16)
    vn = _c(v_new, np.uint16)
    ks = _c(k_scale, np.float32)
    vs = _c(v_scale, np.float32)
    p0 = _c(pos0, np.int32)
    nn = _c(n_new, np.int32)
    B, S, Hq, D = q.shape
    T, Hkv = ck.shape[1], ck.shape[2]
    cos_t, sin_t = rope_table(T, D, theta)
    skipped = lib.ora_append_rope_fp8(_ptr(q), _ptr(kn), _ptr(vn), _ptr(ck), _ptr(cv), _ptr(ks), _ptr(vs),
                                      _ptr(p0), _ptr(nn), B, S, T, Hq, Hkv, D, _ptr(cos_t), _ptr(sin_t))
    return q, ck, cv, int(skipped)


def attention_fp8(q, cache_k, cache_v, k_scale, v_scale, first_vis, n_rows, scale: float,
                  static_mode: bool = False):
    """attention() over an fp8 cache (uint8 codes, per-KV-head scales)."""
    lib = _load()
    q = _c(q, np.uint16)
    ck = _c(cache_k, np.uint8)
    cv = _c(cache_v, np.uint8)
    ks = _c(k_scale, np.float32)
    vs = _c(v_scale, np.float32)
    fv = _c(first_vis, np.int32)
    nr = _c(n_rows, np.int32)
    B, S, Hq, D = q.shape
    T, Hkv = ck.shape[1], ck.shape[2]
    o = np.full((B, S, Hq, D), np.nan, dtype=np.float64)
    lse = np.full((B, Hq, S), np.nan, dtype=np.float64)
    lib.ora_attention_fp8(_ptr(q), _ptr(ck), _ptr(cv), _ptr(ks), _ptr(vs), _ptr(fv), _ptr(nr),
                          B, S, T, Hq, Hkv, D, float(scale), 1 if static_mode else 0, _ptr(o), _ptr(lse))
    return o, lse


def decode_fp8(q, cache_k, cache_v, k_scale, v_scale, kv_len, scale: float, static_mode: bool = False):
    """Single-token decode over an fp8 cache.  Returns o [B,1,Hq,D], lse [B,Hq]."""
    B = q.shape[0]
    o, lse = attention_fp8(q, cache_k, cache_v, k_scale, v_scale, kv_len, np.ones(B, dtype=np.int32),
                           scale, static_mode)
    return o, lse[:, :, 0]


# ------------------------------------------------------ encoder attention ----

def attention_bidir(q, k, v, length, scale: float):
    """Bidirectional multi-head attention of the audio encoder: row i < len[b]
    of clip b and head h attends to rows j < len[b] of the same clip and head.
    q, k, v [B,S,H,D] uint16 (bf16 bits).  Returns o [B,S,H,D] float64 and lse
    [B,H,S] float64, NaN for rows i >= len[b]."""
    lib = _load()
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    ln = _c(length, np.int32)
    B, S, H, D = q.shape
    o = np.full((B, S, H, D), np.nan, dtype=np.float64)
    lse = np.full((B, H, S), np.nan, dtype=np.float64)
    lib.ora_attention_bidir(_ptr(q), _ptr(k), _ptr(v), _ptr(ln), B, S, H, D, float(scale), _ptr(o), _ptr(lse))
    return o, lse


# ------------------------------------------------------ Q/K/V projection ----

def qkv_proj(x, w, bias=None):
    """The Q/K/V projections of a decoder layer as one Linear over the
    concatenated weight [Wq; Wk; Wv] ("ARK-ASR-3B -- INT8 ONNX", model card:
    Q/K/V projections of the Qwen2 decoder, hidden 2048): x [M, K], w [N, K],
    bias [N] or None (bf16 bits) -> out [M, N] bf16 bits, each the bf16 rounding
    of the double-precision sum plus bias."""
    lib = _load()
    x = _c(x, np.uint16)
    w = _c(w, np.uint16)
    M, K = x.shape
    N = w.shape[0]
    assert w.shape[1] == K
    b = None if bias is None else _c(bias, np.uint16)
    out = np.zeros((M, N), dtype=np.uint16)
    lib.ora_qkv_proj(_ptr(x), _ptr(w), None if b is None else _ptr(b), M, K, N, _ptr(out))
    return out


def qkv_rope_append(x, w, bias, cache_k, cache_v, pos0, n_new, Hq: int, Hkv: int, D: int = 128,
                    theta: float = 1e6):
    """The projection step in front of the attention, then RoPE and the delta
    write: x [B, S, K] token rows; q, k, v = the three column blocks of
    qkv_proj(x); then append_rope.  Returns (q_rot [B,S,Hq,D], cache_k,
    cache_v, skipped)."""
    x = _c(x, np.uint16)
    B, S, K = x.shape
    out = qkv_proj(x.reshape(B * S, K), w, bias)
    q = out[:, :Hq * D].reshape(B, S, Hq, D)
    k = out[:, Hq * D:(Hq + Hkv) * D].reshape(B, S, Hkv, D)
    v = out[:, (Hq + Hkv) * D:].reshape(B, S, Hkv, D)
    return append_rope(q, k, v, cache_k, cache_v, pos0, n_new, theta)
