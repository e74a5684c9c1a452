"""Seeded synthetic inputs shaped like the ARK-ASR-3B decoder's attention
workloads.

This module holds no attention or RoPE arithmetic: it only draws random
numbers, picks lengths and fills buffers.  The same tensors feed both the CUDA
library and the fp64 oracle in the tests, and the benchmark.

Shapes follow the "ARK-ASR-3B -- INT8 ONNX" model card, section Shapes: 36
decoder layers, 16 query heads, 2 KV heads, head dim 128, static cache
[B, max_total_len, 2, 128] per layer.  Values are bf16 draws of N(0, 1)
(bf16 is the serving dtype: SGLang-Omni cookbook "ARK-ASR-3B", section dtype).
The pages measure on real audio benchmarks that are not available here; these
synthetic tensors stand in for them, with prompt lengths taken from the audio
token formula below.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import torch

N_LAYERS = 36
HQ = 16
HKV = 2
HEAD_DIM = 128
ROPE_THETA = 1e6


def audio_slots(samples: int) -> int:
    """Number of <|audio|> prompt slots for a clip of ``samples`` 16 kHz samples
    ("ARK-ASR-3B -- INT8 ONNX", section Inference, step 4)."""
    return max(((samples // 160) + 1) // 2 // 4, 1)


def audio_slots_from_mel(mel_frames: int, merge_factor: int = 4) -> int:
    """The same count stated from the mel-frame side (SGLang-Omni cookbook
    "ARK-ASR-3B", section Audio Handling)."""
    return (mel_frames + 1) // 2 // merge_factor


def _gen(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn_bf16(shape, gen: torch.Generator, device: str = "cpu") -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def fill_garbage_(x: torch.Tensor, start: torch.Tensor, gen: torch.Generator, kind: str) -> None:
    """Overwrite rows j >= start[b] of a [B, T, ...] cache with garbage.

    kind: "big"  -> uniform in [-1e4, 1e4] (finite),
          "nan"  -> a mix of NaN, +inf, -inf and +-1e4 values,
          "none" -> leave as is.
    """
    if kind == "none":
        return
    B, T = x.shape[0], x.shape[1]
    dev = x.device
    j = torch.arange(T, device=dev).view(1, T)
    mask = (j >= start.to(dev).view(B, 1).long())
    mask = mask.view(B, T, *([1] * (x.dim() - 2))).expand_as(x)
    big = (torch.rand(x.shape, generator=gen, device=dev) * 2.0 - 1.0) * 1e4
    if kind == "nan":
        sel = torch.randint(0, 4, x.shape, generator=gen, device=dev)
        vals = torch.where(sel == 0, torch.full_like(big, float("nan")),
                           torch.where(sel == 1, torch.full_like(big, float("inf")),
                                       torch.where(sel == 2, torch.full_like(big, float("-inf")), big)))
    elif kind == "big":
        vals = big
    else:
        raise ValueError(kind)
    x[mask] = vals.to(x.dtype)[mask]


def add_row_outliers_(x: torch.Tensor, gen: torch.Generator, frac: float = 0.01,
                      factor: float = 8.0, per: str = "row") -> None:
    """Scale a seeded random ``frac`` of rows (one row = one position of one KV
    head, the last dim) by ``factor``.  ``per="element"`` scales single
    elements instead (the other reading of "1% outliers")."""
    if per == "row":
        shape = x.shape[:-1]
        m = torch.rand(shape, generator=gen, device=x.device) < frac
        x[m] = (x[m].float() * factor).to(x.dtype)
    elif per == "element":
        m = torch.rand(x.shape, generator=gen, device=x.device) < frac
        x[m] = (x[m].float() * factor).to(x.dtype)
    else:
        raise ValueError(per)


@dataclass
class Batch:
    """One batch of per-layer tensors (lists have one entry per layer)."""
    q: List[torch.Tensor]          # [B, S, 16, 128] bf16, new (unrotated) queries
    k_new: List[torch.Tensor]      # [B, S, 2, 128] bf16
    v_new: List[torch.Tensor]      # [B, S, 2, 128] bf16
    cache_k: List[torch.Tensor]    # [B, T, 2, 128] bf16
    cache_v: List[torch.Tensor]    # [B, T, 2, 128] bf16
    pos0: torch.Tensor             # [B] int32, cache_position (valid rows before the call)
    n_new: torch.Tensor            # [B] int32, new rows per request in this call
    T: int
    S: int
    meta: dict = field(default_factory=dict)

    @property
    def B(self) -> int:
        return int(self.pos0.shape[0])

    @property
    def layers(self) -> int:
        return len(self.q)

    @property
    def kv_len(self) -> torch.Tensor:
        """Rows the attention reads after this call's rows are appended."""
        return (self.pos0 + self.n_new).to(torch.int32)


def make_batch(seed: int, B: int, S: int, T: int, pos0, n_new, layers: int = 1,
               garbage: str = "big", outliers: Optional[str] = None,
               device: str = "cpu", hq: int = HQ, hkv: int = HKV, d: int = HEAD_DIM) -> Batch:
    """Seeded batch: caches hold N(0,1) rows below pos0[b] and garbage at and
    past pos0[b]; new q/k/v rows are N(0,1).  ``outliers`` in
    {None, "row", "element"} adds 1% x8 outliers to K/V (cache and new rows)."""
    gen = _gen(seed, device)
    pos0 = torch.as_tensor(pos0, dtype=torch.int32).reshape(B).to(device)
    n_new = torch.as_tensor(n_new, dtype=torch.int32).reshape(B).to(device)
    qs, kn, vn, ck, cv = [], [], [], [], []
    for _ in range(layers):
        q = randn_bf16((B, S, hq, d), gen, device)
        k = randn_bf16((B, S, hkv, d), gen, device)
        v = randn_bf16((B, S, hkv, d), gen, device)
        cache_k = randn_bf16((B, T, hkv, d), gen, device)
        cache_v = randn_bf16((B, T, hkv, d), gen, device)
        if outliers is not None:
            for x in (k, v, cache_k, cache_v):
                add_row_outliers_(x, gen, per=outliers)
        fill_garbage_(cache_k, pos0, gen, garbage)
        fill_garbage_(cache_v, pos0, gen, garbage)
        qs.append(q); kn.append(k); vn.append(v); ck.append(cache_k); cv.append(cache_v)
    return Batch(qs, kn, vn, ck, cv, pos0, n_new, T, S)


# ----------------------------------------------------------- the workloads ---

def cfg_single_decode(seed: int = 1, layers: int = N_LAYERS, garbage: str = "big",
                      device: str = "cpu") -> Batch:
    """Single decode step, batch 1: cache [1,512,2,128] with 64 valid rows and
    large garbage past them; the new k/v row goes to position 64."""
    b = make_batch(seed, B=1, S=1, T=512, pos0=[64], n_new=[1], layers=layers,
                   garbage=garbage, device=device)
    b.meta["name"] = "single decode B=1 T=512 pos 64"
    return b


def sweep_prompt_len() -> int:
    """Prompt of the autoregressive sweep: 37 audio slots (3 s clip) + 13 text."""
    return audio_slots(3 * 16000) + 13


def cfg_sweep_prefill(seed: int = 2, layers: int = N_LAYERS, device: str = "cpu") -> Batch:
    """Prefill of the batch-1 sweep: 50 prompt rows from cache_position 0."""
    L = sweep_prompt_len()
    b = make_batch(seed, B=1, S=L, T=512, pos0=[0], n_new=[L], layers=layers,
                   garbage="big", device=device)
    b.meta["name"] = "sweep prefill B=1 L=50"
    return b


def sweep_step_inputs(seed: int, step: int, layers: int = N_LAYERS, device: str = "cpu"):
    """Fresh N(0,1) q/k/v for decode step ``step`` of the sweep (q [1,1,16,128],
    k/v [1,1,2,128] per layer)."""
    gen = _gen(seed * 100003 + step, device)
    qs = [randn_bf16((1, 1, HQ, HEAD_DIM), gen, device) for _ in range(layers)]
    ks = [randn_bf16((1, 1, HKV, HEAD_DIM), gen, device) for _ in range(layers)]
    vs = [randn_bf16((1, 1, HKV, HEAD_DIM), gen, device) for _ in range(layers)]
    return qs, ks, vs


def sweep_all_step_inputs(seed: int, steps: int, layers: int = N_LAYERS, device: str = "cpu"):
    """Fresh N(0,1) q/k/v for every decode step of the sweep at once, as three
    tensors q [steps, layers, 1, 1, 16, 128], k/v [steps, layers, 1, 1, 2, 128]
    whose [step, layer] slices are one step's per-layer inputs (for the
    benchmark, which replays the whole sweep from device memory)."""
    gen = _gen(seed * 100003 + 7, device)
    q = randn_bf16((steps, layers, 1, 1, HQ, HEAD_DIM), gen, device)
    k = randn_bf16((steps, layers, 1, 1, HKV, HEAD_DIM), gen, device)
    v = randn_bf16((steps, layers, 1, 1, HKV, HEAD_DIM), gen, device)
    return q, k, v


def ragged_lengths(seed: int, B: int, lo: int, hi: int) -> torch.Tensor:
    g = _gen(seed + 7919)
    return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int32)


def cfg_ragged_decode(seed: int = 3, layers: int = N_LAYERS, B: int = 32, T: int = 512,
                      outliers: Optional[str] = "row", garbage: str = "big",
                      device: str = "cpu") -> Batch:
    """Ragged decode batch: 32 requests, valid lengths uniform in [40, 511]
    before the append (so 41..512 rows are read), K/V with 1% x8 outliers."""
    pos0 = ragged_lengths(seed, B, 40, T - 1)
    b = make_batch(seed, B=B, S=1, T=T, pos0=pos0, n_new=torch.ones(B, dtype=torch.int32),
                   layers=layers, garbage=garbage, outliers=outliers, device=device)
    b.meta["name"] = f"ragged decode B={B} T={T} pos0 U[40,{T-1}]"
    return b


def cfg_prefill(seed: int = 4, layers: int = N_LAYERS, B: int = 16, T: int = 512,
                max_len: Optional[int] = None, device: str = "cpu") -> Batch:
    """Coalesced causal prefill: 16 requests, prompt lengths uniform in
    [20, 387] (387 = 375 audio slots for 30 s + 12 text rows), from
    cache_position 0, padded to S = 387."""
    if max_len is None:
        max_len = audio_slots(30 * 16000) + 12
    n_new = ragged_lengths(seed, B, 20, max_len)
    b = make_batch(seed, B=B, S=max_len, T=T, pos0=torch.zeros(B, dtype=torch.int32),
                   n_new=n_new, layers=layers, garbage="big", device=device)
    b.meta["name"] = f"coalesced prefill B={B} S={max_len} T={T}"
    return b


def cfg_long_decode(seed: int = 5, layers: int = N_LAYERS, T: int = 2048, B: int = 32,
                    device: str = "cpu") -> Batch:
    """Long-cache decode: T=2048 with valid lengths uniform in [1500, 2047]
    before the append; or T=1024 full (pos0 = 1023 for every request)."""
    if T == 2048:
        pos0 = ragged_lengths(seed, B, 1500, 2047)
    else:
        pos0 = torch.full((B,), T - 1, dtype=torch.int32)
    b = make_batch(seed, B=B, S=1, T=T, pos0=pos0, n_new=torch.ones(B, dtype=torch.int32),
                   layers=layers, garbage="big", device=device)
    b.meta["name"] = f"long decode B={B} T={T}"
    return b


# ---------------------------------------------------------- fp8 caches ----
# Caches of OCP E4M3 codes (uint8) for the 8-bit cache format.  Drawn as codes
# directly (random sign, exponent field and mantissa bits), so nothing here
# quantises anything.

@dataclass
class Fp8Cache:
    cache_k: List[torch.Tensor]      # per layer [B, T, Hkv, D] uint8 codes
    cache_v: List[torch.Tensor]
    k_scale: List[torch.Tensor]      # per layer [Hkv] fp32
    v_scale: List[torch.Tensor]


def e4m3_codes(shape, gen: torch.Generator, exp_lo: int = 3, exp_hi: int = 10) -> torch.Tensor:
    """Finite e4m3 codes with exponent field in [exp_lo, exp_hi] (magnitudes
    2^(exp_lo-7) .. 1.875 * 2^(exp_hi-7)), random sign and mantissa."""
    sign = torch.randint(0, 2, shape, generator=gen, dtype=torch.int32) << 7
    expo = torch.randint(exp_lo, exp_hi + 1, shape, generator=gen, dtype=torch.int32) << 3
    mant = torch.randint(0, 8, shape, generator=gen, dtype=torch.int32)
    return (sign | expo | mant).to(torch.uint8)


def to_btkd(x):
    """A head-major [B,Hkv,T,D] fp8 cache as [B,T,Hkv,D] (a permuted view;
    works for torch tensors and numpy arrays)."""
    return x.permute(0, 2, 1, 3) if hasattr(x, "permute") else x.transpose(0, 2, 1, 3)


def to_bhtd(x):
    """The inverse of to_btkd: [B,T,Hkv,D] as head-major [B,Hkv,T,D]."""
    return to_btkd(x)


def make_fp8_cache(seed: int, B: int, T: int, valid, layers: int = 1, garbage: str = "nan",
                   Hkv: int = HKV, D: int = HEAD_DIM) -> Fp8Cache:
    """fp8 caches (head-major [B,Hkv,T,D] uint8, the library's fp8 layout;
    `to_btkd` gives the [B,T,Hkv,D] view) whose rows j < valid[b] hold codes
    of moderate magnitude and whose later rows hold `garbage`: "nan" (NaN
    codes 0x7F/0xFF mixed with the
    largest finite codes), "big" (finite codes of magnitude 256..448) or
    "none" (the same distribution as the valid rows).  Scales: uniform in
    [0.02, 0.2], one per KV head for K and for V."""
    g = _gen(seed)
    valid = torch.as_tensor(valid, dtype=torch.int32).view(B)
    out = Fp8Cache([], [], [], [])
    j = torch.arange(T).view(1, T, 1, 1)
    past = j >= valid.view(B, 1, 1, 1)
    for _ in range(layers):
        for lst in (out.cache_k, out.cache_v):
            x = e4m3_codes((B, T, Hkv, D), g)
            if garbage == "nan":
                bad = torch.where(torch.rand((B, T, Hkv, D), generator=g) < 0.5,
                                  torch.randint(0, 2, (B, T, Hkv, D), generator=g, dtype=torch.int32) * 0x80 + 0x7F,
                                  torch.randint(0, 2, (B, T, Hkv, D), generator=g, dtype=torch.int32) * 0x80 + 0x7E)
                x = torch.where(past, bad.to(torch.uint8), x)
            elif garbage == "big":
                x = torch.where(past, e4m3_codes((B, T, Hkv, D), g, 14, 14), x)
            # the library's fp8 cache is head-major [B,Hkv,T,D]; the draws above run in
            # [B,T,Hkv,D] order so that the values stay those of the same seed
            lst.append(x.permute(0, 2, 1, 3).contiguous())
        out.k_scale.append((0.02 + 0.18 * torch.rand(Hkv, generator=g)).float())
        out.v_scale.append((0.02 + 0.18 * torch.rand(Hkv, generator=g)).float())
    return out


# ------------------------------------------------------- encoder batches ----
# The audio encoder's attention: clips of 3..30 s at 16 kHz, 50 encoder frames
# per second after the stride-2 convolution (1500 frames at the 30-second
# Whisper boundary), encoded 8 at a time (SGLang-Omni cookbook "ARK-ASR-3B",
# audio handling: 30 s truncation, encoder_max_batch_size 8); heads of the
# 1280-wide Whisper-large geometry (20 x 64).

ENC_HEADS = 20
ENC_HEAD_DIM = 64
ENC_LAYERS = 32


def encoder_frames(seconds: float) -> int:
    """Encoder frames of a clip: 100 mel frames per second, halved by the
    stride-2 convolution, at most 1500."""
    return max(1, min(1500, int(seconds * 100) // 2))


@dataclass
class EncoderBatch:
    q: List[torch.Tensor]          # per layer [B, S, H, D] bf16
    k: List[torch.Tensor]
    v: List[torch.Tensor]
    length: torch.Tensor           # int32 [B]

    @property
    def B(self) -> int:
        return self.q[0].shape[0]

    @property
    def S(self) -> int:
        return self.q[0].shape[1]


def make_encoder_batch(seed: int, B: int, S: int, lengths, H: int = ENC_HEADS, D: int = ENC_HEAD_DIM,
                       layers: int = 1, garbage: str = "nan") -> EncoderBatch:
    """bf16 N(0,1) q/k/v per layer; frames past each clip's length hold
    garbage ("nan": NaN/inf, "big": +-1e4, "none": N(0,1))."""
    g = _gen(seed)
    length = torch.as_tensor(lengths, dtype=torch.int32).view(B)
    out = EncoderBatch([], [], [], length)
    for _ in range(layers):
        for lst in (out.q, out.k, out.v):
            x = randn_bf16((B, S, H, D), g)
            if garbage != "none":
                fill_garbage_(x, length, g, garbage)
            lst.append(x.contiguous())
    return out


def cfg_encoder(seed: int = 6, layers: int = ENC_LAYERS, B: int = 8) -> EncoderBatch:
    """8 clips of 3..30 s (150..1500 frames), padded to 1500."""
    g = _gen(seed)
    secs = 3.0 + 27.0 * torch.rand(B, generator=g)
    lengths = [encoder_frames(float(s)) for s in secs]
    return make_encoder_batch(seed + 1, B, 1500, lengths, layers=layers)


# ----------------------------------------------- projection weights (synthetic) ----
# The decoder's Q/K/V projections (hidden 2048 -> 16 q heads, 2 k, 2 v heads of
# 128; "ARK-ASR-3B -- INT8 ONNX" model card).  No trained weights: W ~ N(0, 1/K)
# (the scale of an initialised Linear), bias ~ N(0, 0.1^2), hidden states
# ~ N(0, 1) (the scale after the RMSNorm in front of the projection).

HIDDEN = 2048


def make_qkv_weights(seed: int, K: int = HIDDEN, Hq: int = 16, Hkv: int = 2, D: int = 128, bias: bool = True):
    g = _gen(seed)
    N = (Hq + 2 * Hkv) * D
    w = (torch.randn((N, K), generator=g, dtype=torch.float32) / (K ** 0.5)).to(torch.bfloat16)
    b = (torch.randn((N,), generator=g, dtype=torch.float32) * 0.1).to(torch.bfloat16) if bias else None
    return w, b


def make_hidden(seed: int, B: int, S: int, K: int = HIDDEN) -> torch.Tensor:
    return randn_bf16((B, S, K), _gen(seed))
