"""Host-side plumbing for one decode step over L independent layers.

A decode step is, per layer: RoPE on the new q/k rows and the delta write into
that layer's static cache, then split-KV decode attention over the valid rows
with its log-sum-exp merge.  ``batched=True`` issues both for all layers at
once (``ark_attn_append_rope_layers`` + ``ark_attn_decode_layers``: two
launches per step); ``batched=False`` issues the single-layer calls layer by
layer (``ark_attn_append_rope`` + ``ark_attn_decode``: two launches per
layer), the way a decoder that runs its layers one after another would.  All
launches go to one CUDA stream; the step can be captured in a CUDA graph.
This module only owns buffers and orders calls -- every step of the
computation is a libarkattn kernel.
"""
from __future__ import annotations

import math
from typing import List, Optional

import torch

from . import ops


class DecodeStep:
    """Decode step of ``layers`` layers over a batch of B requests.

    Buffers (per layer lists, all on ``device``):
      q [B,1,Hq,D] (rotated in place), k_new/v_new [B,1,Hkv,D],
      cache_k/cache_v [B,T,Hkv,D], o [B,1,Hq,D], lse [B,Hq];
    shared: pos0, n_new, kv_len int32[B], rotary table, workspace, status
    (table, workspace, status and the o/lse lists are allocated here unless
    passed in).
    With k_scale/v_scale (per layer fp32 [Hkv]) the caches are fp8 (uint8 e4m3
    codes, head-major [B,Hkv,T,D]) and the step uses the fp8 entry points.
    """

    def __init__(self, q: List[torch.Tensor], k_new: List[torch.Tensor], v_new: List[torch.Tensor],
                 cache_k: List[torch.Tensor], cache_v: List[torch.Tensor], pos0: torch.Tensor,
                 n_new: torch.Tensor, kv_len: torch.Tensor, max_splits: int = 8,
                 mode: int = ops.ARK_LENGTH_AWARE, rope_theta: float = 1e6,
                 scale: Optional[float] = None, batched: bool = True,
                 k_scale: Optional[List[torch.Tensor]] = None, v_scale: Optional[List[torch.Tensor]] = None,
                 table: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 status: Optional[torch.Tensor] = None, o: Optional[List[torch.Tensor]] = None,
                 lse: Optional[List[torch.Tensor]] = None):
        self.q, self.k_new, self.v_new = q, k_new, v_new
        self.fp8 = cache_k[0].dtype == torch.uint8
        if self.fp8 and (k_scale is None or v_scale is None):
            raise ValueError("an fp8 cache needs k_scale and v_scale")
        self.k_scale, self.v_scale = k_scale, v_scale
        self.cache_k, self.cache_v = cache_k, cache_v
        self.pos0, self.n_new, self.kv_len = pos0, n_new, kv_len
        self.layers = len(q)
        self.B, _, self.Hq, self.D = q[0].shape
        # the fp8 cache is head-major [B,Hkv,T,D], the bf16 cache [B,T,Hkv,D]
        self.Hkv, self.T = (cache_k[0].shape[1], cache_k[0].shape[2]) if self.fp8 else \
            (cache_k[0].shape[2], cache_k[0].shape[1])
        dev = q[0].device
        self.max_splits = max_splits
        self.mode = mode
        self.batched = batched
        self.scale = scale if scale is not None else 1.0 / math.sqrt(self.D)
        # table, workspace, status and outputs may be shared between steps that run one after
        # another on one stream (a decode loop over many positions)
        self.table = table if table is not None else ops.rope_table(self.T, self.D, rope_theta, device=dev)
        self.workspace = workspace if workspace is not None else ops.decode_workspace(
            self.B, self.Hq, self.D, self.T, max_splits, device=dev, layers=self.layers if batched else 1)
        self.status = status if status is not None else torch.zeros(1, dtype=torch.int32, device=dev)
        self.o = o if o is not None else [torch.empty_like(x) for x in q]
        self.lse = lse if lse is not None else [torch.empty(self.B, self.Hq, dtype=torch.float32, device=dev)
                                                for _ in q]

    @property
    def min_tiles(self) -> int:
        """Fewest 16-row tiles one warp takes (the library's split bound)."""
        tiles = -(-self.T // 16)
        return max(1, -(-tiles // self.max_splits))

    def launches_per_step(self) -> int:
        """Kernels per step: append, decode and the merge of cut pieces."""
        return 3 if self.batched else 3 * self.layers

    def append(self, stream=None) -> None:
        if self.fp8:
            if self.batched:
                ops.ark_attn_append_rope_fp8_layers(self.q, self.k_new, self.v_new, self.cache_k, self.cache_v,
                                                    self.k_scale, self.v_scale, self.pos0, self.n_new, self.table,
                                                    self.status, stream)
            else:
                for l in range(self.layers):
                    ops.ark_attn_append_rope_fp8(self.q[l], self.k_new[l], self.v_new[l], self.cache_k[l],
                                                 self.cache_v[l], self.k_scale[l], self.v_scale[l], self.pos0,
                                                 self.n_new, self.table, self.status, stream)
            return
        if self.batched:
            ops.ark_attn_append_rope_layers(self.q, self.k_new, self.v_new, self.cache_k, self.cache_v,
                                            self.pos0, self.n_new, self.table, self.status, stream)
        else:
            for l in range(self.layers):
                ops.ark_attn_append_rope(self.q[l], self.k_new[l], self.v_new[l], self.cache_k[l],
                                         self.cache_v[l], self.pos0, self.n_new, self.table, self.status,
                                         stream)

    def attention(self, stream=None) -> None:
        if self.fp8:
            if self.batched:
                ops.ark_attn_decode_fp8_layers(self.q, self.cache_k, self.cache_v, self.k_scale, self.v_scale,
                                               self.kv_len, self.o, self.lse, self.scale, self.mode, self.max_splits,
                                               self.workspace, self.status, stream)
            else:
                for l in range(self.layers):
                    ops.ark_attn_decode_fp8(self.q[l], self.cache_k[l], self.cache_v[l], self.k_scale[l],
                                            self.v_scale[l], self.kv_len, self.o[l], self.lse[l], self.scale,
                                            self.mode, self.max_splits, self.workspace, self.status, stream)
            return
        if self.batched:
            ops.ark_attn_decode_layers(self.q, self.cache_k, self.cache_v, self.kv_len, self.o, self.lse,
                                       self.scale, self.mode, self.max_splits, self.workspace, self.status,
                                       stream)
        else:
            for l in range(self.layers):
                ops.ark_attn_decode(self.q[l], self.cache_k[l], self.cache_v[l], self.kv_len, self.o[l],
                                    self.lse[l], self.scale, self.mode, self.max_splits, self.workspace,
                                    self.status, stream)

    def run(self, stream=None) -> None:
        self.append(stream)
        self.attention(stream)

    def attention_only(self, stream=None) -> None:
        """The decode attention of every layer without the append (for timing
        the dominant kernel alone)."""
        self.attention(stream)


class PrefillStep:
    """Prefill of one prompt batch over L independent layers: RoPE + delta
    write of the prompt rows for all layers (one launch), then the causal
    tcgen05 prefill of all layers (one launch per 36 layers; one launch per
    layer with batched=False).

    Buffers (per layer lists): q [B,S,Hq,D] (rotated in place), k_new/v_new
    [B,S,Hkv,D], cache_k/cache_v [B,T,Hkv,D]; outputs o [B,S,Hq,D] bf16 and
    lse [B,Hq,S] fp32 (rows t >= n_new[b] are not written).
    """

    def __init__(self, q, k_new, v_new, cache_k, cache_v, pos0, n_new, rope_theta: float = 1e6,
                 scale: Optional[float] = None, batched: bool = True, fused_rope: bool = False):
        self.batched = batched
        # fused_rope: the append writes only the K/V rows and the prefill rotates
        # q as it loads it (q is then left unrotated in memory)
        self.fused_rope = fused_rope
        self.q, self.k_new, self.v_new = q, k_new, v_new
        self.cache_k, self.cache_v = cache_k, cache_v
        self.pos0, self.n_new = pos0, n_new
        self.layers = len(q)
        self.B, self.S, self.Hq, self.D = q[0].shape
        self.T = cache_k[0].shape[1]
        dev = q[0].device
        self.scale = scale if scale is not None else 1.0 / math.sqrt(self.D)
        self.table = ops.rope_table(self.T, self.D, rope_theta, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.o = [torch.empty_like(x) for x in q]
        self.lse = [torch.empty(self.B, self.Hq, self.S, dtype=torch.float32, device=dev) for _ in q]

    # layers the library's prefill kernel takes per launch (kernel-parameter space)
    LAYERS_PER_LAUNCH = 36

    def launches_per_step(self) -> int:
        """The append (one launch) and the prefill (one launch per 36 layers,
        or one per layer with batched=False; the RoPE-on-load form is always
        layer-batched)."""
        if self.batched or self.fused_rope:
            return 1 + -(-self.layers // self.LAYERS_PER_LAUNCH)
        return 1 + self.layers

    def append(self, stream=None) -> None:
        if self.fused_rope:
            ops.ark_attn_append_rope_kv_layers(self.k_new, self.v_new, self.cache_k, self.cache_v, self.pos0,
                                               self.n_new, self.table, self.Hq, self.status, stream)
            return
        ops.ark_attn_append_rope_layers(self.q, self.k_new, self.v_new, self.cache_k, self.cache_v, self.pos0,
                                        self.n_new, self.table, self.status, stream)

    def attention(self, stream=None) -> None:
        if self.fused_rope:
            ops.ark_attn_prefill_rope_layers(self.q, self.cache_k, self.cache_v, self.pos0, self.n_new, self.o,
                                             self.lse, self.scale, self.table, self.status, stream)
            return
        if self.batched:
            ops.ark_attn_prefill_layers(self.q, self.cache_k, self.cache_v, self.pos0, self.n_new, self.o, self.lse,
                                        self.scale, self.status, stream)
        else:
            for l in range(self.layers):
                ops.ark_attn_prefill(self.q[l], self.cache_k[l], self.cache_v[l], self.pos0, self.n_new, self.o[l],
                                     self.lse[l], self.scale, self.status, stream)

    def run(self, stream=None) -> None:
        self.append(stream)
        self.attention(stream)
