"""ark_attn_decode_noalloc: decode for callers that cannot allocate device
memory when they decode (inside a CUDA-graph capture, under an engine that
reserved all memory up front, or in a plugin whose framework owns the
allocator).  It takes no workspace and uses the library's own fixed scratch.

Called here through the C ABI (ctypes, raw device pointers) and checked
against ark_attn_decode, the entry point with a caller workspace, and against
the fp64 oracle, within the same tolerances as every other decode test, on
two calls in a row (the second call finds the scratch as the first one left
it).  This file is collected
last so that a stop-at-first-failure run has run every other test first; it
also passes alone in a fresh process, where its first call sets the scratch
up on the device.
"""
import ctypes
import math

import pytest
import torch

import oracle
from gqa_attention_static_b200 import ops
from gqa_attention_static_b200 import workloads as W
from tests.helpers import bits, check_lse, check_o, f64

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)


def with_workspace(q, ck, cv, kv, mode, max_splits):
    B, _, Hq, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    ws = ops.decode_workspace(B, Hq, D, ck.shape[1], max_splits, device=q.device)
    ops.ark_attn_decode(q, ck, cv, kv, o, lse, SCALE, mode, max_splits, ws)
    return o, lse


def no_alloc_c_abi(lib, q, ck, cv, kv, mode, max_splits, status):
    """Direct C-ABI call: raw device pointers, sizes, the current stream."""
    B, _, Hq, D = q.shape
    T, Hkv = ck.shape[1], ck.shape[2]
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=q.device)
    rc = lib.ark_attn_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(ck.data_ptr()), ctypes.c_void_p(cv.data_ptr()),
        ctypes.c_void_p(kv.data_ptr()), B, T, Hq, Hkv, D, ctypes.c_float(SCALE), mode, max_splits,
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == ops.ARK_OK, ops.status_string(rc)
    return o, lse


@pytest.mark.parametrize("case", ["ragged512", "long2048", "masked"])
def test_no_alloc_matches_workspace_decode_twice(oracle_lib, case):
    lib = ops.load()
    assert lib.ark_attn_decode_noalloc_scratch_bytes() < 8 << 20
    dev = "cuda"
    if case == "long2048":
        batch = W.cfg_long_decode(layers=1, T=2048)
        mode = ops.ARK_LENGTH_AWARE
    else:
        batch = W.cfg_ragged_decode(layers=1)
        mode = ops.ARK_MASKED_STATIC if case == "masked" else ops.ARK_LENGTH_AWARE
    q = batch.q[0].to(dev)
    ck = batch.cache_k[0].to(dev)
    cv = batch.cache_v[0].to(dev)
    kv = batch.pos0.to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    o_or, lse_or = oracle.decode(bits(batch.q[0]), bits(batch.cache_k[0]), bits(batch.cache_v[0]),
                                 batch.pos0.numpy(), SCALE, static_mode=(mode == ops.ARK_MASKED_STATIC))
    for max_splits in (8, 32):
        o_ref, lse_ref = with_workspace(q, ck, cv, kv, mode, max_splits)
        for _ in range(2):
            o, lse = no_alloc_c_abi(lib, q, ck, cv, kv, mode, max_splits, status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            check_o(f64(o), f64(o_ref), "o (no-alloc vs workspace)")
            check_lse(f64(lse), f64(lse_ref), "lse (no-alloc vs workspace)")
            check_o(f64(o), o_or, "o (no-alloc vs oracle)")
            check_lse(f64(lse), lse_or, "lse (no-alloc vs oracle)")


def test_no_alloc_rejects_batches_beyond_its_limits():
    lib = ops.load()
    dev = "cuda"
    B, T = 4097, 16          # more requests than decode takes
    q = torch.zeros(B, 1, 16, 128, dtype=torch.bfloat16, device=dev)
    ck = torch.zeros(B, T, 2, 128, dtype=torch.bfloat16, device=dev)
    kv = torch.ones(B, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(B, 16, dtype=torch.float32, device=dev)
    rc = lib.ark_attn_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(ck.data_ptr()), ctypes.c_void_p(ck.data_ptr()),
        ctypes.c_void_p(kv.data_ptr()), B, T, 16, 2, 128, ctypes.c_float(SCALE), 0, 8,
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == ops.ARK_ERR_UNSUPPORTED
