"""The fp8 (E4M3) KV cache: append into it bit for bit, and decode over it
within the decode tolerances, against the fp64 oracle.

The 8-bit cache is a format of this library's own (the pages quantise weights
only, "ARK-ASR-3B -- INT8 ONNX" introduction); the oracle's reading of it:
one fp32 scale per (layer, KV head) for K and for V, code =
e4m3(fp32(x / scale)), attention over code * scale.  The shapes are the
decoder's ("ARK-ASR-3B -- INT8 ONNX", section Shapes)."""
import math

import numpy as np
import pytest
import torch

import oracle
from gqa_attention_static_b200 import ops
from gqa_attention_static_b200 import workloads as W
from gqa_attention_static_b200.step import DecodeStep
from tests.helpers import bits, check_lse, check_o, f64

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)


def u8(x: torch.Tensor) -> np.ndarray:
    """An fp8 cache (the library's head-major [B,Hkv,T,D]) as a uint8 array in
    the oracle's [B,T,Hkv,D] order."""
    return W.to_btkd(x.detach().cpu()).contiguous().numpy()


def test_append_fp8_bit_exact(oracle_lib):
    B, S, T, L = 3, 5, 64, 2
    batch = W.make_batch(301, B=B, S=S, T=T, pos0=[0, 17, 62], n_new=[5, 3, 2], layers=L)
    fc = W.make_fp8_cache(302, B, T, batch.pos0, layers=L, garbage="none")
    dev = "cuda"
    q = [x.to(dev).clone() for x in batch.q]
    ck = [x.to(dev).clone() for x in fc.cache_k]
    cv = [x.to(dev).clone() for x in fc.cache_v]
    ks = [x.to(dev) for x in fc.k_scale]
    vs = [x.to(dev) for x in fc.v_scale]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.ark_attn_append_rope_fp8_layers(q, [x.to(dev) for x in batch.k_new], [x.to(dev) for x in batch.v_new],
                                        ck, cv, ks, vs, batch.pos0.to(dev), batch.n_new.to(dev),
                                        ops.rope_table(T), status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for l in range(L):
        q_ref, ck_ref, cv_ref, skipped = oracle.append_rope_fp8(
            bits(batch.q[l]), bits(batch.k_new[l]), bits(batch.v_new[l]), u8(fc.cache_k[l]), u8(fc.cache_v[l]),
            fc.k_scale[l].numpy(), fc.v_scale[l].numpy(), batch.pos0.numpy(), batch.n_new.numpy())
        assert skipped == 0
        assert np.array_equal(bits(q[l]), q_ref)
        assert np.array_equal(u8(ck[l]), ck_ref), f"layer {l}: K codes differ at {np.argwhere(u8(ck[l]) != ck_ref)[:5]}"
        assert np.array_equal(u8(cv[l]), cv_ref), f"layer {l}: V codes differ"


def test_append_fp8_saturates_and_single_layer_entry(oracle_lib):
    """Large inputs against small scales: codes saturate at +-448 exactly as the
    oracle's; the single-layer entry point writes the same bytes."""
    B, S, T = 2, 4, 32
    batch = W.make_batch(303, B=B, S=S, T=T, pos0=[3, 20], n_new=[4, 4])
    fc = W.make_fp8_cache(304, B, T, batch.pos0, garbage="none")
    ks = torch.tensor([0.002, 0.5])
    vs = torch.tensor([0.004, 0.01])
    dev = "cuda"
    q = batch.q[0].to(dev).clone()
    ck = fc.cache_k[0].to(dev).clone()
    cv = fc.cache_v[0].to(dev).clone()
    ops.ark_attn_append_rope_fp8(q, batch.k_new[0].to(dev), batch.v_new[0].to(dev) * 8, ck, cv, ks.to(dev),
                                 vs.to(dev), batch.pos0.to(dev), batch.n_new.to(dev), ops.rope_table(T))
    torch.cuda.synchronize()
    q_ref, ck_ref, cv_ref, _ = oracle.append_rope_fp8(
        bits(batch.q[0]), bits(batch.k_new[0]), bits(batch.v_new[0].to(dev) * 8), u8(fc.cache_k[0]),
        u8(fc.cache_v[0]), ks.numpy(), vs.numpy(), batch.pos0.numpy(), batch.n_new.numpy())
    assert np.array_equal(bits(q), q_ref)
    assert np.array_equal(u8(ck), ck_ref) and np.array_equal(u8(cv), cv_ref)
    assert (np.abs(oracle.e4m3_to_f64(ck_ref[0, 3:7])) == 448).any()    # saturation was exercised


def gpu_decode_fp8(q, fc, kv, mode=ops.ARK_LENGTH_AWARE, max_splits=8, layer=0):
    dev = "cuda"
    B, _, Hq, D = q.shape
    T = fc.cache_k[layer].shape[2]
    o = torch.full((B, 1, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
    ws = ops.decode_workspace(B, Hq, D, T, max_splits, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.ark_attn_decode_fp8(q.to(dev), fc.cache_k[layer].to(dev), fc.cache_v[layer].to(dev),
                            fc.k_scale[layer].to(dev), fc.v_scale[layer].to(dev), kv.to(dev), o, lse, SCALE, mode,
                            max_splits, ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, lse


@pytest.mark.parametrize("mode", [ops.ARK_LENGTH_AWARE, ops.ARK_MASKED_STATIC])
@pytest.mark.parametrize("max_splits", [1, 8, 32])
def test_decode_fp8_ragged(oracle_lib, mode, max_splits):
    B, T = 7, 256
    kv = torch.tensor([1, 16, 17, 100, 200, 255, 256], dtype=torch.int32)
    g = torch.Generator().manual_seed(310 + max_splits)
    q = W.randn_bf16((B, 1, 16, 128), g)
    fc = W.make_fp8_cache(311 + max_splits, B, T, kv,
                          garbage="big" if mode == ops.ARK_MASKED_STATIC else "nan")
    o, lse = gpu_decode_fp8(q, fc, kv, mode, max_splits)
    o_ref, lse_ref = oracle.decode_fp8(bits(q), u8(fc.cache_k[0]), u8(fc.cache_v[0]), fc.k_scale[0].numpy(),
                                       fc.v_scale[0].numpy(), kv.numpy(), SCALE,
                                       static_mode=(mode == ops.ARK_MASKED_STATIC))
    check_o(f64(o), o_ref, "o")
    check_lse(f64(lse), lse_ref, "lse")


def test_decode_fp8_long_cache(oracle_lib):
    B, T = 6, 2048
    kv = torch.tensor([1500, 2047, 2048, 1777, 33, 1024], dtype=torch.int32)
    g = torch.Generator().manual_seed(320)
    q = W.randn_bf16((B, 1, 16, 128), g)
    fc = W.make_fp8_cache(321, B, T, kv)
    o, lse = gpu_decode_fp8(q, fc, kv)
    o_ref, lse_ref = oracle.decode_fp8(bits(q), u8(fc.cache_k[0]), u8(fc.cache_v[0]), fc.k_scale[0].numpy(),
                                       fc.v_scale[0].numpy(), kv.numpy(), SCALE)
    check_o(f64(o), o_ref, "o")
    check_lse(f64(lse), lse_ref, "lse")


def test_decode_fp8_step_ragged_batch(oracle_lib):
    """The bench's ragged batch (32 requests, kv_len 41..512) over 4 layers,
    append + decode through the layer-batched fp8 entry points."""
    L = 4
    batch = W.cfg_ragged_decode(layers=L)
    fc = W.make_fp8_cache(330, batch.B, batch.T, batch.pos0, layers=L)
    dev = "cuda"
    kv = (batch.pos0 + batch.n_new).to(torch.int32)
    step = DecodeStep([x.to(dev).clone() for x in batch.q], [x.to(dev) for x in batch.k_new],
                      [x.to(dev) for x in batch.v_new], [x.to(dev).clone() for x in fc.cache_k],
                      [x.to(dev).clone() for x in fc.cache_v], batch.pos0.to(dev), batch.n_new.to(dev), kv.to(dev),
                      k_scale=[x.to(dev) for x in fc.k_scale], v_scale=[x.to(dev) for x in fc.v_scale])
    step.run()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    for l in range(L):
        q_ref, ck_ref, cv_ref, _ = oracle.append_rope_fp8(
            bits(batch.q[l]), bits(batch.k_new[l]), bits(batch.v_new[l]), u8(fc.cache_k[l]), u8(fc.cache_v[l]),
            fc.k_scale[l].numpy(), fc.v_scale[l].numpy(), batch.pos0.numpy(), batch.n_new.numpy())
        assert np.array_equal(u8(step.cache_k[l]), ck_ref) and np.array_equal(u8(step.cache_v[l]), cv_ref)
        o_ref, lse_ref = oracle.decode_fp8(q_ref, ck_ref, cv_ref, fc.k_scale[l].numpy(), fc.v_scale[l].numpy(),
                                           kv.numpy(), SCALE)
        check_o(f64(step.o[l]), o_ref, f"o layer {l}")
        check_lse(f64(step.lse[l]), lse_ref, f"lse layer {l}")


@pytest.mark.parametrize("mode", [ops.ARK_LENGTH_AWARE, ops.ARK_MASKED_STATIC])
def test_decode_fp8_one_kv_head_and_T_not_a_multiple_of_16(oracle_lib, mode):
    """The head-major fp8 cache with a single KV head (8 query heads) and
    T = 100: the last 16-position tile reaches past T, where the copy reads
    zeros; lengths 1, 57 and T."""
    B, T = 3, 100
    kv = torch.tensor([1, 57, 100], dtype=torch.int32)
    g = torch.Generator().manual_seed(340)
    q = W.randn_bf16((B, 1, 8, 128), g)
    fc = W.make_fp8_cache(341, B, T, kv, Hkv=1, garbage="big" if mode == ops.ARK_MASKED_STATIC else "nan")
    o, lse = gpu_decode_fp8(q, fc, kv, mode)
    o_ref, lse_ref = oracle.decode_fp8(bits(q), u8(fc.cache_k[0]), u8(fc.cache_v[0]), fc.k_scale[0].numpy(),
                                       fc.v_scale[0].numpy(), kv.numpy(), SCALE,
                                       static_mode=(mode == ops.ARK_MASKED_STATIC))
    check_o(f64(o), o_ref, "o")
    check_lse(f64(lse), lse_ref, "lse")


def test_append_fp8_one_kv_head_bit_exact(oracle_lib):
    """The append into a head-major fp8 cache with one KV head, T = 100,
    rows landing in the last (partial) 16-position tile."""
    B, S, T = 2, 3, 100
    batch = W.make_batch(342, B=B, S=S, T=T, pos0=[0, 97], n_new=[3, 3], hq=8, hkv=1)
    fc = W.make_fp8_cache(343, B, T, batch.pos0, garbage="none", Hkv=1)
    dev = "cuda"
    q = batch.q[0].to(dev).clone()
    ck, cv = fc.cache_k[0].to(dev).clone(), fc.cache_v[0].to(dev).clone()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.ark_attn_append_rope_fp8(q, batch.k_new[0].to(dev), batch.v_new[0].to(dev), ck, cv, fc.k_scale[0].to(dev),
                                 fc.v_scale[0].to(dev), batch.pos0.to(dev), batch.n_new.to(dev), ops.rope_table(T),
                                 status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    q_ref, ck_ref, cv_ref, skipped = oracle.append_rope_fp8(
        bits(batch.q[0]), bits(batch.k_new[0]), bits(batch.v_new[0]), u8(fc.cache_k[0]), u8(fc.cache_v[0]),
        fc.k_scale[0].numpy(), fc.v_scale[0].numpy(), batch.pos0.numpy(), batch.n_new.numpy())
    assert skipped == 0
    assert np.array_equal(bits(q), q_ref)
    assert np.array_equal(u8(ck), ck_ref) and np.array_equal(u8(cv), cv_ref)
