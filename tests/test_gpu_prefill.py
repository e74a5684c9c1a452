"""Causal prefill on the tcgen05 tensor cores against the fp64 oracle.

The prompt's rows are appended (RoPE + delta write) and then prefilled, on the
GPU through the C ABI and in the oracle from the same inputs
("ARK-ASR-3B -- INT8 ONNX", sections Inference and Shapes: prefill of the
audio+text prompt, rows written at cache_position)."""
import math

import numpy as np
import pytest
import torch

import oracle
from gqa_attention_static_b200 import ops
from gqa_attention_static_b200 import workloads as W
from tests.helpers import bits, check_lse, check_o, f64

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)
SENTINEL = 0x7FC1            # a NaN pattern no kernel writes


def gpu_append_prefill(batch, layer=0, status=None):
    dev = "cuda"
    q = batch.q[layer].to(dev).clone()
    ck = batch.cache_k[layer].to(dev).clone()
    cv = batch.cache_v[layer].to(dev).clone()
    pos0 = batch.pos0.to(dev)
    n_new = batch.n_new.to(dev)
    table = ops.rope_table(batch.T)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.ark_attn_append_rope(q, batch.k_new[layer].to(dev), batch.v_new[layer].to(dev), ck, cv, pos0, n_new,
                             table, status)
    B, S, Hq, D = q.shape
    o = torch.empty_like(q).view(torch.int16).fill_(SENTINEL).view(torch.bfloat16)
    lse = torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=dev)
    ops.ark_attn_prefill(q, ck, cv, pos0, n_new, o, lse, SCALE, status)
    torch.cuda.synchronize()
    return q, ck, cv, o, lse, int(status.item())


def oracle_append_prefill(batch, layer=0):
    q_rot, ck, cv, skipped = oracle.append_rope(bits(batch.q[layer]), bits(batch.k_new[layer]),
                                                bits(batch.v_new[layer]), bits(batch.cache_k[layer]),
                                                bits(batch.cache_v[layer]), batch.pos0.numpy(), batch.n_new.numpy())
    o, lse = oracle.prefill(q_rot, ck, cv, batch.pos0.numpy(), batch.n_new.numpy(), SCALE)
    return q_rot, ck, cv, o, lse


def compare(batch, layer=0, status_expected=0):
    q, ck, cv, o, lse, st = gpu_append_prefill(batch, layer)
    q_ref, ck_ref, cv_ref, o_ref, lse_ref = oracle_append_prefill(batch, layer)
    assert st == status_expected
    assert np.array_equal(bits(q), q_ref) and np.array_equal(bits(ck), ck_ref) and np.array_equal(bits(cv), cv_ref)
    ob = bits(o)
    of = f64(o)
    lf = f64(lse)
    for b in range(batch.B):
        n = int(batch.n_new[b])
        check_o(of[b, :n], o_ref[b, :n], f"o request {b}")
        check_lse(lf[b, :, :n], lse_ref[b, :, :n], f"lse request {b}")
        # rows past n_new are not written
        assert np.all(ob[b, n:] == SENTINEL), f"request {b}: padded rows were written"
        assert np.all(np.isnan(lf[b, :, n:]))


@pytest.mark.parametrize("B,S,T,pos0,n_new", [
    (3, 40, 256, [0, 30, 100], [40, 17, 1]),         # ragged tails, tiles of 16 positions
    (2, 16, 64, [0, 48], [16, 16]),                  # exact one tile, cache ending at T
    (1, 5, 8, [3], [5]),                             # smaller than a tile and than a KV block
    (2, 130, 512, [0, 380], [130, 2]),               # two KV blocks, last one partial
    (1, 200, 2048, [1700], [200]),                   # long context: 15 KV blocks
    (5, 33, 96, [0, 7, 31, 63, 40], [33, 0, 32, 33, 17]),   # empty request, unit = 32 rows + 1, odd positions
])
def test_prefill_small_cases(oracle_lib, B, S, T, pos0, n_new):
    batch = W.make_batch(500 + S + T, B=B, S=S, T=T, pos0=pos0, n_new=n_new, garbage="nan")
    compare(batch)


def test_prefill_sweep_prompt(oracle_lib):
    """The batch-1 prompt of the autoregressive sweep: 50 rows from position 0."""
    batch = W.cfg_sweep_prefill(layers=2)
    for layer in range(2):
        compare(batch, layer)


def test_prefill_coalesced_batch_full_size(oracle_lib):
    """Coalesced prefill at its full size: 16 prompts of 20..387 rows, T=512."""
    batch = W.cfg_prefill(layers=1)
    compare(batch)


def test_prefill_many_requests(oracle_lib):
    """More requests than a warp has lanes (the unit list's per-request counts
    take two rounds), lengths of every residue mod 16 and 32."""
    g = torch.Generator().manual_seed(93)
    n_new = torch.randint(1, 70, (45,), generator=g).tolist()
    pos0 = torch.randint(0, 60, (45,), generator=g).tolist()
    batch = W.make_batch(93, B=45, S=70, T=130, pos0=pos0, n_new=n_new, garbage="nan")
    compare(batch)


def test_prefill_outliers(oracle_lib):
    batch = W.make_batch(77, B=4, S=64, T=128, pos0=[0, 10, 60, 64], n_new=[64, 50, 3, 64], outliers="row")
    compare(batch)


def test_prefill_rows_match_decode(oracle_lib):
    """Causal consistency on the GPU: prefill row t equals a decode over
    pos0 + t + 1 rows of the same cache (both within tolerance of each other)."""
    batch = W.make_batch(91, B=2, S=24, T=128, pos0=[0, 40], n_new=[24, 20])
    q, ck, cv, o, lse, st = gpu_append_prefill(batch)
    assert st == 0
    dev = "cuda"
    for b in range(2):
        for t in range(int(batch.n_new[b])):
            kv = torch.tensor([int(batch.pos0[b]) + t + 1], dtype=torch.int32, device=dev)
            qd = q[b:b + 1, t:t + 1].contiguous()
            od = torch.empty_like(qd)
            ld = torch.empty(1, 16, dtype=torch.float32, device=dev)
            ws = ops.decode_workspace(1, 16, 128, 128, 8, device=dev)
            ops.ark_attn_decode(qd, ck[b:b + 1].contiguous(), cv[b:b + 1].contiguous(), kv, od, ld, SCALE,
                                ops.ARK_LENGTH_AWARE, 8, ws)
            torch.cuda.synchronize()
            check_o(f64(o[b, t]), f64(od[0, 0]), "prefill vs decode")
            check_lse(f64(lse[b, :, t]), f64(ld[0]), "prefill vs decode lse")


def test_prefill_bad_lengths_set_status(oracle_lib):
    batch = W.make_batch(92, B=2, S=8, T=16, pos0=[12, 0], n_new=[8, 4])   # 12 + 8 > 16
    dev = "cuda"
    q = batch.q[0].to(dev)
    ck = batch.cache_k[0].to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(2, 16, 8, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.ark_attn_prefill(q, ck, ck, batch.pos0.to(dev), batch.n_new.to(dev), o, lse, SCALE, status)
    torch.cuda.synchronize()
    assert int(status.item()) & ops.ARK_DEV_BAD_POS


def test_prefill_layers_matches_oracle(oracle_lib):
    """ark_attn_prefill_layers: three layers with their own caches in one
    launch, each against the oracle (the same causal prefill per layer)."""
    L = 3
    batch = W.make_batch(510, B=3, S=40, T=256, pos0=[0, 30, 100], n_new=[40, 17, 5], layers=L, garbage="nan")
    dev = "cuda"
    q = [x.to(dev).clone() for x in batch.q]
    ck = [x.to(dev).clone() for x in batch.cache_k]
    cv = [x.to(dev).clone() for x in batch.cache_v]
    pos0, n_new = batch.pos0.to(dev), batch.n_new.to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.ark_attn_append_rope_layers(q, [x.to(dev) for x in batch.k_new], [x.to(dev) for x in batch.v_new], ck, cv,
                                    pos0, n_new, ops.rope_table(batch.T), status)
    B, S, Hq, D = q[0].shape
    o = [torch.empty_like(x).view(torch.int16).fill_(SENTINEL).view(torch.bfloat16) for x in q]
    lse = [torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=dev) for _ in q]
    ops.ark_attn_prefill_layers(q, ck, cv, pos0, n_new, o, lse, SCALE, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for l in range(L):
        q_ref, ck_ref, cv_ref, o_ref, lse_ref = oracle_append_prefill(batch, l)
        for b in range(B):
            n = int(batch.n_new[b])
            check_o(f64(o[l])[b, :n], o_ref[b, :n], f"o layer {l} request {b}")
            check_lse(f64(lse[l])[b, :, :n], lse_ref[b, :, :n], f"lse layer {l} request {b}")
            assert np.all(bits(o[l])[b, n:] == SENTINEL)


def test_prefill_layers_across_launches_equals_single_layer_calls(oracle_lib):
    """40 layers take two launches (20 + 20); every layer's output is bit for bit
    the single-layer call's (the same tile arithmetic), padded rows untouched."""
    L = 40
    batch = W.make_batch(511, B=2, S=20, T=64, pos0=[0, 37], n_new=[20, 9], layers=L)
    dev = "cuda"
    q = [x.to(dev).clone() for x in batch.q]
    ck = [x.to(dev).clone() for x in batch.cache_k]
    cv = [x.to(dev).clone() for x in batch.cache_v]
    pos0, n_new = batch.pos0.to(dev), batch.n_new.to(dev)
    ops.ark_attn_append_rope_layers(q, [x.to(dev) for x in batch.k_new], [x.to(dev) for x in batch.v_new], ck, cv,
                                    pos0, n_new, ops.rope_table(batch.T))
    B, S, Hq, D = q[0].shape
    o = [torch.empty_like(x).view(torch.int16).fill_(SENTINEL).view(torch.bfloat16) for x in q]
    lse = [torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=dev) for _ in q]
    ops.ark_attn_prefill_layers(q, ck, cv, pos0, n_new, o, lse, SCALE)
    for l in range(L):
        o1 = torch.empty_like(q[l]).view(torch.int16).fill_(SENTINEL).view(torch.bfloat16)
        l1 = torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=dev)
        ops.ark_attn_prefill(q[l], ck[l], cv[l], pos0, n_new, o1, l1, SCALE)
        torch.cuda.synchronize()
        assert torch.equal(o[l].view(torch.int16), o1.view(torch.int16)), f"layer {l}"
        assert torch.equal(torch.nan_to_num(lse[l], nan=-7.0), torch.nan_to_num(l1, nan=-7.0)), f"layer {l}"


def _two_paths(batch, L):
    """(a) append_rope + prefill_layers, (b) append_rope_kv + prefill_rope_layers,
    on identical inputs; returns both results and the untouched q of (b)."""
    dev = "cuda"
    out = []
    for fused in (False, True):
        q = [x.to(dev).clone() for x in batch.q[:L]]
        ck = [x.to(dev).clone() for x in batch.cache_k[:L]]
        cv = [x.to(dev).clone() for x in batch.cache_v[:L]]
        pos0, n_new = batch.pos0.to(dev), batch.n_new.to(dev)
        kn = [x.to(dev) for x in batch.k_new[:L]]
        vn = [x.to(dev) for x in batch.v_new[:L]]
        table = ops.rope_table(batch.T)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        B, S, Hq, D = q[0].shape
        o = [torch.empty_like(x).view(torch.int16).fill_(SENTINEL).view(torch.bfloat16) for x in q]
        lse = [torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=dev) for _ in q]
        if fused:
            ops.ark_attn_append_rope_kv_layers(kn, vn, ck, cv, pos0, n_new, table, Hq, status)
            ops.ark_attn_prefill_rope_layers(q, ck, cv, pos0, n_new, o, lse, SCALE, table, status)
        else:
            ops.ark_attn_append_rope_layers(q, kn, vn, ck, cv, pos0, n_new, table, status)
            ops.ark_attn_prefill_layers(q, ck, cv, pos0, n_new, o, lse, SCALE, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        out.append((q, ck, cv, o, lse))
    return out


@pytest.mark.parametrize("B,S,T,pos0,n_new", [
    (3, 40, 256, [0, 30, 100], [40, 17, 1]),
    (1, 5, 8, [3], [5]),
    (1, 200, 2048, [1700], [200]),
])
def test_prefill_rope_on_load_equals_append_then_prefill(oracle_lib, B, S, T, pos0, n_new):
    """RoPE applied by the prefill as it loads q gives the same o and lse, bit
    for bit, as rotating q in the append first; the K/V-only append writes the
    same cache bytes and leaves q untouched."""
    L = 2
    batch = W.make_batch(520 + S, B=B, S=S, T=T, pos0=pos0, n_new=n_new, layers=L, garbage="nan")
    (qa, cka, cva, oa, la), (qb, ckb, cvb, ob, lb) = _two_paths(batch, L)
    for l in range(L):
        assert torch.equal(cka[l].view(torch.int16), ckb[l].view(torch.int16))
        assert torch.equal(cva[l].view(torch.int16), cvb[l].view(torch.int16))
        assert torch.equal(qb[l].view(torch.int16), batch.q[l].cuda().view(torch.int16))
        assert torch.equal(oa[l].view(torch.int16), ob[l].view(torch.int16)), f"layer {l}: o differs"
        assert torch.equal(torch.nan_to_num(la[l], nan=-7.0), torch.nan_to_num(lb[l], nan=-7.0)), f"layer {l}"


def test_prefill_rope_on_load_coalesced_full_size(oracle_lib):
    batch = W.cfg_prefill(layers=2)
    (qa, cka, cva, oa, la), (qb, ckb, cvb, ob, lb) = _two_paths(batch, 2)
    for l in range(2):
        assert torch.equal(oa[l].view(torch.int16), ob[l].view(torch.int16)), f"layer {l}: o differs"
        assert torch.equal(torch.nan_to_num(la[l], nan=-7.0), torch.nan_to_num(lb[l], nan=-7.0))
        assert torch.equal(cka[l].view(torch.int16), ckb[l].view(torch.int16))


@pytest.mark.parametrize("fused", [False, True])
def test_prefill_36_layers_one_launch_equals_single_layer_calls(oracle_lib, fused):
    """The coalesced batch at full size over 36 layers in one launch, where every
    CTA walks some 54 units through its rings (Q slots, K/V stages, the list
    entries, the output staging), equals 36 single-layer calls (a CTA walks at
    most two units there) bit for bit, padded rows untouched; two layers are
    also compared with the oracle.  Both forms: q rotated by the append, and q
    rotated as the prefill loads it."""
    L = 36
    batch = W.cfg_prefill(layers=L, device="cuda")
    dev = "cuda"
    B, S, Hq, D = batch.q[0].shape
    table = ops.rope_table(batch.T)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ck = [x.clone() for x in batch.cache_k]
    cv = [x.clone() for x in batch.cache_v]
    q = [x.clone() for x in batch.q]
    if fused:
        ops.ark_attn_append_rope_kv_layers(batch.k_new, batch.v_new, ck, cv, batch.pos0, batch.n_new, table, Hq,
                                           status)
    else:
        ops.ark_attn_append_rope_layers(q, batch.k_new, batch.v_new, ck, cv, batch.pos0, batch.n_new, table, status)
    o = [torch.empty_like(x).view(torch.int16).fill_(SENTINEL).view(torch.bfloat16) for x in q]
    lse = [torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=dev) for _ in q]
    if fused:
        ops.ark_attn_prefill_rope_layers(q, ck, cv, batch.pos0, batch.n_new, o, lse, SCALE, table, status)
    else:
        ops.ark_attn_prefill_layers(q, ck, cv, batch.pos0, batch.n_new, o, lse, SCALE, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for l in range(L):
        o1 = torch.empty_like(q[l]).view(torch.int16).fill_(SENTINEL).view(torch.bfloat16)
        l1 = torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=dev)
        if fused:
            ops.ark_attn_prefill_rope_layers([q[l]], [ck[l]], [cv[l]], batch.pos0, batch.n_new, [o1], [l1], SCALE,
                                             table, status)
        else:
            ops.ark_attn_prefill(q[l], ck[l], cv[l], batch.pos0, batch.n_new, o1, l1, SCALE, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(o[l].view(torch.int16), o1.view(torch.int16)), f"layer {l}"
        assert torch.equal(torch.nan_to_num(lse[l], nan=-7.0), torch.nan_to_num(l1, nan=-7.0)), f"layer {l}"
    for l in (0, 35):
        cpu = lambda x: x.cpu()
        one = W.Batch([cpu(batch.q[l])], [cpu(batch.k_new[l])], [cpu(batch.v_new[l])], [cpu(batch.cache_k[l])],
                      [cpu(batch.cache_v[l])], cpu(batch.pos0), cpu(batch.n_new), batch.T, batch.S)
        q_ref, ck_ref, cv_ref, o_ref, lse_ref = oracle_append_prefill(one)
        assert np.array_equal(bits(ck[l]), ck_ref) and np.array_equal(bits(cv[l]), cv_ref)
        for b in range(B):
            n = int(batch.n_new[b])
            check_o(f64(o[l])[b, :n], o_ref[b, :n], f"o layer {l} request {b}")
            check_lse(f64(lse[l])[b, :, :n], lse_ref[b, :, :n], f"lse layer {l} request {b}")
            assert np.all(bits(o[l])[b, n:] == SENTINEL)
