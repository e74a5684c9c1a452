"""Split-KV GQA decode and the log-sum-exp combine on the GPU against the fp64
oracle, on the decode workloads: single decode step (valid length 64 with
large garbage past it), the ragged batch of 32 requests with K/V outliers, the
long cache (T = 2048 ragged, T = 1024 full), in both the length-aware and the
masked static-cache modes ("ARK-ASR-3B -- INT8 ONNX", section Shapes: the
static graph attends over all max_total_len positions)."""
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


def gpu_decode(q, ck, cv, kv_len, mode=ops.ARK_LENGTH_AWARE, max_splits=8, status=None):
    dev = "cuda"
    q = q.to(dev)
    ck = ck.to(dev)
    cv = cv.to(dev)
    kv = kv_len.to(dev)
    B, _, Hq, D = q.shape
    T = ck.shape[1]
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ws = ops.decode_workspace(B, Hq, D, T, max_splits)
    ops.ark_attn_decode(q, ck, cv, kv, o, lse, SCALE, mode, max_splits, ws, status)
    torch.cuda.synchronize()
    return o, lse


def oracle_decode(q, ck, cv, kv_len, static=False):
    return oracle.decode(bits(q), bits(ck), bits(cv), kv_len.numpy(), SCALE, static_mode=static)


@pytest.mark.parametrize("max_splits", [1, 2, 8, 32])
@pytest.mark.parametrize("mode", [ops.ARK_LENGTH_AWARE, ops.ARK_MASKED_STATIC])
def test_decode_ragged_small(oracle_lib, max_splits, mode):
    """Ragged lengths with every tail shape: 1, 15, 16, 17, 63, 64, 65, ..., T."""
    T = 200
    kv = torch.tensor([1, 15, 16, 17, 63, 64, 65, 100, 127, 128, 129, 199, 200, 2, 33, 150],
                      dtype=torch.int32)
    B = kv.numel()
    batch = W.make_batch(200 + max_splits, B=B, S=1, T=T, pos0=kv, n_new=torch.zeros(B, dtype=torch.int32),
                         garbage="big" if mode == ops.ARK_MASKED_STATIC else "nan")
    o, lse = gpu_decode(batch.q[0], batch.cache_k[0], batch.cache_v[0], kv, mode, max_splits)
    o_ref, lse_ref = oracle_decode(batch.q[0], batch.cache_k[0], batch.cache_v[0], kv)
    check_o(f64(o), o_ref)
    check_lse(f64(lse), lse_ref)


def test_decode_single_step_layers(oracle_lib):
    """Batch 1, valid length 64, +-1e4 garbage past it, several independent
    layers (the append of the new row is covered by the step tests)."""
    batch = W.cfg_single_decode(layers=4)
    kv = batch.pos0
    for layer in range(4):
        o, lse = gpu_decode(batch.q[layer], batch.cache_k[layer], batch.cache_v[layer], kv)
        o_ref, lse_ref = oracle_decode(batch.q[layer], batch.cache_k[layer], batch.cache_v[layer], kv)
        check_o(f64(o), o_ref)
        check_lse(f64(lse), lse_ref)


@pytest.mark.parametrize("outliers", ["row", "element"])
def test_decode_ragged_batch_32(oracle_lib, outliers):
    batch = W.cfg_ragged_decode(layers=2, outliers=outliers)
    kv = batch.pos0
    for layer in range(2):
        for mode in (ops.ARK_LENGTH_AWARE, ops.ARK_MASKED_STATIC):
            o, lse = gpu_decode(batch.q[layer], batch.cache_k[layer], batch.cache_v[layer], kv, mode)
            o_ref, lse_ref = oracle_decode(batch.q[layer], batch.cache_k[layer], batch.cache_v[layer], kv)
            check_o(f64(o), o_ref)
            check_lse(f64(lse), lse_ref)


@pytest.mark.parametrize("T", [2048, 1024])
def test_decode_long_cache(oracle_lib, T):
    batch = W.cfg_long_decode(layers=1, T=T)
    kv = batch.pos0
    for mode in (ops.ARK_LENGTH_AWARE, ops.ARK_MASKED_STATIC):
        for ms in (8, 32):
            o, lse = gpu_decode(batch.q[0], batch.cache_k[0], batch.cache_v[0], kv, mode, ms)
            o_ref, lse_ref = oracle_decode(batch.q[0], batch.cache_k[0], batch.cache_v[0], kv)
            check_o(f64(o), o_ref)
            check_lse(f64(lse), lse_ref)


@pytest.mark.parametrize("max_splits", [64, 128])
def test_decode_many_pieces_per_request(oracle_lib, max_splits):
    """One long request cut into up to 129 pieces (every warp takes one or two
    tiles), next to short ones: the in-launch merge over many partials."""
    T = 2048
    kv = torch.tensor([2048, 5, 1000, 17], dtype=torch.int32)
    B = kv.numel()
    batch = W.make_batch(250 + max_splits, B=B, S=1, T=T, pos0=kv, n_new=[0] * B, garbage="nan")
    o, lse = gpu_decode(batch.q[0], batch.cache_k[0], batch.cache_v[0], kv, max_splits=max_splits)
    o_ref, lse_ref = oracle_decode(batch.q[0], batch.cache_k[0], batch.cache_v[0], kv)
    check_o(f64(o), o_ref)
    check_lse(f64(lse), lse_ref)


def test_decode_single_valid_row_is_exact(oracle_lib):
    """kv_len = 1: the output is that V row, exactly, after bf16 rounding."""
    B, T = 8, 64
    batch = W.make_batch(300, B=B, S=1, T=T, pos0=[1] * B, n_new=[0] * B, garbage="nan")
    kv = torch.ones(B, dtype=torch.int32)
    o, lse = gpu_decode(batch.q[0], batch.cache_k[0], batch.cache_v[0], kv)
    v0 = batch.cache_v[0][:, 0]                             # [B, 2, 128]
    want = v0.repeat_interleave(8, dim=1).unsqueeze(1)      # [B, 1, 16, 128]
    assert torch.equal(o.cpu(), want)
    _, lse_ref = oracle_decode(batch.q[0], batch.cache_k[0], batch.cache_v[0], kv)
    check_lse(f64(lse), lse_ref)


def test_decode_equal_scores_mean(oracle_lib):
    """q = 0: every score is 0, o = mean of the visible V rows, lse = ln n."""
    B, T = 4, 300
    kv = torch.tensor([300, 7, 64, 129], dtype=torch.int32)
    batch = W.make_batch(301, B=B, S=1, T=T, pos0=kv, n_new=[0] * B, garbage="nan")
    q = torch.zeros_like(batch.q[0])
    o, lse = gpu_decode(q, batch.cache_k[0], batch.cache_v[0], kv, max_splits=4)
    vf = f64(batch.cache_v[0])
    for b in range(B):
        mean = vf[b, :kv[b]].mean(axis=0)                    # [2, 128]
        check_o(f64(o)[b, 0], np.repeat(mean, 8, axis=0))
        check_lse(f64(lse)[b], np.full(16, math.log(kv[b])))


def test_decode_kv_len_out_of_range_sets_status(oracle_lib):
    B, T = 3, 64
    batch = W.make_batch(302, B=B, S=1, T=T, pos0=[10, 10, 10], n_new=[0] * B, garbage="none")
    kv = torch.tensor([0, 70, -3], dtype=torch.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = gpu_decode(batch.q[0], batch.cache_k[0], batch.cache_v[0], kv, max_splits=2, status=status)
    assert int(status.item()) & ops.ARK_DEV_BAD_KVLEN
    o_c, l_c = o.cpu(), lse.cpu()
    assert torch.all(o_c[0] == 0) and torch.all(torch.isinf(l_c[0]))
    assert torch.all(o_c[2] == 0) and torch.all(torch.isinf(l_c[2]))
    o_ref, lse_ref = oracle_decode(batch.q[0][1:2], batch.cache_k[0][1:2], batch.cache_v[0][1:2],
                                   torch.tensor([T], dtype=torch.int32))
    check_o(f64(o)[1:2], o_ref)
    check_lse(f64(lse)[1:2], lse_ref)


def test_decode_split_invariance(oracle_lib):
    """Different split counts give the same result within fp32 rounding."""
    batch = W.cfg_ragged_decode(layers=1, seed=33)
    kv = batch.pos0
    outs = [gpu_decode(batch.q[0], batch.cache_k[0], batch.cache_v[0], kv, max_splits=ms)
            for ms in (1, 3, 8, 32)]
    o0 = f64(outs[0][0])
    for o, lse in outs[1:]:
        assert np.max(np.abs(f64(o) - o0)) <= 2 * 2.0 ** -8 * max(1.0, np.abs(o0).max())
        assert np.max(np.abs(f64(lse) - f64(outs[0][1]))) < 1e-4


def test_combine_matches_oracle(oracle_lib):
    g = torch.Generator().manual_seed(400)
    B, Hq, n, D = 3, 16, 5, 128
    o_part = torch.randn(B, Hq, n, D, generator=g) * 2
    lse_part = torch.randn(B, Hq, n, generator=g) * 4
    lse_part[0, 0, 1] = -math.inf
    lse_part[1, 3, :] = -math.inf
    o_part[0, 0, 1] = float("nan")                # never read: its weight is zero
    o = torch.empty(B, Hq, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    ops.ark_attn_combine(o_part.cuda(), lse_part.cuda(), o, lse)
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(Hq):
            ro, rl = oracle.combine(o_part[b, h].double().numpy(), lse_part[b, h].double().numpy())
            check_o(f64(o)[b, h], ro)
            check_lse(f64(lse)[b, h:h + 1], np.array([rl]))
