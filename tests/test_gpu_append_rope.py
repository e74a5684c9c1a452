"""RoPE + delta write on the GPU against the fp64 oracle: bit-exact.

"ARK-ASR-3B -- INT8 ONNX", section Shapes: key_delta/value_delta rows go into
the static cache at cache_position; RoPE of the Qwen2 decoder (SGLang-Omni
cookbook "ARK-ASR-3B", introduction) is applied to the new q and k rows.
"""
import numpy as np
import pytest
import torch

import oracle
from gqa_attention_static_b200 import ops
from gqa_attention_static_b200 import workloads as W
from tests.helpers import bits

pytestmark = pytest.mark.gpu


def run_gpu_append(batch, layer=0, theta=1e6, table_rows=None):
    dev = "cuda"
    q = batch.q[layer].to(dev).clone()
    kn = batch.k_new[layer].to(dev)
    vn = batch.v_new[layer].to(dev)
    ck = batch.cache_k[layer].to(dev).clone()
    cv = batch.cache_v[layer].to(dev).clone()
    pos0 = batch.pos0.to(dev)
    n_new = batch.n_new.to(dev)
    table = ops.rope_table(table_rows or batch.T, 128, theta)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.ark_attn_append_rope(q, kn, vn, ck, cv, pos0, n_new, table, status)
    torch.cuda.synchronize()
    return q, ck, cv, int(status.item())


def run_oracle_append(batch, layer=0, theta=1e6):
    return oracle.append_rope(bits(batch.q[layer]), bits(batch.k_new[layer]), bits(batch.v_new[layer]),
                              bits(batch.cache_k[layer]), bits(batch.cache_v[layer]),
                              batch.pos0.numpy(), batch.n_new.numpy(), theta)


def assert_bits_equal(got, want, what):
    g = bits(got)
    if not np.array_equal(g, want):
        diff = np.argwhere(g != want)
        raise AssertionError(f"{what}: {len(diff)} bf16 values differ, first at {diff[0].tolist()}: "
                             f"{hex(int(g[tuple(diff[0])]))} vs {hex(int(want[tuple(diff[0])]))}")


@pytest.mark.parametrize("B,S,T,pos0,n_new", [
    (3, 5, 64, [0, 17, 59], [5, 2, 5]),           # ragged, one row past T
    (1, 1, 512, [64], [1]),                        # single decode step
    (2, 7, 40, [33, 0], [7, 0]),                   # empty request
])
def test_append_rope_bit_exact_small(oracle_lib, B, S, T, pos0, n_new):
    batch = W.make_batch(1000 + B * S, B=B, S=S, T=T, pos0=pos0, n_new=n_new, garbage="nan")
    q, ck, cv, st = run_gpu_append(batch)
    q_ref, ck_ref, cv_ref, skipped = run_oracle_append(batch)
    assert_bits_equal(q, q_ref, "q")
    assert_bits_equal(ck, ck_ref, "cache_k")
    assert_bits_equal(cv, cv_ref, "cache_v")
    assert (st & ops.ARK_DEV_BAD_POS != 0) == (skipped > 0)


def test_append_rope_ragged_decode_batch(oracle_lib):
    """32 requests, positions 40..511, K/V outliers (ragged decode workload)."""
    batch = W.cfg_ragged_decode(layers=2)
    for layer in range(2):
        q, ck, cv, st = run_gpu_append(batch, layer)
        q_ref, ck_ref, cv_ref, skipped = run_oracle_append(batch, layer)
        assert st == 0 and skipped == 0
        assert_bits_equal(q, q_ref, "q")
        assert_bits_equal(ck, ck_ref, "cache_k")
        assert_bits_equal(cv, cv_ref, "cache_v")


def test_append_rope_coalesced_prefill(oracle_lib):
    """16 prompts of 20..387 rows from position 0 (coalesced prefill workload)."""
    batch = W.cfg_prefill(layers=1)
    q, ck, cv, st = run_gpu_append(batch)
    q_ref, ck_ref, cv_ref, skipped = run_oracle_append(batch)
    assert st == 0 and skipped == 0
    assert_bits_equal(q, q_ref, "q")
    assert_bits_equal(ck, ck_ref, "cache_k")
    assert_bits_equal(cv, cv_ref, "cache_v")


def test_append_rope_large_positions(oracle_lib):
    """Positions up to 2047 (long-cache workload), where the angles are large."""
    batch = W.make_batch(77, B=4, S=3, T=2048, pos0=[2045, 1500, 0, 1999], n_new=[3, 3, 3, 2])
    q, ck, cv, st = run_gpu_append(batch)
    q_ref, ck_ref, cv_ref, _ = run_oracle_append(batch)
    assert_bits_equal(q, q_ref, "q")
    assert_bits_equal(ck, ck_ref, "cache_k")
    assert_bits_equal(cv, cv_ref, "cache_v")
    assert st == 0


def test_append_rope_bad_n_new_sets_status(oracle_lib):
    batch = W.make_batch(5, B=2, S=2, T=16, pos0=[0, 3], n_new=[2, 1])
    batch.n_new = torch.tensor([5, -1], dtype=torch.int32)   # > S and < 0
    q, ck, cv, st = run_gpu_append(batch)
    assert st & ops.ARK_DEV_BAD_KVLEN
    # clamped to S = 2 and 0 rows
    fixed = W.make_batch(5, B=2, S=2, T=16, pos0=[0, 3], n_new=[2, 0])
    q_ref, ck_ref, cv_ref, _ = run_oracle_append(fixed)
    assert_bits_equal(q, q_ref, "q")
    assert_bits_equal(ck, ck_ref, "cache_k")
