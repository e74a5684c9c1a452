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


def _bf16_from_bits(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _midpoint_distance(v: np.ndarray) -> np.ndarray:
    """|v - nearest bf16 rounding midpoint| / |v| (v float64, nonzero)."""
    _, e = np.frexp(v)
    spacing = np.ldexp(1.0, e - 8)                   # bf16 keeps 8 significant bits
    frac = np.abs(v) / spacing
    return np.abs(frac - np.floor(frac) - 0.5) * spacing / np.abs(v)


def _near_midpoint_rows(table: np.ndarray, S: int, heads: int, n_cand: int, rng) -> np.ndarray:
    """bf16 rows [S, heads, 128] whose rotations x_i c - x_{i+64} s at position t
    (= the row index) land as close to a bf16 rounding midpoint as n_cand random
    candidate pairs allow."""
    out = np.zeros((S, heads, 128), np.uint16)
    for t in range(S):
        c, s = table[t, :, 0][:, None], table[t, :, 1][:, None]
        for h in range(heads):
            sign = rng.integers(0, 2, (64, n_cand, 2), dtype=np.uint16) << 15
            expo = rng.integers(120, 134, (64, n_cand, 2), dtype=np.uint16) << 7
            mant = rng.integers(0, 128, (64, n_cand, 2), dtype=np.uint16)
            cand = sign | expo | mant
            a, z = _bf16_from_bits(cand[..., 0]), _bf16_from_bits(cand[..., 1])
            v = a * c - z * s                          # products exact in double, one rounding
            d = np.where(v != 0, _midpoint_distance(np.where(v != 0, v, 1.0)), 1.0)
            pick = np.argmin(d, axis=1)
            out[t, h, :64] = cand[np.arange(64), pick, 0]
            out[t, h, 64:] = cand[np.arange(64), pick, 1]
    return out


def test_rotation_near_bf16_midpoints(oracle_lib):
    """Rotations whose double result lies within a few fp32 ulps of a bf16
    rounding midpoint (where any shortcut through fp32 would round the wrong
    way) and ones just outside that zone: q and k rows bit-exact against the
    oracle's double-precision rotation."""
    B, S, T = 1, 24, 64
    rng = np.random.default_rng(20261203)
    table = ops.rope_table(T).cpu().numpy().astype(np.float64)     # [T, 64, 2] {cos, sin}
    batch = W.make_batch(77, B=B, S=S, T=T, pos0=[0], n_new=[S])
    q_rows = _near_midpoint_rows(table, S, 16, 4096, rng)
    k_rows = _near_midpoint_rows(table, S, 2, 4096, rng)
    batch.q[0] = torch.from_numpy(q_rows.view(np.int16)).view(torch.bfloat16).view(B, S, 16, 128).clone()
    batch.k_new[0] = torch.from_numpy(k_rows.view(np.int16)).view(torch.bfloat16).view(B, S, 2, 128).clone()
    # how close the first outputs came: some within 2^-22 of a midpoint, most just outside
    a, z = _bf16_from_bits(q_rows[..., :64]), _bf16_from_bits(q_rows[..., 64:])
    v = a * table[:S, None, :, 0] - z * table[:S, None, :, 1]
    d = _midpoint_distance(v[v != 0])
    assert (d < 2.0 ** -22).sum() > 20 and (d > 2.0 ** -19).sum() > 1000
    q, ck, cv, st = run_gpu_append(batch)
    assert st == 0
    q_ref, ck_ref, cv_ref, skipped = run_oracle_append(batch)
    assert skipped == 0
    assert np.array_equal(bits(q), q_ref), f"q differs at {np.argwhere(bits(q) != q_ref)[:5]}"
    assert np.array_equal(bits(ck), ck_ref) and np.array_equal(bits(cv), cv_ref)
