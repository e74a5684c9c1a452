"""Whole decode steps (RoPE + delta write, then decode attention) on the GPU
against the oracle doing the same steps from the same inputs, on the decode
workloads at their full sizes and in the launch configuration the benchmark
times (gqa_attention_static_b200.step.DecodeStep)."""
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
BENCH_MAX_SPLITS = 8


def run_step(batch, mode=ops.ARK_LENGTH_AWARE, max_splits=BENCH_MAX_SPLITS, batched=True):
    dev = "cuda"
    q = [x.to(dev).clone() for x in batch.q]
    kn = [x.to(dev) for x in batch.k_new]
    vn = [x.to(dev) for x in batch.v_new]
    ck = [x.to(dev).clone() for x in batch.cache_k]
    cv = [x.to(dev).clone() for x in batch.cache_v]
    step = DecodeStep(q, kn, vn, ck, cv, batch.pos0.to(dev), batch.n_new.to(dev), batch.kv_len.to(dev),
                      max_splits=max_splits, mode=mode, batched=batched)
    step.run()
    torch.cuda.synchronize()
    return step


def oracle_step(batch, layer):
    q_rot, ck, cv, skipped = oracle.append_rope(bits(batch.q[layer]), bits(batch.k_new[layer]),
                                                bits(batch.v_new[layer]), bits(batch.cache_k[layer]),
                                                bits(batch.cache_v[layer]), batch.pos0.numpy(),
                                                batch.n_new.numpy())
    assert skipped == 0
    o, lse = oracle.decode(q_rot, ck, cv, batch.kv_len.numpy(), SCALE)
    return q_rot, ck, cv, o, lse


def compare(step, batch, layers):
    assert int(step.status.item()) == 0
    for l in layers:
        q_rot, ck, cv, o_ref, lse_ref = oracle_step(batch, l)
        assert np.array_equal(bits(step.q[l]), q_rot), f"layer {l}: rotated q differs"
        assert np.array_equal(bits(step.cache_k[l]), ck), f"layer {l}: cache_k differs"
        assert np.array_equal(bits(step.cache_v[l]), cv), f"layer {l}: cache_v differs"
        check_o(f64(step.o[l]), o_ref, f"o layer {l}")
        check_lse(f64(step.lse[l]), lse_ref, f"lse layer {l}")


@pytest.mark.parametrize("batched", [True, False])
def test_step_single_decode_36_layers(oracle_lib, batched):
    """Batch 1, 36 layers, 64 valid rows + the new row at position 64."""
    batch = W.cfg_single_decode()
    step = run_step(batch, batched=batched)
    compare(step, batch, range(36))


def test_step_with_lengths_advanced_on_the_device(oracle_lib):
    """Lengths kept on the device and advanced there by a kernel on the same
    stream right before the step (a serving loop that never copies kv_len back
    to the host): the decode reads kv_len only after the kernels before it on
    the stream are done, so it attends over the advanced lengths."""
    batch = W.cfg_ragged_decode(layers=4)
    dev = "cuda"
    q = [x.to(dev).clone() for x in batch.q]
    kn = [x.to(dev) for x in batch.k_new]
    vn = [x.to(dev) for x in batch.v_new]
    ck = [x.to(dev).clone() for x in batch.cache_k]
    cv = [x.to(dev).clone() for x in batch.cache_v]
    kv_dev = batch.pos0.to(dev).clone()          # the lengths before this step's new row
    step = DecodeStep(q, kn, vn, ck, cv, batch.pos0.to(dev), batch.n_new.to(dev), kv_dev,
                      max_splits=BENCH_MAX_SPLITS, batched=True)
    torch.cuda.synchronize()
    kv_dev.add_(batch.n_new.to(dev))             # advanced on the device, on the step's stream
    step.run()
    torch.cuda.synchronize()
    assert torch.equal(kv_dev.cpu(), batch.kv_len)
    compare(step, batch, range(4))


@pytest.mark.parametrize("batched", [True, False])
def test_step_ragged_batch_full_size(oracle_lib, batched):
    """Ragged batch of 32, 36 layers, T = 512: the benchmark's workload at its
    full size and launch configuration, every output compared."""
    batch = W.cfg_ragged_decode()
    step = run_step(batch, batched=batched)
    compare(step, batch, range(36))


def test_step_repeated_calls_reuse_workspace(oracle_lib):
    """The workspace carries nothing from one call to the next: consecutive
    steps give the same results (the same step three times, with q restored),
    also after the workspace has been overwritten with NaN bytes."""
    batch = W.cfg_ragged_decode(layers=3, seed=21)
    step = run_step(batch)
    o1 = [x.clone() for x in step.o]
    for _ in range(2):
        for l in range(3):
            step.q[l].copy_(batch.q[l].cuda())
        step.workspace.fill_(0xFF)
        step.run()
    torch.cuda.synchronize()
    for l in range(3):
        assert torch.equal(step.o[l], o1[l])
    ws = step.workspace
    assert ws is not None


def test_step_ragged_batch_masked_static(oracle_lib):
    batch = W.cfg_ragged_decode(layers=4)
    step = run_step(batch, mode=ops.ARK_MASKED_STATIC)
    compare(step, batch, range(4))


@pytest.mark.parametrize("T", [2048, 1024])
@pytest.mark.parametrize("mode", [ops.ARK_LENGTH_AWARE, ops.ARK_MASKED_STATIC])
@pytest.mark.parametrize("max_splits", [8, 32])
def test_step_long_cache(oracle_lib, T, mode, max_splits):
    """T = 2048 with 1501..2048 rows read, and T = 1024 full (1024 rows)."""
    batch = W.cfg_long_decode(layers=2, T=T)
    step = run_step(batch, mode=mode, max_splits=max_splits)
    compare(step, batch, range(2))


def test_step_is_graph_capturable(oracle_lib):
    """The step captured in a CUDA graph gives the eager result."""
    batch = W.cfg_ragged_decode(layers=3, seed=11)
    eager = run_step(batch)
    dev = "cuda"
    q = [x.to(dev).clone() for x in batch.q]
    ck = [x.to(dev).clone() for x in batch.cache_k]
    cv = [x.to(dev).clone() for x in batch.cache_v]
    step = DecodeStep(q, [x.to(dev) for x in batch.k_new], [x.to(dev) for x in batch.v_new], ck, cv,
                      batch.pos0.to(dev), batch.n_new.to(dev), batch.kv_len.to(dev))
    q0 = [x.clone() for x in q]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step.run()
    for a, b_ in zip(q, q0):
        a.copy_(b_)
    g.replay()
    torch.cuda.synchronize()
    for l in range(3):
        assert torch.equal(step.o[l], eager.o[l])
        assert torch.equal(step.lse[l], eager.lse[l])
