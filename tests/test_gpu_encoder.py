"""Bidirectional multi-head attention of the audio encoder on the tcgen05
tensor cores against the fp64 oracle ("Inside ARK-ASR-3B's Whisper and Qwen
architecture", encoder components; "ARK-ASR-3B -- INT8 ONNX", Inference step 1;
clip lengths and batch from the SGLang-Omni cookbook "ARK-ASR-3B", audio
handling).  Heads of 64 dims, every frame of a clip attends to every frame of
the same clip, frames past a clip's length neither attend nor are attended."""
import math

import numpy as np
import pytest
import torch

import oracle
from gqa_attention_static_b200 import ops
from gqa_attention_static_b200 import workloads as W
from tests.helpers import bits, check_lse, check_o, f64

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(64)
SENTINEL = 0x7FC1            # a NaN pattern the kernel never writes


def gpu_encoder(q, k, v, length, status=None):
    dev = "cuda"
    q, k, v = (x.to(dev).contiguous() for x in (q, k, v))
    B, S, H, D = q.shape
    o = torch.empty_like(q).view(torch.int16).fill_(SENTINEL).view(torch.bfloat16)
    lse = torch.full((B, H, S), float("nan"), dtype=torch.float32, device=dev)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.ark_attn_encoder(q, k, v, length.to(dev), o, lse, SCALE, status)
    torch.cuda.synchronize()
    return o, lse, int(status.item())


def compare(q, k, v, length, heads=None, status_expected=0):
    """GPU over all heads; the oracle over `heads` (all by default): heads are
    independent problems, so a subset is compared element by element."""
    o, lse, st = gpu_encoder(q, k, v, length)
    assert st == status_expected
    H = q.shape[2]
    hs = list(range(H)) if heads is None else list(heads)
    sel = lambda x: np.ascontiguousarray(bits(x)[:, :, hs])
    o_ref, lse_ref = oracle.attention_bidir(sel(q), sel(k), sel(v), length.numpy(), SCALE)
    ob = bits(o)
    of = f64(o)[:, :, hs]
    lf = f64(lse)[:, hs]
    lf_all = f64(lse)
    S = q.shape[1]
    for b in range(q.shape[0]):
        n = min(max(int(length[b]), 0), S)
        check_o(of[b, :n], o_ref[b, :n], f"o clip {b}")
        check_lse(lf[b, :, :n], lse_ref[b, :, :n], f"lse clip {b}")
        assert np.all(ob[b, n:] == SENTINEL), f"clip {b}: frames past the length were written"
        assert np.all(np.isnan(lf_all[b, :, n:]))
        assert np.isfinite(f64(o)[b, :n]).all() and np.isfinite(lf_all[b, :, :n]).all()


@pytest.mark.parametrize("B,S,H,lengths", [
    (3, 300, 3, [300, 1, 131]),             # ragged tails: 3 tiles of 128 frames, key blocks of 64
    (2, 128, 2, [128, 64]),                 # exactly one tile / one key block
    (2, 70, 4, [5, 70]),                    # shorter than a key block; one partial block
    (1, 1500, 2, [1500]),                   # the 30-second clip: 12 tiles, 24 key blocks
    (4, 200, 1, [0, 200, 199, 65]),         # an empty clip writes nothing
])
def test_encoder_small_cases(oracle_lib, B, S, H, lengths):
    e = W.make_encoder_batch(900 + S + B, B=B, S=S, lengths=lengths, H=H, garbage="nan")
    compare(e.q[0], e.k[0], e.v[0], e.length)


def test_encoder_large_scores_rescale(oracle_lib):
    """q scaled by 8: scores spread over tens of units, so the running maximum
    moves past the lazy-rescale threshold many times along a row."""
    e = W.make_encoder_batch(31, B=2, S=700, lengths=[700, 333], H=2, garbage="big")
    q = (e.q[0].float() * 8).to(torch.bfloat16)
    compare(q, e.k[0], e.v[0], e.length)


def test_encoder_outlier_keys(oracle_lib):
    """A few keys 8x larger than the rest dominate their rows' softmax."""
    e = W.make_encoder_batch(32, B=2, S=400, lengths=[400, 257], H=2, garbage="none")
    g = torch.Generator().manual_seed(5)
    k = e.k[0].clone()
    W.add_row_outliers_(k, g)
    compare(e.q[0], k, e.v[0], e.length)


def test_encoder_batch_full_size(oracle_lib):
    """The encoder batch at its full size: 8 clips of 3..30 s padded to 1500
    frames, 20 heads; every head computed, heads 0, 7 and 19 compared with the
    oracle element by element."""
    e = W.cfg_encoder(layers=1)
    compare(e.q[0], e.k[0], e.v[0], e.length, heads=[0, 7, 19])


def test_encoder_heads_are_independent(oracle_lib):
    """The full batch and the same batch with one head's inputs alone give the
    same bits for that head (no cross-head mixing in the tiling)."""
    e = W.cfg_encoder(layers=1, seed=40)
    o_all, lse_all, _ = gpu_encoder(e.q[0], e.k[0], e.v[0], e.length)
    h = 11
    one = lambda x: x[:, :, h:h + 1].contiguous()
    o_one, lse_one, _ = gpu_encoder(one(e.q[0]), one(e.k[0]), one(e.v[0]), e.length)
    for b in range(e.B):
        n = int(e.length[b])
        assert torch.equal(o_all[b, :n, h], o_one[b, :n, 0])
        assert torch.equal(lse_all[b, h, :n], lse_one[b, 0, :n])


def test_encoder_bad_length_clamped_and_reported(oracle_lib):
    """A length above S is clamped to S and flagged in the device status."""
    e = W.make_encoder_batch(33, B=2, S=150, lengths=[150, 90], H=1, garbage="none")
    length = torch.tensor([150, 999], dtype=torch.int32)
    o, lse, st = gpu_encoder(e.q[0], e.k[0], e.v[0], length)
    assert st & ops.ARK_DEV_BAD_KVLEN
    o_ref, lse_ref = oracle.attention_bidir(bits(e.q[0]), bits(e.k[0]), bits(e.v[0]), np.array([150, 150]), SCALE)
    check_o(f64(o), o_ref)
    check_lse(f64(lse), lse_ref)
