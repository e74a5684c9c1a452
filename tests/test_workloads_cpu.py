"""The synthetic input recipes of the encoder attention and the projection
step (no GPU): clip lengths from the audio handling of the SGLang-Omni cookbook
"ARK-ASR-3B" (30 s truncation, stride-2 convolution after 100 mel frames per
second, batches of up to 8), garbage past each clip's length, and the scales
of the random-init projection."""
import math

import torch

from gqa_attention_static_b200 import workloads as W


def test_encoder_frames_follow_the_mel_rate_and_truncation():
    assert W.encoder_frames(30.0) == 1500
    assert W.encoder_frames(3.0) == 150
    assert W.encoder_frames(45.0) == 1500          # truncated at 30 s
    assert W.encoder_frames(0.001) == 1


def test_encoder_batch_lengths_and_garbage():
    e = W.cfg_encoder(layers=1)
    assert e.B == 8 and e.S == 1500
    lengths = e.length.tolist()
    assert all(150 <= n <= 1500 for n in lengths)
    for x in (e.q[0], e.k[0], e.v[0]):
        assert tuple(x.shape) == (8, 1500, W.ENC_HEADS, W.ENC_HEAD_DIM) and x.dtype == torch.bfloat16
        for b, n in enumerate(lengths):
            assert torch.isfinite(x[b, :n].float()).all()
            if n < 1500:
                # NaN / +-inf / +-1e4 past the clip: not N(0, 1)
                tail = x[b, n:].float()
                assert (~torch.isfinite(tail)).any() or tail.abs().max() > 100


def test_projection_weights_have_the_stated_scales():
    w, b = W.make_qkv_weights(1)
    assert tuple(w.shape) == (2560, 2048) and tuple(b.shape) == (2560,)
    assert abs(w.float().std().item() - 1 / math.sqrt(2048)) < 0.02 / math.sqrt(2048)
    assert abs(b.float().std().item() - 0.1) < 0.01
    x = W.make_hidden(2, 4, 8)
    assert tuple(x.shape) == (4, 8, 2048) and abs(x.float().std().item() - 1.0) < 0.05
