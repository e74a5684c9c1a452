"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
brute force on tiny inputs, closed forms, invariants of softmax attention and of
the rotary embedding, a library routine on a special case, and the prompt-length
worked values of the pages.  CPU only.

Pages cited: "ARK-ASR-3B -- INT8 ONNX" model card (sections Shapes, Inference),
SGLang-Omni cookbook "ARK-ASR-3B" (introduction, Audio Handling, dtype).
"""
import math
import os


import numpy as np
import pytest
import torch

import oracle
from gqa_attention_static_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def rand_bits(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return bf16_bits(torch.randn(shape, generator=g) * scale)


# ------------------------------------------------------------------ bf16 ----

def _all_bf16_finite_sorted():
    pats = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    vals = oracle.bf16_array_to_f64(pats)
    fin = np.isfinite(vals)
    pats, vals = pats[fin], vals[fin]
    # one entry per value (+0/-0 collapse); keep +0
    order = np.lexsort((pats, vals))
    vals, pats = vals[order], pats[order]
    keep = np.concatenate([[True], vals[1:] != vals[:-1]])
    return vals[keep], pats[keep]


def brute_nearest_bf16(x: float, vals, pats) -> int:
    """Nearest bf16 by exhaustive search over all finite bf16 values; ties go
    to the one with an even last mantissa bit."""
    i = np.searchsorted(vals, x)
    cands = [k for k in (i - 1, i) if 0 <= k < len(vals)]
    best = min(cands, key=lambda k: (abs(vals[k] - x), int(pats[k]) & 1))
    return int(pats[best])


def test_bf16_widening_known_patterns(oracle_lib):
    assert oracle.bf16_to_f64(np.array([0x3F80], np.uint16))[0] == 1.0
    assert oracle.bf16_to_f64(np.array([0xC000], np.uint16))[0] == -2.0
    assert oracle.bf16_to_f64(np.array([0x0001], np.uint16))[0] == 2.0 ** -133
    assert oracle.bf16_to_f64(np.array([0x7F7F], np.uint16))[0] == (2 - 2 ** -7) * 2.0 ** 127
    assert math.isinf(oracle.bf16_to_f64(np.array([0x7F80], np.uint16))[0])


def test_bf16_rounding_matches_exhaustive_search(oracle_lib):
    vals, pats = _all_bf16_finite_sorted()
    rng = np.random.default_rng(0)
    xs = list(rng.standard_normal(3000) * np.exp(rng.uniform(-20, 20, 3000)))
    # exact midpoints between neighbours (the tie cases), and near-boundaries
    for k in rng.integers(1, len(vals) - 2, 500):
        mid = (vals[k] + vals[k + 1]) / 2.0
        xs += [mid, np.nextafter(mid, np.inf), np.nextafter(mid, -np.inf)]
    xs += [2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, 2.0 ** -126 * 1.00390625, 1e-300,
           (2 - 2 ** -7) * 2.0 ** 127, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8]
    got = oracle.f64_to_bf16(np.array(xs))
    for x, g in zip(xs, got):
        want = brute_nearest_bf16(float(x), vals, pats)
        # signed zero: brute force returns +0 for tiny negatives; compare values
        if oracle.bf16_array_to_f64(np.array([want], np.uint16))[0] == 0.0:
            assert oracle.bf16_array_to_f64(np.array([g], np.uint16))[0] == 0.0
        else:
            assert int(g) == want, (x, hex(int(g)), hex(want))


def test_bf16_overflow_and_specials(oracle_lib):
    top = (2 - 2 ** -7) * 2.0 ** 127
    half_ulp = 2.0 ** (127 - 8)
    assert int(oracle.f64_to_bf16(np.array([top + half_ulp]))[0]) == 0x7F80  # tie rounds up to inf
    assert int(oracle.f64_to_bf16(np.array([top + half_ulp * 0.99]))[0]) == 0x7F7F
    assert int(oracle.f64_to_bf16(np.array([-np.inf]))[0]) == 0xFF80
    assert int(oracle.f64_to_bf16(np.array([np.nan]))[0]) & 0x7F80 == 0x7F80


# ------------------------------------------------------------------ RoPE ----

def test_rope_rotation_preserves_norm(oracle_lib):
    """A rotation of each (i, i+64) pair preserves the row norm exactly in
    real arithmetic: a wrong sign or a wrong partner breaks it."""
    rng = np.random.default_rng(1)
    for _ in range(20):
        x = rng.standard_normal(128)
        ang = rng.uniform(-50, 50, 64)
        y = oracle.rope_rotate(x, np.cos(ang), np.sin(ang))
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12 * np.linalg.norm(x)


def test_rope_pairs_rotate_as_complex_numbers(oracle_lib):
    """Rotate-half RoPE read as complex multiplication:
    (x_i + i x_{i+64}) * (c_i + i s_i) = y_i + i y_{i+64}."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal(128)
    ang = rng.uniform(-5, 5, 64)
    y = oracle.rope_rotate(x, np.cos(ang), np.sin(ang))
    for i in range(64):
        z = complex(x[i], x[i + 64]) * complex(math.cos(ang[i]), math.sin(ang[i]))
        assert abs(z.real - y[i]) < 1e-13 and abs(z.imag - y[i + 64]) < 1e-13


def test_rope_table_frequencies_closed_form(oracle_lib):
    """With theta = 1e6 and head dim 128 the pair frequencies form a geometric
    sequence from 1 (pair 0) to 1e6^-0.5 = 1e-3 (pair 32).  Read the angles back
    from the fp32 table at position 1 and check them against that closed form."""
    c, s = oracle.rope_table(4, 128, 1e6)
    ang = np.arctan2(s[1].astype(np.float64), c[1].astype(np.float64))
    expect = np.array([1e-3 ** (i / 32.0) for i in range(64)])
    assert abs(ang[0] - 1.0) < 1e-6
    assert abs(ang[32] - 1e-3) < 1e-9
    np.testing.assert_allclose(ang, expect, rtol=2e-6, atol=1e-12)
    # position 0 is the identity: cos = 1, sin = 0 exactly
    assert np.all(c[0] == 1.0) and np.all(s[0] == 0.0)
    # fp32 rounding of the true cos/sin (one rounding, so within half an fp32 ulp)
    p = 3
    true_c = np.cos(p * expect)
    assert np.all(np.abs(c[p] - true_c) <= np.spacing(np.abs(c[p]).astype(np.float32)).astype(np.float64))


def test_rope_relative_position(oracle_lib):
    """<R_p q, R_r k> depends only on p - r (fp32 table, so to 1e-5)."""
    T = 300
    c, s = oracle.rope_table(T, 128, 1e6)
    rng = np.random.default_rng(3)
    q = rng.standard_normal(128)
    k = rng.standard_normal(128)

    def rot(x, p):
        return oracle.rope_rotate(x, c[p].astype(np.float64), s[p].astype(np.float64))

    for p, r, dlt in [(10, 3, 100), (0, 0, 250), (57, 200, 41), (5, 9, 7)]:
        a = float(np.dot(rot(q, p), rot(k, r)))
        b = float(np.dot(rot(q, p + dlt), rot(k, r + dlt)))
        assert abs(a - b) < 1e-4 * np.linalg.norm(q) * np.linalg.norm(k), (p, r, dlt, a, b)


def test_append_rope_position0_identity_and_bit_copies(oracle_lib):
    """At position 0 the rotation is the identity (bit-exact after rounding);
    V rows are copied bit for bit; rows outside [pos0, pos0+n_new) keep their
    bits; padded rows t >= n_new are not written."""
    B, S, T = 2, 3, 8
    q = rand_bits((B, S, 16, 128), 10)
    kn = rand_bits((B, S, 2, 128), 11)
    vn = rand_bits((B, S, 2, 128), 12)
    ck = rand_bits((B, T, 2, 128), 13)
    cv = rand_bits((B, T, 2, 128), 14)
    pos0 = np.array([0, 4], np.int32)
    n_new = np.array([3, 2], np.int32)
    q2, ck2, cv2, skipped = oracle.append_rope(q, kn, vn, ck, cv, pos0, n_new)
    assert skipped == 0
    assert np.array_equal(q2[0, 0], q[0, 0]) and np.array_equal(ck2[0, 0], kn[0, 0])
    for b in range(B):
        for t in range(n_new[b]):
            assert np.array_equal(cv2[b, pos0[b] + t], vn[b, t])
        written = set(range(pos0[b], pos0[b] + n_new[b]))
        for j in range(T):
            if j not in written:
                assert np.array_equal(ck2[b, j], ck[b, j]) and np.array_equal(cv2[b, j], cv[b, j])
    assert np.array_equal(q2[1, 2], q[1, 2])  # t = 2 >= n_new[1]: untouched


def test_append_rope_unit_vector_gives_table_entries(oracle_lib):
    """x = e_i (1 at pair index i) rotates to (cos, sin) of that pair's angle:
    out[i] = bf16(c_i), out[i+64] = bf16(s_i) -- the sign convention of the
    rotation (positive angle turns x_i towards x_{i+64})."""
    T = 100
    c, s = oracle.rope_table(T, 128, 1e6)
    for p, i in [(1, 0), (37, 5), (99, 63), (50, 32)]:
        q = np.zeros((1, 1, 16, 128), np.uint16)
        q[0, 0, 0, i] = 0x3F80  # 1.0
        kn = np.zeros((1, 1, 2, 128), np.uint16)
        vn = np.zeros((1, 1, 2, 128), np.uint16)
        ck = np.zeros((1, T, 2, 128), np.uint16)
        q2, _, _, _ = oracle.append_rope(q, kn, vn, ck, ck.copy(), np.array([p], np.int32),
                                         np.array([1], np.int32))
        got_c = oracle.bf16_array_to_f64(q2[0, 0, 0, i:i + 1])[0]
        got_s = oracle.bf16_array_to_f64(q2[0, 0, 0, i + 64:i + 65])[0]
        assert got_c == float(torch.tensor(float(c[p, i])).to(torch.bfloat16))
        assert got_s == float(torch.tensor(float(s[p, i])).to(torch.bfloat16))


def test_append_rope_skips_rows_past_T(oracle_lib):
    q = rand_bits((1, 3, 16, 128), 20)
    kn = rand_bits((1, 3, 2, 128), 21)
    ck = rand_bits((1, 8, 2, 128), 22)
    q2, ck2, _, skipped = oracle.append_rope(q, kn, kn, ck, ck, np.array([6], np.int32),
                                             np.array([3], np.int32))
    assert skipped == 1
    assert np.array_equal(q2[0, 2], q[0, 2])


# ------------------------------------------------------------- attention ----

def brute_attention_py(q, k, v, vis, scale):
    """Independent pure-Python softmax attention (lists, math.exp with the
    largest score subtracted), one query row over rows j < vis."""
    qf = [float(x) for x in q]
    scores = []
    for j in range(vis):
        scores.append(scale * sum(a * float(b) for a, b in zip(qf, k[j])))
    mx = max(scores)
    ws = [math.exp(x - mx) for x in scores]
    tot = math.fsum(ws)
    out = [math.fsum(w * float(v[j][d]) for j, w in enumerate(ws)) / tot for d in range(len(qf))]
    return out, mx + math.log(tot)


@pytest.mark.parametrize("Hq,Hkv,D,T", [(4, 2, 4, 8), (2, 1, 8, 5), (8, 2, 4, 7)])
def test_attention_brute_force_tiny(oracle_lib, Hq, Hkv, D, T):
    B, S = 2, 3
    q = rand_bits((B, S, Hq, D), 30)
    ck = rand_bits((B, T, Hkv, D), 31)
    cv = rand_bits((B, T, Hkv, D), 32)
    first_vis = np.array([2, T - S + 1], np.int32)
    n_rows = np.array([S, S], np.int32)
    scale = 1.0 / math.sqrt(D)
    o, lse = oracle.attention(q, ck, cv, first_vis, n_rows, scale)
    qf = oracle.bf16_array_to_f64(q)
    kf = oracle.bf16_array_to_f64(ck)
    vf = oracle.bf16_array_to_f64(cv)
    G = Hq // Hkv
    for b in range(B):
        for t in range(S):
            for h in range(Hq):
                g = h // G
                vis = first_vis[b] + t
                ref_o, ref_l = brute_attention_py(qf[b, t, h], kf[b, :, g], vf[b, :, g], vis, scale)
                np.testing.assert_allclose(o[b, t, h], ref_o, rtol=0, atol=1e-12)
                assert abs(lse[b, h, t] - ref_l) < 1e-12


def test_attention_matches_torch_sdpa_fp64(oracle_lib):
    """Cross-check against torch's SDPA in float64 on CPU, with each KV head
    repeated for its 8 query heads and an explicit causal/length mask."""
    B, S, T, Hq, Hkv, D = 2, 5, 40, 16, 2, 128
    q = rand_bits((B, S, Hq, D), 40)
    ck = rand_bits((B, T, Hkv, D), 41)
    cv = rand_bits((B, T, Hkv, D), 42)
    pos0 = np.array([7, 30], np.int32)
    n_new = np.array([5, 3], np.int32)
    scale = 1.0 / math.sqrt(D)
    o, lse = oracle.prefill(q, ck, cv, pos0, n_new, scale)
    qt = torch.from_numpy(oracle.bf16_array_to_f64(q)).permute(0, 2, 1, 3)        # B,Hq,S,D
    kt = torch.from_numpy(oracle.bf16_array_to_f64(ck)).permute(0, 2, 1, 3)       # B,Hkv,T,D
    vt = torch.from_numpy(oracle.bf16_array_to_f64(cv)).permute(0, 2, 1, 3)
    kt = kt.repeat_interleave(Hq // Hkv, dim=1)
    vt = vt.repeat_interleave(Hq // Hkv, dim=1)
    j = torch.arange(T).view(1, 1, 1, T)
    t = torch.arange(S).view(1, 1, S, 1)
    mask = j <= (torch.from_numpy(pos0).view(B, 1, 1, 1) + t)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    ref = ref.permute(0, 2, 1, 3).numpy()
    for b in range(B):
        np.testing.assert_allclose(o[b, :n_new[b]], ref[b, :n_new[b]], rtol=0, atol=1e-12)


def test_single_valid_position_returns_its_v_row(oracle_lib):
    B, T = 3, 16
    q = rand_bits((B, 1, 16, 128), 50)
    ck = rand_bits((B, T, 2, 128), 51)
    cv = rand_bits((B, T, 2, 128), 52)
    o, lse = oracle.decode(q, ck, cv, np.ones(B, np.int32), 1.0 / math.sqrt(128))
    vf = oracle.bf16_array_to_f64(cv)
    qf = oracle.bf16_array_to_f64(q)
    kf = oracle.bf16_array_to_f64(ck)
    for b in range(B):
        for h in range(16):
            assert np.array_equal(o[b, 0, h], vf[b, 0, h // 8])
            s0 = float(np.dot(qf[b, 0, h], kf[b, 0, h // 8])) / math.sqrt(128)
            assert abs(lse[b, h] - s0) < 1e-12


def test_equal_scores_give_mean_of_v(oracle_lib):
    """q = 0 makes every score 0: o is the mean of the visible V rows and
    lse = ln(n)."""
    B, T = 2, 33
    q = np.zeros((B, 1, 16, 128), np.uint16)
    ck = rand_bits((B, T, 2, 128), 60)
    cv = rand_bits((B, T, 2, 128), 61)
    kv = np.array([33, 17], np.int32)
    o, lse = oracle.decode(q, ck, cv, kv, 1.0 / math.sqrt(128))
    vf = oracle.bf16_array_to_f64(cv)
    for b in range(B):
        for h in range(16):
            np.testing.assert_allclose(o[b, 0, h], vf[b, :kv[b], h // 8].mean(axis=0), atol=1e-14)
            assert abs(lse[b, h] - math.log(kv[b])) < 1e-14
    # all K rows equal: same result for any q
    ck2 = np.repeat(ck[:, :1], T, axis=1)
    q2 = rand_bits((B, 1, 16, 128), 62)
    o2, _ = oracle.decode(q2, ck2, cv, kv, 1.0 / math.sqrt(128))
    for b in range(B):
        np.testing.assert_allclose(o2[b, 0, 0], vf[b, :kv[b], 0].mean(axis=0), atol=1e-13)


def test_gqa_equals_mha_with_repeated_kv(oracle_lib):
    B, S, T = 2, 4, 24
    q = rand_bits((B, S, 16, 128), 70)
    ck = rand_bits((B, T, 2, 128), 71)
    cv = rand_bits((B, T, 2, 128), 72)
    pos0 = np.array([3, 19], np.int32)
    n_new = np.array([4, 2], np.int32)
    sc = 1.0 / math.sqrt(128)
    o1, l1 = oracle.prefill(q, ck, cv, pos0, n_new, sc)
    ckr = np.repeat(ck, 8, axis=2)
    cvr = np.repeat(cv, 8, axis=2)
    o2, l2 = oracle.prefill(q, ckr, cvr, pos0, n_new, sc)
    np.testing.assert_array_equal(np.nan_to_num(o1, nan=7.0), np.nan_to_num(o2, nan=7.0))
    np.testing.assert_array_equal(np.nan_to_num(l1, nan=7.0), np.nan_to_num(l2, nan=7.0))


def test_garbage_past_valid_length_changes_nothing(oracle_lib):
    B, T = 4, 64
    kv = torch.tensor([1, 20, 63, 64], dtype=torch.int32)
    b1 = W.make_batch(80, B=B, S=1, T=T, pos0=kv, n_new=torch.zeros(B, dtype=torch.int32),
                      garbage="none")
    b2 = W.make_batch(80, B=B, S=1, T=T, pos0=kv, n_new=torch.zeros(B, dtype=torch.int32),
                      garbage="nan")
    sc = 1.0 / math.sqrt(128)
    q = bf16_bits(b1.q[0])
    o1, l1 = oracle.decode(q, bf16_bits(b1.cache_k[0]), bf16_bits(b1.cache_v[0]), kv.numpy(), sc)
    o2, l2 = oracle.decode(q, bf16_bits(b2.cache_k[0]), bf16_bits(b2.cache_v[0]), kv.numpy(), sc)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    assert np.isfinite(o2).all()


def test_static_masked_equals_length_aware(oracle_lib):
    """Attending over all T rows with rows past the valid length masked
    ("ARK-ASR-3B -- INT8 ONNX", section Shapes) gives the valid-prefix result
    when the garbage is finite."""
    B, T = 3, 48
    kv = torch.tensor([5, 30, 48], dtype=torch.int32)
    b = W.make_batch(90, B=B, S=1, T=T, pos0=kv, n_new=torch.zeros(B, dtype=torch.int32),
                     garbage="big")
    sc = 1.0 / math.sqrt(128)
    q, ck, cv = bf16_bits(b.q[0]), bf16_bits(b.cache_k[0]), bf16_bits(b.cache_v[0])
    o1, l1 = oracle.decode(q, ck, cv, kv.numpy(), sc)
    o2, l2 = oracle.decode(q, ck, cv, kv.numpy(), sc, static_mode=True)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_split_and_combine_equals_unsplit(oracle_lib):
    """Attention over [0, n) equals the log-sum-exp merge of attention over
    any partition of [0, n) into chunks (empty chunks included)."""
    T = 100
    qrow = rand_bits((128,), 100)
    k = rand_bits((T, 128), 101, scale=3.0)
    v = rand_bits((T, 128), 102)
    sc = 1.0 / math.sqrt(128)
    o_ref, l_ref = oracle.attend_one(qrow, k, v, 0, T, sc)
    for cuts in ([0, 64, 100], [0, 1, 2, 50, 99, 100], [0, 16, 16, 80, 100], [0, 100]):
        parts = [oracle.attend_one(qrow, k, v, a, b_, sc) for a, b_ in zip(cuts[:-1], cuts[1:])]
        o, l = oracle.combine(np.stack([p[0] for p in parts]), np.array([p[1] for p in parts]))
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        assert abs(l - l_ref) < 1e-12


def test_combine_closed_forms(oracle_lib):
    a = np.arange(8, dtype=np.float64)
    o, l = oracle.combine(np.stack([a, a + 2]), np.array([1.5, 1.5]))
    np.testing.assert_allclose(o, a + 1)
    assert abs(l - (1.5 + math.log(2))) < 1e-15
    o, l = oracle.combine(np.stack([a, np.full(8, np.nan)]), np.array([0.25, -np.inf]))
    np.testing.assert_array_equal(o, a)
    assert l == 0.25
    o, l = oracle.combine(np.stack([a, a]), np.array([-np.inf, -np.inf]))
    assert np.all(o == 0) and l == -np.inf


def test_prefill_row_equals_decode_at_that_length(oracle_lib):
    """Causal consistency: prefill row t of a request equals a decode at
    kv_len = pos0 + t + 1 over the same cache."""
    B, S, T = 2, 6, 32
    q = rand_bits((B, S, 16, 128), 110)
    ck = rand_bits((B, T, 2, 128), 111)
    cv = rand_bits((B, T, 2, 128), 112)
    pos0 = np.array([0, 20], np.int32)
    n_new = np.array([6, 4], np.int32)
    sc = 1.0 / math.sqrt(128)
    o, lse = oracle.prefill(q, ck, cv, pos0, n_new, sc)
    for b in range(B):
        for t in range(n_new[b]):
            od, ld = oracle.decode(q[b:b + 1, t:t + 1], ck[b:b + 1], cv[b:b + 1],
                                   np.array([pos0[b] + t + 1], np.int32), sc)
            np.testing.assert_array_equal(o[b, t], od[0, 0])
            assert lse[b, :, t].tolist() == ld[0].tolist()


def test_empty_visible_range(oracle_lib):
    q = rand_bits((1, 1, 16, 128), 120)
    ck = rand_bits((1, 8, 2, 128), 121)
    o, lse = oracle.decode(q, ck, ck, np.array([0], np.int32), 0.1)
    assert np.all(o == 0) and np.all(lse == -np.inf)


# -------------------------------------------------------- prompt lengths ----

def test_audio_slots_golden():
    rows = []
    with open(os.path.join(GOLDEN, "audio_slots.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([int(x) for x in line.split()])
    assert rows
    for samples, mel, slots in rows:
        assert W.audio_slots(samples) == slots
        assert mel == samples // 160
        assert max(W.audio_slots_from_mel(mel), 1) == slots
    assert W.sweep_prompt_len() == 50
    assert W.audio_slots(30 * 16000) + 12 == 387


# ----------------------------------------------------------- fp8 (e4m3) ----
# The 8-bit cache format is a reading of its own (the pages quantise weights
# only): OCP E4M3 codes, one fp32 scale per (layer, KV head), code =
# e4m3(fp32(x / scale)).  The pins tie the oracle's encoder and decoder to
# torch's float8_e4m3fn conversions and to the format's defining constants,
# and the fp8 attention to the bf16 attention pinned above.

def test_e4m3_decode_all_codes_matches_torch(oracle_lib):
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.isnan(ours).sum() == 2                       # S.1111.111 only: no infinities


def test_e4m3_defining_constants(oracle_lib):
    v = oracle.e4m3_to_f64(np.array([0x7E, 0x01, 0x08, 0x07, 0x38, 0x80], np.uint8))
    assert v[0] == 448.0                                   # largest finite: 1.75 * 2^8
    assert v[1] == 2.0 ** -9                               # smallest subnormal
    assert v[2] == 2.0 ** -6                               # smallest normal
    assert v[3] == 7 * 2.0 ** -9                           # largest subnormal
    assert v[4] == 1.0 and v[5] == 0.0 and np.signbit(v[5])
    pos = oracle.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)                        # codes 0..126 increase strictly


def test_e4m3_encode_roundtrip_ties_and_saturation(oracle_lib):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle.e4m3_to_f64(codes).astype(np.float32)
    assert np.array_equal(oracle.f32_to_e4m3(vals), codes)                 # every finite code round-trips
    pos = oracle.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)                   # exact in fp32
    got = oracle.f32_to_e4m3(mids).astype(int)
    lo = np.arange(0x7E)
    assert np.array_equal(got, np.where(lo % 2 == 0, lo, lo + 1))          # ties to the even code
    assert np.array_equal(oracle.f32_to_e4m3(np.nextafter(mids, np.float32(0))), lo)
    assert np.array_equal(oracle.f32_to_e4m3(np.nextafter(mids, np.float32(1e9))), lo + 1)
    sat = oracle.f32_to_e4m3(np.array([448.5, 463.9, 464.0, 1e30, np.inf, -np.inf, -1e9], np.float32))
    assert list(sat) == [0x7E] * 5 + [0xFE, 0xFE]
    assert oracle.f32_to_e4m3(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F


def test_e4m3_encode_matches_torch_in_range(oracle_lib):
    g = torch.Generator().manual_seed(31)
    x = torch.cat([torch.randn(4000, generator=g) * s for s in (0.003, 0.1, 1.0, 30.0)])
    x = torch.clamp(x, -448.0, 448.0).float()
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.f32_to_e4m3(x.numpy()), ref)


def _rn_binary(q, mant_bits: int, min_exp: int):
    """Exact round-to-nearest-even of the rational q onto a binary grid with
    mant_bits bits after the point and exponents >= min_exp (subnormals below
    2^min_exp); no overflow handling.  Plain exponent/ulp arithmetic, written
    from the IEEE definition, not a search."""
    from fractions import Fraction
    if q == 0:
        return Fraction(0)
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1                                   # now 2^e <= a < 2^(e+1)
    e = max(e, min_exp)
    ulp = Fraction(2) ** (e - mant_bits)
    m = a / ulp
    lo = m.numerator // m.denominator
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    v = lo * ulp
    return v if q > 0 else -v


def _e4m3_reference(x: float, scale: float) -> int:
    """e4m3(fp32(x / scale)) by exact rational arithmetic: the fp64 quotient
    (Python's correctly rounded float division), rounded to fp32, rounded to
    e4m3 (nearest even, saturating at +-448), encoded from its exponent and
    mantissa."""
    from fractions import Fraction
    q64 = x / float(np.float32(scale))
    y = _rn_binary(Fraction(q64), 23, -126)              # fp32 (the quotients here stay in range)
    sign = 0x80 if (y < 0 or (y == 0 and math.copysign(1.0, q64) < 0)) else 0
    a = abs(y)
    if a >= 448:
        return sign | 0x7E
    v = _rn_binary(a, 3, -6)
    if v == 0:
        return sign
    if v >= 448:
        return sign | 0x7E
    e = v.numerator.bit_length() - v.denominator.bit_length()
    if Fraction(2) ** e > v:
        e -= 1
    if e < -6:                                           # subnormal: multiples of 2^-9
        return sign | int(v / Fraction(2) ** -9)
    mant = int((v / Fraction(2) ** e - 1) * 8)
    return sign | ((e + 7) << 3) | mant


def test_quantize_e4m3_exact_including_double_rounding(oracle_lib):
    """ora_quantize_e4m3 equals the exact e4m3(fp32(x / scale)) everywhere
    tested, including quotients that sit within half an fp32 step of an e4m3
    midpoint: there the fp32 rounding lands ON the midpoint and the tie goes
    to the even code, while rounding the fp64 quotient straight to e4m3 would
    go the other way -- a version that skipped the fp32 step fails here."""
    from fractions import Fraction
    pos = oracle.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))
    xs, scales, flips = [], [], 0
    for c in range(0x7E):
        mid = (pos[c] + pos[c + 1]) / 2                  # exact in fp64 and fp32
        for sc in (1.0, 0.5, 4.0):
            for sgn in (1.0, -1.0):
                for d in (2.0 ** -30, -(2.0 ** -30)):
                    x = sgn * (mid + d * max(mid, 2.0 ** -9)) * sc    # power-of-two scale: exact quotient
                    xs.append(x)
                    scales.append(sc)
                    # the exact quotient is off the midpoint, its fp32 rounding is the midpoint
                    direct = _rn_binary(Fraction(x / sc), 3, -6)
                    via32 = _rn_binary(_rn_binary(Fraction(x / sc), 23, -126), 3, -6)
                    flips += int(direct != via32)
    assert flips > 100                                   # the cases really discriminate
    g = np.random.default_rng(17)
    for sc in (0.0371, 0.1, 0.2, 1.7, 3.0e-3):
        for v in np.concatenate([g.standard_normal(300) * m for m in (1e-4, 0.01, 1.0, 30.0)]):
            xs.append(float(v))
            scales.append(sc)
    xs += [500.0, -1e6, 0.0, -0.0, 2.0 ** -12]
    scales += [1.0, 1.0, 1.0, 1.0, 1.0]
    for x, sc in zip(xs, scales):
        got = int(oracle.quantize_e4m3(np.array([x]), sc)[0])
        assert got == _e4m3_reference(x, sc), (x, sc, got, _e4m3_reference(x, sc))


def test_append_fp8_within_half_code_of_fp64_rotation(oracle_lib):
    """Dequantised fp8 keys sit within half an e4m3 step of the fp64 rotation
    (then divided by the scale); values reproduce exactly when they are
    representable; rows outside the written range keep their codes."""
    B, S, T = 2, 3, 16
    q = rand_bits((B, S, 16, 128), 40)
    kn = rand_bits((B, S, 2, 128), 41)
    g = torch.Generator().manual_seed(42)
    rep = oracle.e4m3_to_f64(torch.randint(0x18, 0x58, (B, S, 2, 128), generator=g).to(torch.uint8).numpy())
    vscale = np.array([0.25, 2.0], np.float32)
    vn = bf16_bits(torch.from_numpy(rep * vscale[None, None, :, None]))   # exact: power-of-two scales
    ck = torch.randint(0, 0x70, (B, T, 2, 128), generator=g).to(torch.uint8).numpy()
    cv = torch.randint(0, 0x70, (B, T, 2, 128), generator=g).to(torch.uint8).numpy()
    kscale = np.array([0.05, 0.013], np.float32)
    pos0 = np.array([2, 9], np.int32)
    n_new = np.array([3, 2], np.int32)
    q2, ck2, cv2, skipped = oracle.append_rope_fp8(q, kn, vn, ck, cv, kscale, vscale, pos0, n_new)
    assert skipped == 0
    q_ref, _, _, _ = oracle.append_rope(q, kn, vn, np.zeros((B, T, 2, 128), np.uint16),
                                        np.zeros((B, T, 2, 128), np.uint16), pos0, n_new)
    assert np.array_equal(q2, q_ref)                       # q is rotated exactly as on the bf16 path
    cos_t, sin_t = oracle.rope_table(T)
    for b in range(B):
        for t in range(n_new[b]):
            p = pos0[b] + t
            for h in range(2):
                y = oracle.rope_rotate(oracle.bf16_array_to_f64(kn[b, t, h]), cos_t[p].astype(np.float64),
                                       sin_t[p].astype(np.float64)) / kscale[h]
                d = oracle.e4m3_to_f64(ck2[b, p, h])
                step = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** -6))) - 3), 2.0 ** -9)
                assert np.all(np.abs(d - np.clip(y, -448, 448)) <= step / 2 + 1e-12)
                assert np.array_equal(oracle.e4m3_to_f64(cv2[b, p, h]), rep[b, t, h])
        written = set(range(pos0[b], pos0[b] + n_new[b]))
        for j in range(T):
            if j not in written:
                assert np.array_equal(ck2[b, j], ck[b, j]) and np.array_equal(cv2[b, j], cv[b, j])


def test_fp8_attention_equals_bf16_attention_of_dequantised_cache(oracle_lib):
    """With power-of-two scales every dequantised code is a bf16 value, so the
    fp8 attention must give exactly the bf16 attention of those values (length
    aware and masked static); NaN codes past the valid length change nothing."""
    B, T = 3, 40
    g = torch.Generator().manual_seed(50)
    codes_k = torch.randint(0x10, 0x60, (B, T, 2, 128), generator=g).to(torch.uint8)
    codes_v = torch.randint(0x10, 0x60, (B, T, 2, 128), generator=g).to(torch.uint8)
    sign_k = torch.randint(0, 2, codes_k.shape, generator=g).to(torch.uint8) << 7
    codes_k = (codes_k | sign_k).numpy()
    codes_v = codes_v.numpy()
    ks = np.array([0.125, 0.5], np.float32)
    vs = np.array([0.25, 1.0], np.float32)
    q = rand_bits((B, 1, 16, 128), 51)
    kv = np.array([1, 17, 40], np.int32)
    kd = oracle.e4m3_to_f64(codes_k) * ks[None, None, :, None]
    vd = oracle.e4m3_to_f64(codes_v) * vs[None, None, :, None]
    kb = bf16_bits(torch.from_numpy(kd))
    vb = bf16_bits(torch.from_numpy(vd))
    assert np.array_equal(oracle.bf16_array_to_f64(kb), kd)   # exact in bf16
    for static in (False, True):
        o8, l8 = oracle.decode_fp8(q, codes_k, codes_v, ks, vs, kv, 0.0884, static)
        o16, l16 = oracle.decode(q, kb, vb, kv, 0.0884, static)
        assert np.array_equal(o8, o16) and np.array_equal(l8, l16)
    garbage_k = codes_k.copy()
    garbage_v = codes_v.copy()
    for b in range(B):
        garbage_k[b, kv[b]:] = 0x7F
        garbage_v[b, kv[b]:] = 0xFF
    o8g, l8g = oracle.decode_fp8(q, garbage_k, garbage_v, ks, vs, kv, 0.0884)
    o8, l8 = oracle.decode_fp8(q, codes_k, codes_v, ks, vs, kv, 0.0884)
    assert np.array_equal(o8g, o8) and np.array_equal(l8g, l8)


# ------------------------------------------------------ encoder attention ----

def test_encoder_attention_matches_torch_sdpa_fp64(oracle_lib):
    """Bidirectional multi-head attention per clip against torch's SDPA in
    fp64 (no mask inside the clip's length), and against a pure-Python loop on
    one row."""
    B, S, H, D = 3, 20, 4, 64
    q = rand_bits((B, S, H, D), 60)
    k = rand_bits((B, S, H, D), 61)
    v = rand_bits((B, S, H, D), 62)
    length = np.array([20, 7, 1], np.int32)
    scale = 1 / 8.0
    o, lse = oracle.attention_bidir(q, k, v, length, scale)
    qd, kd, vd = (torch.from_numpy(oracle.bf16_array_to_f64(x)) for x in (q, k, v))
    for b in range(B):
        n = int(length[b])
        ref = torch.nn.functional.scaled_dot_product_attention(
            qd[b, :n].transpose(0, 1), kd[b, :n].transpose(0, 1), vd[b, :n].transpose(0, 1), scale=scale)
        assert np.allclose(o[b, :n], ref.transpose(0, 1).numpy(), rtol=1e-12, atol=1e-12)
        assert np.all(np.isnan(o[b, n:])) and np.all(np.isnan(lse[b, :, n:]))
    b, i, h = 1, 3, 2
    n = int(length[b])
    s = [scale * sum(float(qd[b, i, h, d]) * float(kd[b, j, h, d]) for d in range(D)) for j in range(n)]
    m = max(s)
    w = [math.exp(x - m) for x in s]
    l = sum(w)
    assert abs(lse[b, h, i] - (m + math.log(l))) < 1e-12
    for d in (0, 31, 63):
        assert abs(o[b, i, h, d] - sum(w[j] * float(vd[b, j, h, d]) for j in range(n)) / l) < 1e-12


def test_encoder_attention_ignores_frames_past_length(oracle_lib):
    B, S, H, D = 2, 16, 2, 64
    q = rand_bits((B, S, H, D), 63)
    k = rand_bits((B, S, H, D), 64)
    v = rand_bits((B, S, H, D), 65)
    length = np.array([9, 16], np.int32)
    o, lse = oracle.attention_bidir(q, k, v, length, 0.125)
    k2, v2 = k.copy(), v.copy()
    k2[0, 9:] = 0x7FC0           # NaN
    v2[0, 9:] = 0x7F80           # +inf
    o2, lse2 = oracle.attention_bidir(q, k2, v2, length, 0.125)
    assert np.array_equal(o[0, :9], o2[0, :9]) and np.array_equal(lse[0, :, :9], lse2[0, :, :9])


# ------------------------------------------------------ Q/K/V projection ----

def _bf16_value(bits):
    """Exact value of a bf16 bit pattern as a Fraction (no float arithmetic)."""
    from fractions import Fraction
    b = int(bits)
    sign = -1 if b >> 15 else 1
    e = (b >> 7) & 0xFF
    m = b & 0x7F
    assert e != 0xFF
    if e == 0:
        return sign * Fraction(m, 1 << 7) * Fraction(1, 1 << 126)
    return sign * (1 + Fraction(m, 1 << 7)) * (Fraction(2) ** (e - 127))


def _bf16_round_exact(v):
    """Nearest bf16 to the rational v, ties to even mantissa, by exact
    comparison among the candidates around float(v)."""
    import struct
    f = float(v)
    u = struct.unpack("<I", struct.pack("<f", f))[0] >> 16 if f == f else 0x7FC0
    cands = set()
    for d in range(-3, 4):
        c = (u + d) & 0xFFFF
        if ((c >> 7) & 0xFF) != 0xFF:
            cands.add(c)
    best = min(cands, key=lambda c: (abs(_bf16_value(c) - v), c & 1))
    return best


def test_qkv_proj_matches_exact_rational_sum():
    """Every output of a small Linear equals the bf16 nearest to the exact
    rational sum + bias (brute force in Fractions, independent rounding)."""
    rng = np.random.default_rng(5)
    M, K, N = 3, 37, 5
    x = oracle.f64_to_bf16(rng.standard_normal((M, K)))
    w = oracle.f64_to_bf16(rng.standard_normal((N, K)) * 0.3)
    b = oracle.f64_to_bf16(rng.standard_normal(N))
    got = oracle.qkv_proj(x, w, b)
    got_nb = oracle.qkv_proj(x, w, None)
    for m in range(M):
        for n in range(N):
            exact = sum(_bf16_value(x[m, k]) * _bf16_value(w[n, k]) for k in range(K))
            assert got_nb[m, n] == _bf16_round_exact(exact), (m, n)
            assert got[m, n] == _bf16_round_exact(exact + _bf16_value(b[n])), (m, n)


def test_qkv_proj_selection_matrix_copies_inputs():
    """W[n, k] = [k == perm[n]] selects input columns: out[m, n] is x[m, perm[n]]
    bit for bit (fixes the operand orientation and the indexing)."""
    rng = np.random.default_rng(6)
    M, K = 4, 64
    x = oracle.f64_to_bf16(rng.standard_normal((M, K)))
    perm = rng.permutation(K)[:40]
    w = np.zeros((40, K), dtype=np.uint16)
    w[np.arange(40), perm] = 0x3F80           # 1.0
    assert np.array_equal(oracle.qkv_proj(x, w), x[:, perm])


def test_qkv_rope_append_splits_columns_q_k_v():
    """With W the identity the projection is the input itself, so the fused
    step equals RoPE + delta write of the input's three column blocks
    (q: heads 0..Hq-1, then k, then v)."""
    rng = np.random.default_rng(7)
    Hq, Hkv, D, B, S, T = 2, 1, 128, 2, 3, 16
    N = (Hq + 2 * Hkv) * D
    x = oracle.f64_to_bf16(rng.standard_normal((B, S, N)))
    w = np.zeros((N, N), dtype=np.uint16)
    w[np.arange(N), np.arange(N)] = 0x3F80
    ck = oracle.f64_to_bf16(rng.standard_normal((B, T, Hkv, D)))
    cv = oracle.f64_to_bf16(rng.standard_normal((B, T, Hkv, D)))
    pos0, n_new = np.array([0, 9], np.int32), np.array([3, 2], np.int32)
    got = oracle.qkv_rope_append(x, w, None, ck, cv, pos0, n_new, Hq, Hkv, D)
    want = oracle.append_rope(x[:, :, :Hq * D].reshape(B, S, Hq, D),
                              x[:, :, Hq * D:(Hq + Hkv) * D].reshape(B, S, Hkv, D),
                              x[:, :, (Hq + Hkv) * D:].reshape(B, S, Hkv, D), ck, cv, pos0, n_new)
    for a, b_ in zip(got[:3], want[:3]):
        assert np.array_equal(a, b_)
