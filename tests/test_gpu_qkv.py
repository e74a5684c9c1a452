"""The Q/K/V projection step in front of the attention on the tcgen05 tensor
cores against the fp64 oracle ("ARK-ASR-3B -- INT8 ONNX" model card: Q/K/V
projections of the Qwen2 decoder, hidden 2048, 16 query and 2 KV heads of 128;
section Shapes: new key/value rows land in the cache at cache_position).

The GPU accumulates in fp32, the oracle in double, so a projection value may
round to the neighbouring bf16: per element the test allows one bf16 ulp of
the result plus the fp32 summation bound K * 2^-24 * sum_k |x_k W_nk| (and,
after the rotation, the same for each of the two rotated inputs).  The fused
RoPE + delta write is checked bit for bit against the projection followed by
the append kernel, and rows not written must keep their bits."""
import numpy as np
import pytest
import torch

import oracle
from gqa_attention_static_b200 import ops
from gqa_attention_static_b200 import workloads as W
from tests.helpers import bits

pytestmark = pytest.mark.gpu

HQ, HKV, D = 16, 2, 128
U16_NAN = 0x7FC1
# (what, values, bit-identical, one bf16 step off, more, largest step distance) per comparison,
# printed after the run
ULP_COUNTS = []


def f32_of(b):
    return oracle.bf16_array_to_f64(b)


def abs_dot(x_bits, w_bits, bias_bits):
    """sum_k |x_mk W_nk| (+ |bias_n|) in double: the scale of the fp32 summation error."""
    x = np.abs(f32_of(x_bits))
    w = np.abs(f32_of(w_bits))
    s = x @ w.T
    if bias_bits is not None:
        s = s + np.abs(f32_of(bias_bits))[None, :]
    return s


def ulp_distance(a_bits, b_bits):
    """Distance in bf16 steps between two arrays of bf16 bit patterns (the
    patterns mapped to a monotone integer line, so -0 and +0 coincide)."""
    def line(x):
        x = x.astype(np.int64)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(line(a_bits) - line(b_bits))


def check_close_bf16(got_bits, ref_bits, err_bound, what):
    got = f32_of(got_bits)
    ref = f32_of(ref_bits)
    tol = 2.0 ** -7 * np.abs(ref) + err_bound
    bad = ~(np.abs(got - ref) <= tol)
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside; e.g. {got[bad][:3]} vs {ref[bad][:3]}"
    d = ulp_distance(got_bits, ref_bits)
    ULP_COUNTS.append((what, got_bits.size, int(np.sum(d == 0)), int(np.sum(d == 1)), int(np.sum(d > 1)),
                       int(d.max()) if d.size else 0))
    exact = float(np.mean(got_bits == ref_bits))
    assert exact > 0.98, f"{what}: only {exact:.4f} bit-identical"


@pytest.mark.parametrize("M,bias", [(200, True), (128, False), (37, True), (64, False), (1, True)])
def test_qkv_proj_against_oracle(oracle_lib, M, bias):
    """Ragged M (several 128-row tiles and a tail; and up to 64 rows, the
    narrow form with the token rows on the MMA's N), K = 2048, N = 2560."""
    w, b = W.make_qkv_weights(11 + M, bias=bias)
    x = W.make_hidden(12 + M, 1, M)[0]
    out = torch.full((M, w.shape[0]), 0, dtype=torch.bfloat16, device="cuda")
    ops.ark_attn_qkv_proj(x.cuda(), w.cuda(), None if b is None else b.cuda(), out)
    torch.cuda.synchronize()
    bb = None if b is None else bits(b)
    ref = oracle.qkv_proj(bits(x), bits(w), bb)
    bound = 2048 * 2.0 ** -24 * abs_dot(bits(x), bits(w), bb)
    check_close_bf16(bits(out), ref, bound, "projection")


@pytest.mark.parametrize("M,K", [(32, 4096), (48, 1024), (20, 512)])
def test_qkv_proj_narrow_other_hidden_sizes(oracle_lib, M, K):
    """The narrow form (up to 64 token rows) at other hidden sizes: K = 4096
    gives each cluster rank more K chunks than its ring has stages (the ring is
    reused), K = 1024 and 512 the 4-stage form with one and two chunks a rank."""
    w, b = W.make_qkv_weights(500 + K, K=K)
    x = W.make_hidden(501 + K, 1, M, K=K)[0]
    out = torch.full((M, w.shape[0]), 0, dtype=torch.bfloat16, device="cuda")
    ops.ark_attn_qkv_proj(x.cuda(), w.cuda(), b.cuda(), out)
    torch.cuda.synchronize()
    ref = oracle.qkv_proj(bits(x), bits(w), bits(b))
    bound = K * 2.0 ** -24 * abs_dot(bits(x), bits(w), bits(b))
    check_close_bf16(bits(out), ref, bound, f"projection M={M} K={K}")


def run_fused(x, w, b, pos0, n_new, T, ck0, cv0):
    dev = "cuda"
    B, S, _ = x.shape
    q = torch.empty((B, S, HQ, D), dtype=torch.bfloat16, device=dev).view(torch.int16).fill_(U16_NAN).view(torch.bfloat16)
    ck, cv = ck0.to(dev).clone(), cv0.to(dev).clone()
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.ark_attn_qkv_rope_append(x.to(dev), w.to(dev), None if b is None else b.to(dev), pos0.to(dev),
                                 n_new.to(dev), ops.rope_table(T), q, ck, cv, st)
    torch.cuda.synchronize()
    return q, ck, cv, int(st.item())


def make_case(seed, B, S, T, pos0, n_new, bias=True):
    w, b = W.make_qkv_weights(seed, bias=bias)
    x = W.make_hidden(seed + 1, B, S)
    g = torch.Generator().manual_seed(seed + 2)
    ck = torch.randn((B, T, HKV, D), generator=g).to(torch.bfloat16)
    cv = torch.randn((B, T, HKV, D), generator=g).to(torch.bfloat16)
    return x, w, b, torch.tensor(pos0, dtype=torch.int32), torch.tensor(n_new, dtype=torch.int32), ck, cv


def check_fused_against_oracle(x, w, b, pos0, n_new, ck0, cv0, q, ck, cv, rows=None):
    """Compare the live rows (all, or the (b, t) pairs in `rows`) with the oracle
    on exactly those rows; rows of the caches not written keep their bits."""
    B, S, K = x.shape
    T = ck0.shape[1]
    bb = None if b is None else bits(b)
    live = [(i, t) for i in range(B) for t in range(int(n_new[i]))] if rows is None else rows
    xs = np.stack([bits(x)[i, t] for i, t in live])[:, None, :]            # [R, 1, K]
    p0 = np.array([int(pos0[i]) + t for i, t in live], np.int32)
    if rows is None:
        # every live row: the oracle on the whole batch, its results gathered per row
        qa, cka, cva, skipped = oracle.qkv_rope_append(bits(x), bits(w), bb, bits(ck0), bits(cv0),
                                                       np.asarray(pos0, np.int32), np.asarray(n_new, np.int32),
                                                       HQ, HKV, D)
        q_ref = np.stack([qa[i, t] for i, t in live])[:, None]
        rk = np.stack([cka[i, int(pos0[i]) + t] for i, t in live])
        rv = np.stack([cva[i, int(pos0[i]) + t] for i, t in live])
    else:
        ones = np.ones(len(live), np.int32)
        ck_rows = np.stack([bits(ck0)[i] for i, _ in live])
        cv_rows = np.stack([bits(cv0)[i] for i, _ in live])
        q_ref, ck_ref, cv_ref, skipped = oracle.qkv_rope_append(xs, bits(w), bb, ck_rows, cv_rows, p0, ones, HQ,
                                                                HKV, D)
        rk = np.stack([ck_ref[r, p0[r]] for r in range(len(live))])
        rv = np.stack([cv_ref[r, p0[r]] for r in range(len(live))])
    assert skipped == 0
    # error scale of each projection value, then of each rotated value (|c|, |s| <= 1)
    s = abs_dot(xs[:, 0], bits(w), bb) * (2048 * 2.0 ** -24)                # [R, N]
    pq = s[:, :HQ * D].reshape(-1, HQ, D)
    pk = s[:, HQ * D:(HQ + HKV) * D].reshape(-1, HKV, D)
    pv = s[:, (HQ + HKV) * D:].reshape(-1, HKV, D)
    rot = lambda e: np.concatenate([e[..., :64] + e[..., 64:], e[..., :64] + e[..., 64:]], axis=-1)
    proj = oracle.qkv_proj(xs[:, 0], bits(w), bb)
    pref = f32_of(proj)
    # one ulp of a rotation input moves the output by at most that ulp
    ulp_in = 2.0 ** -7 * np.abs(pref)
    uq = ulp_in[:, :HQ * D].reshape(-1, HQ, D)
    uk = ulp_in[:, HQ * D:(HQ + HKV) * D].reshape(-1, HKV, D)
    qb, kb, vb = bits(q), bits(ck), bits(cv)
    gq = np.stack([qb[i, t] for i, t in live])
    gk = np.stack([kb[i, int(pos0[i]) + t] for i, t in live])
    gv = np.stack([vb[i, int(pos0[i]) + t] for i, t in live])
    rq = q_ref[:, 0]
    check_close_bf16(gq, rq, rot(pq + uq), "q")
    check_close_bf16(gk, rk, rot(pk + uk), "cache_k")
    check_close_bf16(gv, rv, pv, "cache_v")


def check_untouched(pos0, n_new, ck0, cv0, ck, cv):
    B, T = ck0.shape[0], ck0.shape[1]
    for i in range(B):
        keep = np.ones(T, bool)
        keep[int(pos0[i]):int(pos0[i]) + int(n_new[i])] = False
        assert np.array_equal(bits(ck)[i][keep], bits(ck0)[i][keep])
        assert np.array_equal(bits(cv)[i][keep], bits(cv0)[i][keep])


@pytest.mark.parametrize("B,S,T,pos0,n_new", [
    (3, 40, 256, [0, 30, 200], [40, 17, 1]),     # prompt rows, ragged
    (32, 1, 512, list(range(40, 520, 15)), [1] * 32),  # a decode step of 32 requests
    (2, 130, 512, [0, 380], [130, 2]),           # two 128-row tiles and a tail
])
def test_qkv_rope_append_against_oracle(oracle_lib, B, S, T, pos0, n_new):
    x, w, b, p0, nn, ck0, cv0 = make_case(300 + B + S, B, S, T, pos0, n_new)
    q, ck, cv, st = run_fused(x, w, b, p0, nn, T, ck0, cv0)
    assert st == 0
    check_fused_against_oracle(x, w, b, p0, nn, ck0, cv0, q, ck, cv)
    check_untouched(p0, nn, ck0, cv0, ck, cv)
    # padded q rows are not written
    qb = bits(q)
    for i in range(B):
        assert np.all(qb[i, int(nn[i]):] == U16_NAN)


@pytest.mark.parametrize("B,S,pos0,n_new", [
    (4, 70, [0, 100, 441, 7], [70, 33, 70, 1]),   # 128-row tiles
    (32, 1, list(range(3, 480, 15)), [1] * 32),   # a decode step: the narrow form
    (5, 3, [0, 9, 500, 77, 1], [3, 1, 2, 0, 3]),  # 15 token rows, padded ones among them
])
def test_qkv_fused_equals_projection_then_append(oracle_lib, B, S, pos0, n_new):
    """Bit for bit: the fused epilogue == ark_attn_qkv_proj + ark_attn_append_rope."""
    T = 512
    x, w, b, p0, nn, ck0, cv0 = make_case(77 + B, B, S, T, pos0, n_new)
    q, ck, cv, st = run_fused(x, w, b, p0, nn, T, ck0, cv0)
    assert st == 0
    dev = "cuda"
    proj = torch.empty((B * S, w.shape[0]), dtype=torch.bfloat16, device=dev)
    ops.ark_attn_qkv_proj(x.to(dev).view(B * S, -1), w.to(dev), b.to(dev), proj)
    proj = proj.view(B, S, -1)
    q2 = proj[:, :, :HQ * D].contiguous().view(B, S, HQ, D)
    k2 = proj[:, :, HQ * D:(HQ + HKV) * D].contiguous().view(B, S, HKV, D)
    v2 = proj[:, :, (HQ + HKV) * D:].contiguous().view(B, S, HKV, D)
    ck2, cv2 = ck0.to(dev).clone(), cv0.to(dev).clone()
    st2 = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.ark_attn_append_rope(q2, k2, v2, ck2, cv2, p0.to(dev), nn.to(dev), ops.rope_table(T), st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    assert torch.equal(ck, ck2) and torch.equal(cv, cv2)
    for i in range(B):
        n = int(nn[i])
        assert torch.equal(q[i, :n], q2[i, :n])


def test_qkv_rope_append_prefill_full_size(oracle_lib):
    """The coalesced prefill batch at full size (16 prompts of 20..387 rows,
    T = 512): every live row (3293 of them) compared with the oracle."""
    pf = W.cfg_prefill(layers=1)
    B, S, T = pf.B, pf.n_new.max().item(), pf.T
    x, w, b, _, _, ck0, cv0 = make_case(91, B, S, T, [0] * B, [1] * B)
    p0, nn = pf.pos0, pf.n_new
    q, ck, cv, st = run_fused(x, w, b, p0, nn, T, ck0, cv0)
    assert st == 0
    check_fused_against_oracle(x, w, b, p0, nn, ck0, cv0, q, ck, cv)
    check_untouched(p0, nn, ck0, cv0, ck, cv)


def test_qkv_bad_position_reported(oracle_lib):
    """A row whose position falls past T is skipped and flagged."""
    x, w, b, p0, nn, ck0, cv0 = make_case(5, 2, 4, 16, [0, 14], [4, 4])
    q, ck, cv, st = run_fused(x, w, b, p0, nn, 16, ck0, cv0)
    assert st & ops.ARK_DEV_BAD_POS
    # request 0 fully written, request 1 rows 0..1 (positions 14, 15) written, 2..3 skipped
    check_fused_against_oracle(x, w, b, p0, nn, ck0, cv0, q, ck, cv,
                               rows=[(0, 0), (0, 1), (0, 2), (0, 3), (1, 0), (1, 1)])
