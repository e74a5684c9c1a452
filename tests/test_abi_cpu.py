"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad host-visible arguments before it touches
CUDA (so these calls are safe on a machine with no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from gqa_attention_static_b200 import build as B
from gqa_attention_static_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "arkattn.h")

FAKE = 0x10000        # an aligned non-null address; never dereferenced by these checks
FAKE_MIS = 0x10002    # misaligned


@pytest.fixture(scope="module")
def lib():
    B.build()
    return ops.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(ark_attn_\w+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(ops.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", ops.LIB_PATH], text=True)
    exported = set(re.findall(r"\bT (ark_attn_\w+)", out))
    missing = [s for s in declared_symbols() if s not in exported]
    assert not missing, missing
    for s in declared_symbols():
        assert hasattr(lib, s)


def test_status_strings(lib):
    for code in range(6):
        assert ops.status_string(code)
    assert ops.status_string(0) == "ok"
    assert ops.status_string(99) == "unknown status"


def test_rope_table_arg_checks(lib):
    assert lib.ark_attn_rope_table_bytes(512, 128) == 512 * 64 * 8
    assert lib.ark_attn_rope_table_bytes(0, 128) == 0
    assert lib.ark_attn_rope_table_init(None, 512, 128, 1e6, None) == ops.ARK_ERR_INVALID_ARG
    assert lib.ark_attn_rope_table_init(FAKE, 0, 128, 1e6, None) == ops.ARK_ERR_INVALID_ARG
    assert lib.ark_attn_rope_table_init(FAKE, 70000, 128, 1e6, None) == ops.ARK_ERR_UNSUPPORTED
    assert lib.ark_attn_rope_table_init(FAKE, 512, 64, 1e6, None) == ops.ARK_ERR_UNSUPPORTED
    assert lib.ark_attn_rope_table_init(FAKE, 512, 128, 0.5, None) == ops.ARK_ERR_INVALID_ARG


def append(lib, q=FAKE, kn=FAKE, vn=FAKE, ck=FAKE, cv=FAKE, p0=FAKE, nn=FAKE, B=2, S=1, T=512,
           Hq=16, Hkv=2, D=128, table=FAKE):
    return lib.ark_attn_append_rope(q, kn, vn, ck, cv, p0, nn, B, S, T, Hq, Hkv, D, table, None, None)


def test_append_rope_arg_checks(lib):
    assert append(lib, q=None) == ops.ARK_ERR_INVALID_ARG
    assert append(lib, table=None) == ops.ARK_ERR_INVALID_ARG
    assert append(lib, B=0) == ops.ARK_ERR_INVALID_ARG
    assert append(lib, S=-1) == ops.ARK_ERR_INVALID_ARG
    assert append(lib, Hq=15) == ops.ARK_ERR_INVALID_ARG
    assert append(lib, D=64) == ops.ARK_ERR_UNSUPPORTED
    assert append(lib, Hq=32) == ops.ARK_ERR_UNSUPPORTED
    assert append(lib, T=70000) == ops.ARK_ERR_UNSUPPORTED
    assert append(lib, ck=FAKE_MIS) == ops.ARK_ERR_INVALID_ARG


def decode(lib, q=FAKE, ck=FAKE, cv=FAKE, kv=FAKE, B=32, T=512, Hq=16, Hkv=2, D=128, scale=0.088,
           mode=0, ms=8, ws=None, ws_bytes=0, o=FAKE, lse=FAKE):
    return lib.ark_attn_decode(q, ck, cv, kv, B, T, Hq, Hkv, D, scale, mode, ms, ws, ws_bytes, o, lse,
                               None, None)


def test_decode_arg_checks(lib):
    need = lib.ark_attn_decode_workspace_size(32, 16, 128, 512, 8)
    assert need > 0
    assert decode(lib, q=None, ws=FAKE, ws_bytes=need) == ops.ARK_ERR_INVALID_ARG
    assert decode(lib, o=None, ws=FAKE, ws_bytes=need) == ops.ARK_ERR_INVALID_ARG
    assert decode(lib, D=96, ws=FAKE, ws_bytes=need) == ops.ARK_ERR_UNSUPPORTED
    assert decode(lib, Hkv=4, ws=FAKE, ws_bytes=need) == ops.ARK_ERR_UNSUPPORTED
    assert decode(lib, Hkv=3, ws=FAKE, ws_bytes=need) == ops.ARK_ERR_INVALID_ARG
    assert decode(lib, ms=0, ws=FAKE, ws_bytes=need) == ops.ARK_ERR_INVALID_ARG
    assert decode(lib, mode=7, ws=FAKE, ws_bytes=need) == ops.ARK_ERR_INVALID_ARG
    assert decode(lib, scale=0.0, ws=FAKE, ws_bytes=need) == ops.ARK_ERR_INVALID_ARG
    assert decode(lib, q=FAKE_MIS, ws=FAKE, ws_bytes=need) == ops.ARK_ERR_INVALID_ARG
    assert decode(lib) == ops.ARK_ERR_WORKSPACE
    assert decode(lib, ws=FAKE, ws_bytes=need - 1) == ops.ARK_ERR_WORKSPACE


def test_decode_workspace_size(lib):
    ws = lib.ark_attn_decode_workspace_size
    wsl = lib.ark_attn_decode_layers_workspace_size
    n = ws(32, 16, 128, 512, 8)
    # two partial slots [8 heads x 128] fp32 (and their 8 lse) for each of up to 2048 warps
    assert n >= 2048 * 2 * 8 * 128 * 4 + 2048 * 2 * 8 * 4
    assert n == ws(32, 16, 128, 2048, 1)          # independent of T and the split bound
    assert wsl(36, 32, 16, 128, 512, 8) == n      # and of the layer count and batch
    assert ws(4096, 16, 128, 512, 8) == n
    assert ws(0, 16, 128, 512, 8) == 0
    assert wsl(0, 32, 16, 128, 512, 8) == 0


def test_combine_arg_checks(lib):
    c = lib.ark_attn_combine
    assert c(None, FAKE, 2, 16, 4, 128, FAKE, FAKE, None) == ops.ARK_ERR_INVALID_ARG
    assert c(FAKE, FAKE, 2, 16, 0, 128, FAKE, FAKE, None) == ops.ARK_ERR_INVALID_ARG
    assert c(FAKE, FAKE, 2, 16, 4, 64, FAKE, FAKE, None) == ops.ARK_ERR_UNSUPPORTED
    assert c(FAKE_MIS, FAKE, 2, 16, 4, 128, FAKE, FAKE, None) == ops.ARK_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 1, 16, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.ark_attn_decode(q, q, q, torch.zeros(1, dtype=torch.int32), q, torch.zeros(16), 0.1)


def test_encoder_arg_checks(lib):
    def enc(q=FAKE, k=FAKE, v=FAKE, ln=FAKE, B=2, S=100, H=20, D=64, scale=0.125, o=FAKE, lse=FAKE):
        return lib.ark_attn_encoder(q, k, v, ln, B, S, H, D, scale, o, lse, None, None)
    assert enc(q=None) == ops.ARK_ERR_INVALID_ARG
    assert enc(lse=None) == ops.ARK_ERR_INVALID_ARG
    assert enc(B=0) == ops.ARK_ERR_INVALID_ARG
    assert enc(S=-3) == ops.ARK_ERR_INVALID_ARG
    assert enc(scale=0.0) == ops.ARK_ERR_INVALID_ARG
    assert enc(D=128) == ops.ARK_ERR_UNSUPPORTED
    assert enc(H=70000) == ops.ARK_ERR_UNSUPPORTED
    assert enc(v=FAKE_MIS) == ops.ARK_ERR_INVALID_ARG
    assert enc(lse=FAKE + 2) == ops.ARK_ERR_INVALID_ARG


def test_qkv_arg_checks(lib):
    def proj(x=FAKE, w=FAKE, bias=None, M=32, K=2048, N=2560, out=FAKE):
        return lib.ark_attn_qkv_proj(x, w, bias, M, K, N, out, None, None)
    assert proj(x=None) == ops.ARK_ERR_INVALID_ARG
    assert proj(out=None) == ops.ARK_ERR_INVALID_ARG
    assert proj(M=0) == ops.ARK_ERR_INVALID_ARG
    assert proj(K=2000) == ops.ARK_ERR_INVALID_ARG          # K % 64
    assert proj(N=2500) == ops.ARK_ERR_INVALID_ARG          # N % 128
    assert proj(w=FAKE_MIS) == ops.ARK_ERR_INVALID_ARG
    assert proj(bias=FAKE + 1) == ops.ARK_ERR_INVALID_ARG   # bf16 bias must be 2-byte aligned

    def fused(x=FAKE, w=FAKE, pos0=FAKE, n_new=FAKE, B=32, S=1, T=512, Hq=16, Hkv=2, D=128, K=2048,
              table=FAKE, q=FAKE, ck=FAKE, cv=FAKE):
        return lib.ark_attn_qkv_rope_append(x, w, None, pos0, n_new, B, S, T, Hq, Hkv, D, K, table, q, ck, cv,
                                            None, None)
    assert fused(table=None) == ops.ARK_ERR_INVALID_ARG
    assert fused(n_new=None) == ops.ARK_ERR_INVALID_ARG
    assert fused(B=0) == ops.ARK_ERR_INVALID_ARG
    assert fused(K=100) == ops.ARK_ERR_INVALID_ARG
    assert fused(D=64) == ops.ARK_ERR_UNSUPPORTED
    assert fused(ck=FAKE_MIS) == ops.ARK_ERR_INVALID_ARG
