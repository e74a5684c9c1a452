"""Failure detection on the GPU without a GPU fault: the library's bounded
mbarrier wait gives up, reports ARK_DEV_TIMEOUT in the caller's status word and
returns, and the CUDA context stays usable.

Every kernel of the library waits on its TMA copies and MMA completions with
the same bounded wait (csrc/common.cuh); a copy that never lands would
otherwise hold the GPU.  The test-only library built here from
tests/csrc/wait_timeout.cu arms an mbarrier for bytes no copy delivers and
calls that wait, once with a 1 ms limit and once with the library's own limit.
Nothing faults, traps or hangs: the kernel ends by itself after the limit."""
import ctypes
import math
import os
import subprocess

import pytest
import torch

from gqa_attention_static_b200 import build as B
from gqa_attention_static_b200 import ops

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def waitlib():
    os.makedirs(B.BUILD_DIR, exist_ok=True)
    out = os.path.join(B.BUILD_DIR, "libark_wait_timeout_test.so")
    src = os.path.join(HERE, "csrc", "wait_timeout.cu")
    cmd = [B.NVCC] + B.ARCH + B.FLAGS + ["-shared", src, "-o", out, "-cudart", "static"]
    subprocess.check_call(cmd)
    lib = ctypes.CDLL(out)
    lib.ark_test_wait_timeout.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.c_void_p]
    lib.ark_test_wait_timeout.restype = ctypes.c_int
    lib.ark_test_wait_limit_ns.restype = ctypes.c_ulonglong
    return lib


def _run(lib, short):
    dev = "cuda"
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    elapsed = torch.zeros(1, dtype=torch.int64, device=dev)
    returned = torch.zeros(1, dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    assert lib.ark_test_wait_timeout(status.data_ptr(), elapsed.data_ptr(), returned.data_ptr(), int(short), s) == 0
    torch.cuda.synchronize()                 # raises if the kernel faulted
    return int(status.item()), int(elapsed.item()), int(returned.item())


def test_short_wait_gives_up_and_reports(waitlib):
    st, ns, ret = _run(waitlib, True)
    assert ret == 1, "the waiting thread did not return"
    assert st & ops.ARK_DEV_TIMEOUT
    assert 1_000_000 <= ns < 200_000_000, ns


def test_library_limit_gives_up_and_context_stays_usable(waitlib):
    limit = waitlib.ark_test_wait_limit_ns()
    st, ns, ret = _run(waitlib, False)
    assert ret == 1 and st & ops.ARK_DEV_TIMEOUT
    assert limit <= ns < 3 * limit, (ns, limit)
    # the context still runs the library's kernels
    ops.load()
    dev = "cuda"
    q = torch.randn(1, 1, 16, 128, device=dev).to(torch.bfloat16)
    ck = torch.randn(1, 16, 2, 128, device=dev).to(torch.bfloat16)
    cv = torch.randn(1, 16, 2, 128, device=dev).to(torch.bfloat16)
    kv = torch.tensor([16], dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(1, 16, dtype=torch.float32, device=dev)
    ws = ops.decode_workspace(1, 16, 128, 16, 8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.ark_attn_decode(q, ck, cv, kv, o, lse, 1.0 / math.sqrt(128), ops.ARK_LENGTH_AWARE, 8, ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
