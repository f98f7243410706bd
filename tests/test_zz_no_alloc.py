"""fa2_backward_noalloc: the backward pass for callers that cannot allocate
device memory (e.g. code inside an engine whose memory pool owns the GPU's
memory and that is handed only its input and output buffers).  It keeps its
scratch in a fixed device array inside the library instead of a
caller-provided workspace.

Called here through the C ABI with ctypes, twice in a row, and compared with
fa2_backward on the same inputs.  This file is collected last so that a run
stopping at the first failure has already run every other test."""
import ctypes
import math

import pytest
import torch

import fa2_inputs
from parity_util import TOL

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 << 20


DTYPE_CODE = {"bf16": 0, "fp32": 1, "fp16": 2}


def _call_noalloc(lib, q, k, v, o, lse, do, dq, dk, dv, causal, scale, dtype):
    B, H, N, d = q.shape
    return lib.fa2_backward_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, int(causal), float(scale),
        DTYPE_CODE[dtype], ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


# fp32 inputs keep TF32-rounded copies of q, k, v and dO in the scratch as well
# (most of its use); fp16 runs the 16-bit kernels with fp16 operands.
CASES = [(2, 4, 1000, 64, True, "bf16"), (1, 8, 2048, 128, False, "bf16"),
         (1, 4, 700, 128, True, "fp32"), (2, 2, 333, 80, False, "fp32"),
         (1, 3, 500, 64, True, "fp32"), (1, 2, 300, 32, False, "fp32"),
         (1, 4, 1000, 64, True, "fp16")]


@pytest.mark.parametrize("B,H,N,d,causal,dtype", CASES)
def test_noalloc_matches_workspace_backward_twice(B, H, N, d, causal, dtype):
    import causal_attention_fa2_b200 as fa2
    from causal_attention_fa2_b200 import _native
    lib = _native.lib()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    scale = 1.0 / math.sqrt(d)
    inp = fa2_inputs.make_inputs(B, H, N, d, dtype, seed=123 + N)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    assert fa2.backward_workspace_bytes(B, H, N, d, q.dtype) <= SCRATCH_BYTES
    o, lse = fa2.forward(q, k, v, causal=causal, scale=scale)
    # fa2_backward_noalloc runs the two-pass form; compare with the same form.
    ref = fa2.backward(q, k, v, o, lse, do, causal=causal, scale=scale, mode="two-pass")
    atol, rtol = TOL[dtype]
    for _ in range(2):
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        st = _call_noalloc(lib, q, k, v, o, lse, do, dq, dk, dv, causal, scale, dtype)
        assert st == 0, _native.status_string(st)
        torch.cuda.synchronize()
        for got, want in zip((dq, dk, dv), ref):
            torch.testing.assert_close(got.float(), want.float(), atol=atol, rtol=rtol)
        # The backward is deterministic: same inputs, same bits.
        assert torch.equal(dq, ref[0]) and torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
    assert fa2.last_device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from causal_attention_fa2_b200 import _native
    lib = _native.lib()
    # B=1, H=1024, N=16384 needs 128 MiB of scratch (> 64 MiB).
    assert lib.fa2_backward_workspace_bytes(1, 1024, 16384, 128, 0) > SCRATCH_BYTES
    fake = 0x10000  # never dereferenced: the size check fails before any launch
    st = lib.fa2_backward_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                  1, 1024, 16384, 128, 1, 0.088, 0, None)
    assert st == 11, _native.status_string(st)   # FA2_ERR_SCRATCH_TOO_SMALL
    assert "64 MiB" in _native.status_string(st)
