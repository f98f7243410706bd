"""Host-only checks of the C ABI: libfa2.so builds for sm_100a, loads without a
GPU, exports every function include/fa2.h declares, and rejects bad
arguments with the documented status codes before touching the device."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa2.h")


@pytest.fixture(scope="module")
def fa2lib():
    from causal_attention_fa2_b200 import build, _native
    build.build()
    return _native.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa2_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_function(fa2lib):
    from causal_attention_fa2_b200 import _native
    declared = header_functions()
    assert declared, "no declarations parsed from fa2.h"
    assert set(declared) == set(_native.SIGNATURES), "binding and header disagree"
    for name in declared:
        assert hasattr(fa2lib, name), f"libfa2.so does not export {name}"


def test_status_strings(fa2lib):
    from causal_attention_fa2_b200 import _native
    seen = set()
    for code in range(12):
        s = _native.status_string(code)
        assert s.startswith("FA2_"), s
        seen.add(s)
    assert len(seen) == 12
    assert "unknown" in _native.status_string(99)


# Fake, 256-byte aligned, never dereferenced: every call below fails host-side
# validation before anything reaches the device.
P = 0x10000
BAD = 0x10002


def fwd(lib, q=P, k=P, v=P, o=P, lse=P, B=1, H=1, N=128, d=64, causal=1, scale=0.125, dtype=0):
    return lib.fa2_forward(q, k, v, o, lse, B, H, N, d, causal, scale, dtype, None)


def bwd(lib, ws_bytes=1 << 30, ws=P, d=64, dtype=0, N=128, dq=P, lse=P, causal=1):
    return lib.fa2_backward(P, P, P, P, lse, P, dq, P, P, 1, 1, N, d, causal, 0.125, dtype, ws,
                            ws_bytes, None)


def test_forward_validation(fa2lib):
    L = fa2lib
    assert fwd(L, q=None) == 1                     # FA2_ERR_NULL_PTR
    assert fwd(L, lse=None) == 1
    assert fwd(L, N=0) == 2                        # FA2_ERR_BAD_SHAPE
    assert fwd(L, B=0) == 2
    assert fwd(L, H=-1) == 2
    assert fwd(L, N=(1 << 24) + 1) == 2
    for d in (0, 8, 48, 96, 256):
        assert fwd(L, d=d) == 3                    # FA2_ERR_UNSUPPORTED_HEAD_DIM
    assert fwd(L, dtype=3) == 4                    # FA2_ERR_UNSUPPORTED_DTYPE
    assert fwd(L, q=BAD) == 5                      # FA2_ERR_MISALIGNED
    assert fwd(L, o=P + 8) == 5
    assert fwd(L, lse=P + 2) == 5
    assert fwd(L, causal=2) == 10                  # FA2_ERR_BAD_ARGUMENT
    assert fwd(L, scale=float("inf")) == 10
    assert fwd(L, scale=float("nan")) == 10
    assert fwd(L, scale=0.0) == 10                 # the scale must be positive
    assert fwd(L, scale=-0.125) == 10


def test_backward_validation(fa2lib):
    L = fa2lib
    need = L.fa2_backward_workspace_bytes(1, 1, 128, 64, 0)
    assert bwd(L, ws_bytes=need - 1) == 6          # FA2_ERR_WORKSPACE_TOO_SMALL
    assert bwd(L, ws=P + 16) == 5                  # workspace must be 256-byte aligned
    assert bwd(L, dq=None) == 1
    assert bwd(L, d=96) == 3
    assert bwd(L, dtype=5) == 4
    assert bwd(L, causal=-1) == 10


@pytest.mark.parametrize("B,H,N,d", [(1, 1, 1, 16), (2, 3, 200, 80), (1, 36, 4096, 128)])
def test_workspace_size(fa2lib, B, H, N, d):
    """D and log2-scaled L (fp32, padded to whole 128-row tiles), each region
    rounded up to 256 bytes; for 16-bit inputs with more than one key tile
    also the one-pass backward's fp32 dQ accumulator; for fp32 inputs four
    operand copies instead."""
    def up(x):
        return (x + 255) // 256 * 256
    n_pad = (N + 127) // 128 * 128
    expect = 2 * up(B * H * n_pad * 4)
    acc = up(B * H * n_pad * d * 4) if N > 128 else 0
    assert fa2lib.fa2_backward_workspace_bytes(B, H, N, d, 0) == expect + acc
    assert fa2lib.fa2_backward_workspace_bytes(B, H, N, d, 2) == expect + acc  # fp16
    for dt in (0, 1, 2):
        assert fa2lib.fa2_backward_workspace_bytes_ex(B, H, H, N, N, d, dt) == \
            fa2lib.fa2_backward_workspace_bytes(B, H, N, d, dt)
    # fp32 with other key/value shapes: the k and v copies follow H_kv and Nk.
    nk, hkv = N + 77, 1
    assert fa2lib.fa2_backward_workspace_bytes_ex(B, H, hkv, N, nk, d, 1) == \
        expect + 2 * up(B * H * N * d * 4) + 2 * up(B * hkv * nk * d * 4)
    # fp32 inputs: plus TF32-rounded copies of q, k, v and dout.
    assert fa2lib.fa2_backward_workspace_bytes(B, H, N, d, 1) == expect + 4 * up(B * H * N * d * 4)
    assert fa2lib.fa2_backward_workspace_bytes(B, H, N, 24, 0) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path only")
def test_valid_call_without_gpu_reports_cuda_error(fa2lib):
    assert fwd(fa2lib) in (7, 9)                   # FA2_ERR_CUDA / UNSUPPORTED_DEVICE
    assert fa2lib.fa2_last_device_status() in (7, 9)
    assert fa2lib.fa2_watchdog_selftest(1_000_000, None) in (7, 9)


def test_watchdog_selftest_limit_validation(fa2lib):
    for bad in (0, 999, 10**10 + 1, 2**64 - 1):
        assert fa2lib.fa2_watchdog_selftest(bad, None) == 10      # FA2_ERR_BAD_ARGUMENT


def test_binding_rejects_cpu_tensors():
    import causal_attention_fa2_b200 as fa2
    x = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa2.forward(x, x, x)


def test_ex_shape_validation(fa2lib):
    """fa2_forward_ex / fa2_backward_ex: H must be a positive multiple of H_kv,
    and the key length is bounded like the query length."""
    L = fa2lib

    def fwd_ex(H, H_kv, Nk=128):
        return L.fa2_forward_ex(P, P, P, P, P, 1, H, H_kv, 128, Nk, 64, 1, 0.125, 0, None)

    def bwd_ex(H, H_kv, Nk=128):
        return L.fa2_backward_ex(P, P, P, P, P, P, P, P, P, 1, H, H_kv, 128, Nk, 64, 1, 0.125, 0,
                                 P, 1 << 30, None)

    for H, H_kv in ((4, 3), (4, 0), (4, 8), (6, -2)):
        assert fwd_ex(H, H_kv) == 2, (H, H_kv)      # FA2_ERR_BAD_SHAPE
        assert bwd_ex(H, H_kv) == 2, (H, H_kv)
    assert fwd_ex(0, 1) == 2
    for Nk in (0, -5, (1 << 24) + 1):
        assert fwd_ex(4, 2, Nk) == 2, Nk
        assert bwd_ex(4, 2, Nk) == 2, Nk


def test_block_sparse_validation(fa2lib):
    """fa2_forward_block_sparse / fa2_backward_block_sparse: the mask pointer is
    required, checked before touching the device (every input type and any
    number of tiles per side are accepted)."""
    L = fa2lib

    def fwd(mask, N=256, Nk=256, dtype=0):
        return L.fa2_forward_block_sparse(P, P, P, P, P, 1, 4, 2, N, Nk, 64, 1, 0.125, dtype,
                                          mask, None)

    def bwd(mask, N=256, Nk=256, dtype=0):
        return L.fa2_backward_block_sparse(P, P, P, P, P, P, P, P, P, 1, 4, 2, N, Nk, 64, 1, 0.125,
                                           dtype, mask, P, 1 << 30, None)

    assert fwd(None) == 1 and bwd(None) == 1                # FA2_ERR_NULL_PTR
    assert fwd(None, dtype=1) == 1 and bwd(None, dtype=1) == 1


def test_binding_block_mask_checks():
    import causal_attention_fa2_b200 as fa2
    q = torch.zeros(1, 1, 300, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa2._check_block_mask(torch.ones(2, 3, dtype=torch.bool), q, 300, 300)   # wrong shape
    with pytest.raises(ValueError):
        fa2._check_block_mask(torch.ones(3, 3, dtype=torch.bool), q, 300, 300)   # not on CUDA


def test_workspace_size_split_groups(fa2lib):
    """16-bit grouped-query shapes with fewer than 148 (key tile, key/value
    head) blocks: the workspace adds fp32 partial dK, dV for S splits."""
    def up(x):
        return (x + 255) // 256 * 256
    for B, H, hkv, N, nk, d in ((1, 8, 1, 512, 512, 64), (2, 36, 4, 4096, 4096, 128), (1, 4, 2, 300, 300, 80)):
        n_pad = -(-N // 128) * 128
        tk = -(-nk // 128)
        base = 2 * up(B * H * n_pad * 4)
        ctas = tk * B * hkv
        S = 1 if ctas >= 148 else min(H // hkv, -(-296 // ctas))
        part = up(2 * S * B * hkv * tk * 128 * d * 4) if S > 1 else 0
        # no split and more than one key tile: the one-pass form's dQ accumulator
        acc = up(B * H * n_pad * d * 4) if (S == 1 and tk > 1) else 0
        for dt in (0, 2):
            assert fa2lib.fa2_backward_workspace_bytes_ex(B, H, hkv, N, nk, d, dt) == base + part + acc, (B, H, hkv, S)
    # multi-head: never split
    assert fa2lib.fa2_backward_workspace_bytes_ex(1, 4, 4, 256, 256, 64, 0) == \
        fa2lib.fa2_backward_workspace_bytes(1, 4, 256, 64, 0)


def test_plain_c_caller(fa2lib, tmp_path):
    """include/fa2.h compiles as strict C11 and a C program linked against
    libfa2.so gets the documented validation codes (tests/c_abi_check.c)."""
    import subprocess
    pkg = os.path.join(ROOT, "causal_attention_fa2_b200")
    exe = tmp_path / "c_abi_check"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"),
                    "-L", pkg, "-lfa2", f"-Wl,-rpath,{pkg}", "-lm", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr


def test_binding_buffer_checks():
    """Caller-supplied outputs and workspace must match what the library writes
    through their raw pointers (checked before any call; CPU tensors suffice)."""
    from causal_attention_fa2_b200 import _check_buffer, _check_workspace
    cpu = torch.device("cpu")
    good = torch.empty(2, 3, 5, 8, dtype=torch.bfloat16)
    _check_buffer("o", good, (2, 3, 5, 8), torch.bfloat16, cpu)
    bad = [
        torch.empty(2, 3, 5, 4, dtype=torch.bfloat16),                 # wrong shape
        torch.empty(2, 3, 5, 8, dtype=torch.float16),                  # wrong dtype
        torch.empty(2, 3, 8, 5, dtype=torch.bfloat16).transpose(2, 3),  # not contiguous
    ]
    for t in bad:
        with pytest.raises(ValueError):
            _check_buffer("o", t, (2, 3, 5, 8), torch.bfloat16, cpu)
    with pytest.raises(ValueError):
        _check_buffer("o", good, (2, 3, 5, 8), torch.bfloat16, torch.device("cuda", 0))
    _check_workspace(torch.empty(1024, dtype=torch.uint8), cpu)
    for t in (torch.empty(256, dtype=torch.float32), torch.empty(4, 256, dtype=torch.uint8),
              torch.empty(2048, dtype=torch.uint8)[::2]):
        with pytest.raises(ValueError):
            _check_workspace(t, cpu)
