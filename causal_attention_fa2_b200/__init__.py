"""FlashAttention-2 (causal multi-head attention forward and recomputation
backward) for NVIDIA B200, sm_100a.

Every step of the computation runs in the CUDA kernels of ``libfa2.so``
(C ABI declared in ``include/fa2.h``).  This module only marshals arguments:
it checks tensors, allocates outputs with PyTorch, passes raw device pointers
and the current CUDA stream to the library, and turns status codes into
exceptions.  There is no CPU or PyTorch fallback: without the library or a
B200 the calls raise.

Semantics follow the CS336 A2 Systems handout, section 4.2.2: Algorithm 1 for
the forward (O and the logsumexp L), Eqs. 13-19 with D = rowsum(O o dO) for
the backward, and the causal rule of Problem flash_forward (c).
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional, Tuple

import torch

from . import _native
from ._native import (FA2_BF16, FA2_FP16, FA2_FP32, FA2Error, clear_device_status,  # noqa: F401
                      last_device_status, library_path, status_string)

__all__ = [
    "forward", "backward", "backward_workspace_bytes", "flash_attention",
    "FlashAttention2Function", "last_device_status", "clear_device_status",
    "status_string", "FA2Error", "library_path", "watchdog_selftest",
]

SUPPORTED_HEAD_DIMS = (16, 32, 64, 80, 128)
_DTYPES = {torch.bfloat16: FA2_BF16, torch.float32: FA2_FP32, torch.float16: FA2_FP16}


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16, torch.float16 or torch.float32")


def _check_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
    """q [B, H, N, d]; k, v [B, H_kv, Nk, d] with H a multiple of H_kv (H_kv < H:
    grouped-query attention; Nk != N: different key length).  Returns
    (B, H, H_kv, N, Nk, d)."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("expected q of shape [B, H, N, d] and k, v of shape [B, H_kv, Nk, d]")
    B, H, N, d = q.shape
    if (k.shape != v.shape or k.shape[0] != B or k.shape[3] != d
            or k.shape[1] < 1 or H % k.shape[1]):
        raise ValueError(f"q, k, v shapes do not fit [B, H, N, d] / [B, H_kv, Nk, d] with H a multiple "
                         f"of H_kv: {tuple(q.shape)}, {tuple(k.shape)}, {tuple(v.shape)}")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous [B, H, N, d]")
    if k.device != q.device or v.device != q.device:
        raise ValueError("q, k, v must be on one device")
    return B, H, k.shape[1], N, k.shape[2], d


def _stream_handle(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_buffer(name: str, t: torch.Tensor, shape, dtype: torch.dtype, device: torch.device) -> None:
    """A caller-supplied output or scratch tensor must be exactly what the
    library will write through its raw pointer."""
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or t.device != device or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} on "
                         f"{device}; got {t.dtype} {tuple(t.shape)} on {t.device}"
                         f"{'' if t.is_contiguous() else ' (not contiguous)'}")


def _check_workspace(t: torch.Tensor, device: torch.device) -> None:
    if t.dtype != torch.uint8 or t.dim() != 1 or t.device != device or not t.is_contiguous():
        raise ValueError(f"workspace must be a contiguous 1-D torch.uint8 tensor on {device}; got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


BLOCK = 128  # rows per block of a block-sparse mask (the kernels' tile size)

# backward(mode=...) -> flags of fa2_backward_opts
_BWD_MODES = {"default": 0, "two-pass": _native.FA2_BWD_DETERMINISTIC,
              "one-pass": _native.FA2_BWD_ONE_PASS}


def _check_block_mask(block_mask: torch.Tensor, q: torch.Tensor, N: int, Nk: int) -> torch.Tensor:
    """block_mask: CUDA bool / uint8 tensor [ceil(N / 128), ceil(Nk / 128)] on q's
    device; returned as a contiguous uint8 tensor (nonzero = block computed)."""
    want = ((N + BLOCK - 1) // BLOCK, (Nk + BLOCK - 1) // BLOCK)
    if tuple(block_mask.shape) != want:
        raise ValueError(f"block_mask must have shape {want} (blocks of {BLOCK} rows), got "
                         f"{tuple(block_mask.shape)}")
    if not block_mask.is_cuda or block_mask.device != q.device:
        raise ValueError("block_mask must be a CUDA tensor on the device of q")
    if block_mask.dtype not in (torch.bool, torch.uint8):
        raise TypeError("block_mask must be torch.bool or torch.uint8")
    return block_mask.to(torch.uint8).contiguous()


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True,
            scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
            lse: Optional[torch.Tensor] = None,
            block_mask: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """O = softmax(scale * Q K^T (+ causal mask)) V and L = logsumexp (fp32).

    q: contiguous CUDA tensor [B, H, N, d] (bf16, fp16 or fp32); k, v:
    [B, H_kv, Nk, d] with H a multiple of H_kv (grouped-query attention when
    H_kv < H: query head h uses key/value head h // (H // H_kv)); with
    causal, key j is visible to query i iff j <= i.  ``block_mask`` (optional):
    block-sparse attention, a CUDA bool / uint8 tensor
    [ceil(N / 128), ceil(Nk / 128)]; zero blocks of 128 x 128 rows are skipped,
    rows that see no key get O = 0 and L = -inf.
    Returns (o [B, H, N, d] in the input dtype, lse [B, H, N] float32).
    """
    B, H, H_kv, N, Nk, d = _check_qkv(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_buffer("out", out, q.shape, q.dtype, q.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    else:
        _check_buffer("lse", lse, (B, H, N), torch.float32, q.device)
    if block_mask is not None:
        bm = _check_block_mask(block_mask, q, N, Nk)
        with torch.cuda.device(q.device):
            _native.check(_native.lib().fa2_forward_block_sparse(
                q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                B, H, H_kv, N, Nk, d, int(bool(causal)), float(scale), _dtype_code(q),
                bm.data_ptr(), _stream_handle(q.device)))
        return out, lse
    with torch.cuda.device(q.device):
        if H_kv == H and Nk == N:
            _native.check(_native.lib().fa2_forward(
                q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                B, H, N, d, int(bool(causal)), float(scale), _dtype_code(q),
                _stream_handle(q.device)))
        else:
            _native.check(_native.lib().fa2_forward_ex(
                q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                B, H, H_kv, N, Nk, d, int(bool(causal)), float(scale), _dtype_code(q),
                _stream_handle(q.device)))
    return out, lse


def backward_workspace_bytes(B: int, H: int, N: int, d: int, dtype: torch.dtype,
                             H_kv: Optional[int] = None, Nk: Optional[int] = None) -> int:
    """Workspace bytes of backward(); H_kv and Nk default to H and N."""
    H_kv = H if H_kv is None else H_kv
    Nk = N if Nk is None else Nk
    return int(_native.lib().fa2_backward_workspace_bytes_ex(B, H, H_kv, N, Nk, d, _DTYPES[dtype]))


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
             lse: torch.Tensor, do: torch.Tensor, causal: bool = True,
             scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
             dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
             dv: Optional[torch.Tensor] = None, events=None,
             block_mask: Optional[torch.Tensor] = None, mode: str = "default"):
    """dQ, dK, dV of sum(dO * O) via the recomputation backward.

    ``o`` and ``lse`` are the forward's outputs; ``workspace`` (optional) is a
    uint8 CUDA tensor of at least backward_workspace_bytes(...) bytes.
    ``events`` (optional, for profiling): four recorded-once torch.cuda.Event
    objects the library records at its kernel boundaries (before the D/L
    pre-pass, after it, after the query-tile pass, after the key-tile pass).
    ``block_mask``: the forward's block-sparse mask (see forward()).
    ``mode``: "default" (the library's choice, flags = 0), "two-pass"
    (FA2_BWD_DETERMINISTIC: every output bitwise reproducible) or "one-pass"
    (FA2_BWD_ONE_PASS where it applies: one pass over key tiles with dQ summed
    by fp32 reduce-add, so dQ bits can change from run to run; dK and dV are
    bitwise reproducible either way).
    """
    flags = _BWD_MODES.get(mode)
    if flags is None:
        raise ValueError(f"mode must be one of {sorted(_BWD_MODES)}, got {mode!r}")
    B, H, H_kv, N, Nk, d = _check_qkv(q, k, v)
    for name, t in (("o", o), ("do", do)):
        _check_buffer(name, t, q.shape, q.dtype, q.device)
    _check_buffer("lse", lse, (B, H, N), torch.float32, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = backward_workspace_bytes(B, H, N, d, q.dtype, H_kv, Nk)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    else:
        _check_workspace(workspace, q.device)
    for name, t, like in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if t is not None:
            _check_buffer(name, t, like.shape, like.dtype, like.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ev_arr = None
    if events is not None:
        if len(events) != 4:
            raise ValueError("events must hold four torch.cuda.Event objects")
        if H_kv != H or Nk != N:
            raise ValueError("events are supported for H_kv == H and Nk == N only")
        ev_arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    if events is None:
        bm = None if block_mask is None else _check_block_mask(block_mask, q, N, Nk)
        with torch.cuda.device(q.device):
            _native.check(_native.lib().fa2_backward_opts(
                q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, H_kv, N, Nk, d,
                int(bool(causal)), float(scale), _dtype_code(q),
                None if bm is None else bm.data_ptr(), flags, workspace.data_ptr(),
                workspace.numel() * workspace.element_size(), _stream_handle(q.device)))
        return dq, dk, dv
    if block_mask is not None or flags:
        raise ValueError("events are supported for the default mode without a block mask only")
    with torch.cuda.device(q.device):
        _native.check(_native.lib().fa2_backward_timed(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
            do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
            int(bool(causal)), float(scale), _dtype_code(q), workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), _stream_handle(q.device), ev_arr))
    return dq, dk, dv


def watchdog_selftest(limit_ns: int = 1_000_000, device: Optional[torch.device] = None) -> None:
    """Enqueue the library's watchdog self-test on the current stream of
    ``device`` (default: the current CUDA device): one wait that nothing
    satisfies ends after ``limit_ns`` ns and records FA2_ERR_DEVICE_TIMEOUT in
    the status word, which last_device_status() returns after a synchronize."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _native.check(_native.lib().fa2_watchdog_selftest(int(limit_ns), _stream_handle(dev)))


class FlashAttention2Function(torch.autograd.Function):
    """autograd wrapper with the handout's interface: forward(ctx, Q, K, V,
    is_causal=False) saves L, Q, K, V, O and the causal flag; backward(dO)
    returns dQ, dK, dV (handout section 4.2.2, Problems flash_forward and
    flash_backward)."""

    @staticmethod
    def forward(ctx, Q, K, V, is_causal=False):
        o, lse = forward(Q, K, V, causal=is_causal)
        ctx.save_for_backward(lse, Q, K, V, o)
        ctx.is_causal = bool(is_causal)
        return o

    @staticmethod
    def backward(ctx, dO):
        lse, Q, K, V, o = ctx.saved_tensors
        dq, dk, dv = backward(Q, K, V, o, lse, dO.contiguous(), causal=ctx.is_causal)
        return dq, dk, dv, None


def flash_attention(q, k, v, is_causal: bool = False):
    """Differentiable attention: FlashAttention2Function.apply(q, k, v, is_causal)."""
    return FlashAttention2Function.apply(q, k, v, is_causal)
