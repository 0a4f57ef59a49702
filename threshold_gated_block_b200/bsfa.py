"""Python binding of the BSFA C ABI (include/bsfa.h).

Argument marshalling only: every step of the forward runs in the CUDA kernels
of libbsfa.so. PyTorch supplies device memory and streams. There is no CPU
fallback: if the library is missing or the device is not sm_100, calls fail
loudly.

The functions named like the C entry points (``bsfa_forward``,
``bsfa_forward_tau_table``, ``bsfa_forward_gap``, ``bsfa_forward_heads``, ``bsfa_forward_rows``, ``bsfa_forward_host``,
``bsfa_forward_varlen``, ``bsfa_validate``,
``bsfa_get_status``, ``bsfa_get_debug_counts``,
``bsfa_selftest_lost_arrival``, ``bsfa_status_string``, ``bsfa_last_error``)
take the same arguments; pointer arguments accept an int
address, None, or a torch tensor (its ``data_ptr()``). ``forward`` and
``forward_host`` are conveniences over ``bsfa_forward`` for torch tensors.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsfa.so")

BSFA_OK = 0
BSFA_ERR_INVALID_ARG = 1
BSFA_ERR_UNSUPPORTED = 2
BSFA_ERR_CUDA = 3
BSFA_ERR_DEVICE_TIMEOUT = 4

EXPORTED = ("bsfa_forward", "bsfa_forward_tau_table", "bsfa_forward_gap", "bsfa_forward_heads", "bsfa_forward_rows",
            "bsfa_forward_host",
            "bsfa_forward_varlen", "bsfa_validate", "bsfa_get_status", "bsfa_get_debug_counts",
            "bsfa_selftest_lost_arrival", "bsfa_status_string", "bsfa_last_error")

_lib = None


class BsfaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{bsfa_status_string(status)}: {detail}")
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libbsfa.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with threshold_gated_block_b200.build.build()")
    lib = ctypes.CDLL(path)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.bsfa_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp]
    lib.bsfa_forward.restype = i
    lib.bsfa_forward_tau_table.argtypes = [vp, vp, vp, vp, i, vp, vp, vp, i, i, i, i, i, i, i, i, vp]
    lib.bsfa_forward_tau_table.restype = i
    lib.bsfa_forward_gap.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp]
    lib.bsfa_forward_gap.restype = i
    lib.bsfa_forward_heads.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, i, vp]
    lib.bsfa_forward_heads.restype = i
    lib.bsfa_forward_rows.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, i, vp]
    lib.bsfa_forward_rows.restype = i
    lib.bsfa_forward_host.argtypes = [vp] * 12 + [i] * 9 + [vp]
    lib.bsfa_forward_host.restype = i
    lib.bsfa_forward_varlen.argtypes = [vp, vp, vp, vp, i, i, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    lib.bsfa_forward_varlen.restype = i
    lib.bsfa_validate.argtypes = [i] * 8
    lib.bsfa_validate.restype = i
    lib.bsfa_get_status.argtypes = [vp]
    lib.bsfa_get_status.restype = i
    lib.bsfa_get_debug_counts.argtypes = [vp, vp, vp]
    lib.bsfa_get_debug_counts.restype = i
    lib.bsfa_selftest_lost_arrival.argtypes = [vp]
    lib.bsfa_selftest_lost_arrival.restype = i
    lib.bsfa_status_string.argtypes = [i]
    lib.bsfa_status_string.restype = ctypes.c_char_p
    lib.bsfa_last_error.argtypes = []
    lib.bsfa_last_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ----------------------------------------------------------------------------- C entry points

def bsfa_forward(q, k, v, tau, out, lse, block_mask, B, Hq, Hkv, N, D, Bq, Bk, causal, stream) -> int:
    return load().bsfa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(tau), _ptr(out), _ptr(lse), _ptr(block_mask),
                               B, Hq, Hkv, N, D, Bq, Bk, int(bool(causal)), _stream(stream))


def bsfa_forward_tau_table(q, k, v, tau_table, tau_tiles, out, lse, block_mask, B, Hq, Hkv, N, D, Bq, Bk, causal,
                           stream) -> int:
    return load().bsfa_forward_tau_table(_ptr(q), _ptr(k), _ptr(v), _ptr(tau_table), int(tau_tiles), _ptr(out),
                                         _ptr(lse), _ptr(block_mask), B, Hq, Hkv, N, D, Bq, Bk, int(bool(causal)),
                                         _stream(stream))


def bsfa_forward_gap(q, k, v, gamma, out, lse, block_mask, B, Hq, Hkv, N, D, Bq, Bk, causal, stream) -> int:
    return load().bsfa_forward_gap(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(out), _ptr(lse), _ptr(block_mask),
                                   B, Hq, Hkv, N, D, Bq, Bk, int(bool(causal)), _stream(stream))


def bsfa_forward_rows(q, k, v, tau, out, lse, block_mask, B, Hq, Hkv, N, D, Bq, Bk, causal, row_begin, row_end,
                      stream) -> int:
    return load().bsfa_forward_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(tau), _ptr(out), _ptr(lse), _ptr(block_mask),
                                    B, Hq, Hkv, N, D, Bq, Bk, int(bool(causal)), int(row_begin), int(row_end),
                                    _stream(stream))


def bsfa_forward_heads(q, k, v, tau, out, lse, block_mask, B, Hq, Hkv, N, D, Bq, Bk, causal, kv_begin, kv_count,
                       stream) -> int:
    return load().bsfa_forward_heads(_ptr(q), _ptr(k), _ptr(v), _ptr(tau), _ptr(out), _ptr(lse), _ptr(block_mask),
                                     B, Hq, Hkv, N, D, Bq, Bk, int(bool(causal)), int(kv_begin), int(kv_count),
                                     _stream(stream))


def bsfa_forward_host(q_host, k_host, v_host, tau_host, out_host, lse_host, q_dev, k_dev, v_dev, tau_dev, out_dev,
                      lse_dev, B, Hq, Hkv, N, D, Bq, Bk, causal, chunks, stream) -> int:
    return load().bsfa_forward_host(*(_ptr(t) for t in (q_host, k_host, v_host, tau_host, out_host, lse_host, q_dev,
                                                        k_dev, v_dev, tau_dev, out_dev, lse_dev)),
                                    B, Hq, Hkv, N, D, Bq, Bk, int(bool(causal)), int(chunks), _stream(stream))


def bsfa_forward_varlen(q, k, v, cu_seqlens, nseq, max_seqlen, tau, out, lse, block_mask, total, Hq, Hkv, D, Bq, Bk,
                        causal, stream) -> int:
    return load().bsfa_forward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), int(nseq), int(max_seqlen),
                                      _ptr(tau), _ptr(out), _ptr(lse), _ptr(block_mask), total, Hq, Hkv, D, Bq, Bk,
                                      int(bool(causal)), _stream(stream))


def bsfa_validate(B, Hq, Hkv, N, D, Bq, Bk, causal) -> int:
    return load().bsfa_validate(B, Hq, Hkv, N, D, Bq, Bk, int(bool(causal)))


def bsfa_get_status(stream=None) -> int:
    return load().bsfa_get_status(_stream(stream))


def bsfa_get_debug_counts(stream, v_tiles, pv_products) -> int:
    """v_tiles, pv_products: ctypes.c_ulonglong objects (passed by reference) or int addresses."""
    conv = lambda x: ctypes.addressof(x) if isinstance(x, ctypes.c_ulonglong) else _ptr(x)
    return load().bsfa_get_debug_counts(_stream(stream), conv(v_tiles), conv(pv_products))


def debug_counts(stream=None) -> tuple[int, int]:
    """(V tiles loaded, PV products issued) by mask-writing launches since the last read; clears them."""
    v, pv = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
    _check(bsfa_get_debug_counts(stream, v, pv))
    return v.value, pv.value


def bsfa_selftest_lost_arrival(stream=None) -> int:
    return load().bsfa_selftest_lost_arrival(_stream(stream))


def bsfa_status_string(status: int) -> str:
    return load().bsfa_status_string(status).decode()


def bsfa_last_error() -> str:
    return load().bsfa_last_error().decode()


# ----------------------------------------------------------------------------- torch conveniences

def _check(status: int):
    if status != BSFA_OK:
        raise BsfaError(status, bsfa_last_error())


def forward(q, k, v, tau, *, Bq: int, Bk: int, causal: bool, want_lse: bool = True, want_mask: bool = False,
            out=None, lse=None, block_mask=None, stream=None, gate: str = "tau"):
    """Run the forward on device tensors. q: bf16 [B,N,Hq,D]; k, v: bf16 [B,N,Hkv,D].

    tau: fp32 [Hq] (one threshold per head, ``bsfa_forward``) or contiguous fp32
    [Hq, T] (per head and query tile, ``bsfa_forward_tau_table`` with tau_tiles = T).
    gate="gap": ``bsfa_forward_gap`` with tau holding gamma [Hq].
    Returns (out, lse or None, block_mask or None). Outputs are allocated with torch
    unless given.
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D bf16 CUDA tensor")
    if (tau.dtype != torch.float32 or not tau.is_cuda or not tau.is_contiguous() or tau.dim() not in (1, 2)
            or tau.shape[0] != q.shape[2]):
        raise ValueError("tau must be a contiguous float32 CUDA tensor [Hq] or [Hq, tiles]")
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, N, Hkv, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B, N, Hkv, D] with q's B, N and D")
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    if want_mask and block_mask is None:
        block_mask = torch.empty((B, Hq, -(-N // Bq), -(-N // Bk)), dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    lse_arg = lse if want_lse else None
    mask_arg = block_mask if want_mask else None
    if gate == "gap":
        if tau.dim() != 1:
            raise ValueError("the gap gate takes one gamma per head")
        _check(bsfa_forward_gap(q, k, v, tau, out, lse_arg, mask_arg, B, Hq, Hkv, N, D, Bq, Bk, causal, stream))
    elif tau.dim() == 1:
        _check(bsfa_forward(q, k, v, tau, out, lse_arg, mask_arg, B, Hq, Hkv, N, D, Bq, Bk, causal, stream))
    else:
        _check(bsfa_forward_tau_table(q, k, v, tau, tau.shape[1], out, lse_arg, mask_arg, B, Hq, Hkv, N, D, Bq, Bk,
                                      causal, stream))
    return out, (lse if want_lse else None), (block_mask if want_mask else None)


def forward_varlen(q, k, v, cu_seqlens, max_seqlen: int, tau, *, Bq: int, Bk: int, causal: bool,
                   want_lse: bool = True, want_mask: bool = False, stream=None):
    """Packed mixed-length batch on device tensors. q: bf16 [total, Hq, D]; k, v: bf16
    [total, Hkv, D]; cu_seqlens: int32 [nseq + 1] CUDA tensor; tau: fp32 [Hq].
    Returns (out [total, Hq, D], lse [Hq, total] or None, block_mask or None)."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous 3-D bf16 CUDA tensor")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be a 1-D int32 CUDA tensor")
    total, Hq, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (total, Hkv, D) or v.shape != k.shape:
        raise ValueError("k and v must be [total, Hkv, D] with q's total and D")
    if tau.dtype != torch.float32 or not tau.is_cuda or not tau.is_contiguous() or tau.shape != (Hq,):
        raise ValueError("tau must be a contiguous float32 CUDA tensor with one value per query head")
    nseq = cu_seqlens.numel() - 1
    if nseq < 1:
        raise ValueError("cu_seqlens needs at least two offsets")
    out = torch.empty_like(q)
    lse = torch.empty((Hq, total), dtype=torch.float32, device=q.device) if want_lse else None
    mask = None
    if want_mask:
        mask = torch.empty((nseq, Hq, -(-max_seqlen // Bq), -(-max_seqlen // Bk)), dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    _check(bsfa_forward_varlen(q, k, v, cu_seqlens, nseq, max_seqlen, tau, out, lse, mask, total, Hq, Hkv, D, Bq, Bk,
                               causal, stream))
    return out, lse, mask


def forward_host(q, k, v, tau, *, Bq: int, Bk: int, causal: bool, device=None, stream=None, bufs=None,
                 gate: str = "tau", chunks: int | None = None):
    """End-to-end call on host tensors: copy inputs to the device, run, copy out and lse back.

    q, k, v: bf16 CPU tensors (pinned for asynchronous copies); tau: fp32 CPU tensor, [Hq] or [Hq, T].
    ``bufs`` (from ``device_buffers``) holds reusable device and pinned host buffers.
    With one threshold per head this is ``bsfa_forward_host``: the copies run in
    ``chunks`` runs of query rows (whole 256-row units, shrinking towards the end;
    default min(ceil(N/256), 8)) overlapped with the kernel.
    Other gates copy, run and copy back in turn on ``stream``.
    Returns (out_host, lse_host).
    """
    import torch
    _check_host_inputs(q, k, v, tau, bufs)
    device = torch.device("cuda") if device is None else device
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if bufs is None:
        bufs = device_buffers(q.shape, k.shape, device, tuple(tau.shape))
    if gate == "tau" and tau.dim() == 1:
        B, N, Hq, D = q.shape
        Hkv = k.shape[2]
        _check(bsfa_forward_host(q, k, v, tau, bufs["out_host"], bufs["lse_host"], bufs["q"], bufs["k"], bufs["v"],
                                 bufs["tau"], bufs["out"], bufs["lse"], B, Hq, Hkv, N, D, Bq, Bk, causal,
                                 chunks or min(-(-N // 256), 8), stream))
        stream.synchronize()
        return bufs["out_host"], bufs["lse_host"]
    with torch.cuda.stream(stream):
        for name, src in (("q", q), ("k", k), ("v", v), ("tau", tau)):
            bufs[name].copy_(src, non_blocking=True)
        forward(bufs["q"], bufs["k"], bufs["v"], bufs["tau"], Bq=Bq, Bk=Bk, causal=causal, out=bufs["out"],
                lse=bufs["lse"], stream=stream, gate=gate)
        bufs["out_host"].copy_(bufs["out"], non_blocking=True)
        bufs["lse_host"].copy_(bufs["lse"], non_blocking=True)
    stream.synchronize()
    return bufs["out_host"], bufs["lse_host"]


def _check_host_inputs(q, k, v, tau, bufs):
    """The host-buffer call reads q, k, v and tau by raw address and copies into
    ``bufs`` by size, so their layouts are checked here, before any copy."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D bf16 host tensor")
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, N, Hkv, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B, N, Hkv, D] with q's B, N and D")
    if (tau.dtype != torch.float32 or tau.is_cuda or not tau.is_contiguous() or tau.dim() not in (1, 2)
            or tau.shape[0] != Hq):
        raise ValueError("tau must be a contiguous float32 host tensor [Hq] or [Hq, tiles]")
    if bufs is None:
        return
    want = {"q": tuple(q.shape), "k": tuple(k.shape), "v": tuple(k.shape), "tau": tuple(tau.shape),
            "out": tuple(q.shape), "lse": (B, Hq, N), "out_host": tuple(q.shape), "lse_host": (B, Hq, N)}
    for name, shape in want.items():
        t = bufs.get(name)
        if t is None or tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"bufs[{name!r}] must be a contiguous tensor of shape {shape}")
        if t.dtype != (torch.bfloat16 if name in ("q", "k", "v", "out", "out_host") else torch.float32):
            raise ValueError(f"bufs[{name!r}] has dtype {t.dtype}")


def device_buffers(q_shape, kv_shape, device, tau_shape=None):
    """Device inputs/outputs plus pinned host outputs for ``forward_host``."""
    import torch
    B, N, Hq, D = q_shape
    return {
        "q": torch.empty(q_shape, dtype=torch.bfloat16, device=device),
        "k": torch.empty(kv_shape, dtype=torch.bfloat16, device=device),
        "v": torch.empty(kv_shape, dtype=torch.bfloat16, device=device),
        "tau": torch.empty(tau_shape or (Hq,), dtype=torch.float32, device=device),
        "out": torch.empty(q_shape, dtype=torch.bfloat16, device=device),
        "lse": torch.empty((B, Hq, N), dtype=torch.float32, device=device),
        "out_host": torch.empty(q_shape, dtype=torch.bfloat16, pin_memory=True),
        "lse_host": torch.empty((B, Hq, N), dtype=torch.float32, pin_memory=True),
    }
