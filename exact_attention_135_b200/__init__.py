"""B200-native (sm_100a) fused exact attention: Python binding of libattn_b200.so.

The binding only marshals arguments: it checks dtypes, shapes and devices,
allocates outputs with torch when the caller passes none, and calls the C ABI
(include/attn_b200.h) on torch's current CUDA stream.  Every step of the
computation runs in the library's CUDA kernels; there is no fallback.  If the
library is missing the calls raise instead of computing anything.

    o, lse = fwd(q, k, v, causal=True, scale=None)          # prefill
    o, lse = decode_paged(q, kv_pages, block_table, cache_seqlens, scale)
"""

from __future__ import annotations

import ctypes
import math
import os
import re

import torch

__all__ = ["fwd", "fwd_fp8", "bwd", "bwd_workspace_size", "bwd_head_group", "decode_paged", "decode_paged_mtp",
           "decode_paged_noalloc", "decode_workspace_size", "decode_mtp_workspace_size", "decode_paged_gqa",
           "decode_gqa_workspace_size", "read_device_status", "library", "AttnError", "exported_symbols", "STATUS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libattn_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "attn_b200.h")

STATUS = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_CUDA",
          4: "ATTN_ERR_TIMEOUT", 5: "ATTN_ERR_WORKSPACE"}


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where} failed: {STATUS.get(code, code)}")


_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t

_SIGNATURES = {
    "attn_abi_version": (_i, []),
    "attn_status_string": (ctypes.c_char_p, [_i]),
    "attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "attn_decode_paged_workspace_size": (_sz, [_i, _i, _i, _i]),
    "attn_decode_paged": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp, _sz, _vp]),
    "attn_read_device_status": (_i, [_i]),
    "attn_decode_paged_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "attn_decode_paged_noalloc_max_bytes": (_sz, []),
    "attn_selftest_wait_timeout": (_i, [ctypes.c_uint, _vp]),
    "attn_decode_paged_gqa_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "attn_decode_paged_mtp_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "attn_decode_paged_mtp": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _vp, _sz, _vp]),
    "attn_decode_paged_gqa": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp, _sz, _vp]),
    "attn_fwd_fp8": (_i, [_vp, _vp, _vp, _f, _f, _f, _vp, _vp] + [_i] * 7 + [_f, _vp]),
    "attn_bwd_workspace_size": (_sz, [_i, _i, _i, _i]),
    "attn_bwd_head_group": (_i, [_i] * 8),
    "attn_bwd": (_i, [_vp] * 9 + [_i] * 8 + [_f, _vp, _sz, _vp]),
}


def library():
    """Load the in-tree CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run: python -m exact_attention_135_b200.build)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def exported_symbols():
    """Function names declared in include/attn_b200.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text)))


def _check(rc: int, where: str):
    if rc != 0:
        raise AttnError(rc, where)


def _stream_handle(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False, scale: float | None = None,
        out: torch.Tensor | None = None, lse: torch.Tensor | None = None):
    """Fused exact attention forward.

    q [B,Nq,Hq,D], k [B,Nk,Hkv,D], v [B,Nk,Hkv,Dv], bf16 CUDA tensors.
    Returns (o [B,Nq,Hq,Dv] bf16, lse [B,Hq,Nq] fp32).  scale defaults to
    1/sqrt(D).  Runs on torch's current stream of q's device.
    """
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    B, Nq, Hq, D = q.shape
    Bk, Nk, Hkv, Dk = k.shape
    Dv = v.shape[3]
    if Bk != B or Dk != D or tuple(v.shape[:3]) != (B, Nk, Hkv):
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((B, Nq, Hq, Dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    if tuple(out.shape) != (B, Nq, Hq, Dv) or tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("out/lse shape mismatch")
    with torch.cuda.device(q.device):
        rc = library().attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                B, Hq, Hkv, Nq, Nk, D, Dv, int(bool(causal)), float(scale),
                                _stream_handle(q.device))
    _check(rc, "attn_fwd")
    return out, lse


def fwd_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_descale: float, k_descale: float,
            v_descale: float, causal: bool = False, scale: float | None = None, out: torch.Tensor | None = None,
            lse: torch.Tensor | None = None):
    """Fused exact attention forward on e4m3 inputs.

    q [B,Nq,Hq,D], k [B,Nk,Hkv,D], v [B,Nk,Hkv,D] CUDA tensors of e4m3 bytes
    (torch.float8_e4m3fn or uint8); the represented values are descale * e4m3.
    Returns (o [B,Nq,Hq,D] bf16, lse [B,Hq,Nq] fp32).  D must be 128.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if t.dtype not in (torch.float8_e4m3fn, torch.uint8):
            raise TypeError(f"{n} must hold e4m3 bytes (float8_e4m3fn or uint8), got {t.dtype}")
        _need(t, n, t.dtype, 4)
    B, Nq, Hq, D = q.shape
    Bk, Nk, Hkv, Dk = k.shape
    if Bk != B or Dk != D or tuple(v.shape) != (B, Nk, Hkv, D):
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((B, Nq, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    with torch.cuda.device(q.device):
        rc = library().attn_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), float(q_descale), float(k_descale),
                                    float(v_descale), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, Nk, D,
                                    int(bool(causal)), float(scale), _stream_handle(q.device))
    _check(rc, "attn_fwd_fp8")
    return out, lse


def bwd_workspace_size(B: int, Hq: int, Nq: int, D: int) -> int:
    return int(library().attn_bwd_workspace_size(B, Hq, Nq, D))


def bwd_head_group(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, D: int, causal: bool, sm_count: int) -> int:
    """(batch, KV head) pairs per group in bwd's unit order for this shape
    on a device with sm_count SMs (host-only; 0 for rejected arguments)."""
    return int(library().attn_bwd_head_group(B, Hq, Hkv, Nq, Nk, D, int(bool(causal)), sm_count))


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor, dout: torch.Tensor,
        causal: bool = False, scale: float | None = None, dq: torch.Tensor | None = None,
        dk: torch.Tensor | None = None, dv: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """Gradients of ``fwd`` with respect to q, k, v for the upstream gradient dout.

    q, o, dout [B,Nq,Hq,D]; k, v [B,Nk,Hkv,D] bf16; lse [B,Hq,Nq] fp32 from
    ``fwd`` on the same inputs.  Returns (dq, dk, dv) bf16 with the shapes of
    q, k, v.  Runs on torch's current stream of q's device.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, n, torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    B, Nq, Hq, D = q.shape
    _, Nk, Hkv, _ = k.shape
    Dv = v.shape[3]
    if (tuple(k.shape) != (B, Nk, Hkv, D) or tuple(v.shape[:3]) != (B, Nk, Hkv) or o.shape != dout.shape
            or tuple(o.shape) != (B, Nq, Hq, Dv) or tuple(lse.shape) != (B, Hq, Nq)):
        raise ValueError("shape mismatch")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n, ref in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
        _need(t, n, torch.bfloat16, 4)
        if t.shape != ref.shape:
            raise ValueError(f"{n} shape mismatch")
    need = bwd_workspace_size(B, Hq, Nq, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        rc = library().attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                                lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Nq, Nk,
                                D, Dv, int(bool(causal)), float(scale), workspace.data_ptr(), workspace.numel(),
                                _stream_handle(q.device))
    _check(rc, "attn_bwd")
    return dq, dk, dv


def _device_index(device) -> int:
    if device is None:
        return torch.cuda.current_device()
    if isinstance(device, int):
        return device
    d = torch.device(device)
    return d.index if d.index is not None else torch.cuda.current_device()


def decode_workspace_size(B: int, Hq: int, Dv: int, device=None) -> int:
    """Workspace bytes of decode_paged on `device` (0: unsupported shape or device)."""
    return int(library().attn_decode_paged_workspace_size(B, Hq, Dv, _device_index(device)))


def decode_paged(q: torch.Tensor, kv_pages: torch.Tensor, block_table: torch.Tensor, cache_seqlens: torch.Tensor,
                 scale: float, dv: int = 512, out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None):
    """Paged MLA (MQA-absorb) decode, one query token per sequence.

    q [B,1,Hq,Dk] bf16; kv_pages [num_pages,page_size,1,Dk] bf16;
    block_table [B,max_pages] int32; cache_seqlens [B] int32.
    Returns (o [B,1,Hq,dv] bf16, lse [B,Hq] fp32).
    """
    _need(q, "q", torch.bfloat16, 4)
    _need(kv_pages, "kv_pages", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    B, sq, Hq, Dk = q.shape
    num_pages, page_size, hkv, Dk2 = kv_pages.shape
    if sq != 1 or hkv != 1 or Dk2 != Dk or block_table.shape[0] != B or cache_seqlens.shape[0] != B:
        raise ValueError("decode_paged shape mismatch")
    if out is None:
        out = torch.empty((B, 1, Hq, dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 2)
    with torch.cuda.device(q.device):
        need = int(library().attn_decode_paged_workspace_size(B, Hq, dv, q.device.index))
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
        if not workspace.is_cuda or workspace.numel() * workspace.element_size() < need:
            raise ValueError("workspace too small")
        rc = library().attn_decode_paged(q.data_ptr(), kv_pages.data_ptr(), block_table.data_ptr(),
                                         cache_seqlens.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Dk, dv,
                                         page_size, num_pages, block_table.shape[1], float(scale),
                                         workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                         _stream_handle(q.device))
    _check(rc, "attn_decode_paged")
    return out, lse


def decode_mtp_workspace_size(B: int, s_q: int, Hq: int, Dv: int, device=None) -> int:
    """Workspace bytes of decode_paged_mtp on `device` (0: unsupported shape or device)."""
    return int(library().attn_decode_paged_mtp_workspace_size(B, s_q, Hq, Dv, _device_index(device)))


def decode_paged_mtp(q: torch.Tensor, kv_pages: torch.Tensor, block_table: torch.Tensor, cache_seqlens: torch.Tensor,
                     scale: float, dv: int = 512, out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None):
    """Paged MLA decode with s_q query tokens per sequence (the last s_q cached
    tokens; token i sees positions 0 .. L - s_q + i).

    q [B,s_q,Hq,Dk] bf16; kv_pages [num_pages,page_size,1,Dk] bf16;
    block_table [B,max_pages] int32; cache_seqlens [B] int32.
    Returns (o [B,s_q,Hq,dv] bf16, lse [B,s_q,Hq] fp32).
    """
    _need(q, "q", torch.bfloat16, 4)
    _need(kv_pages, "kv_pages", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    B, sq, Hq, Dk = q.shape
    num_pages, page_size, hkv, Dk2 = kv_pages.shape
    if hkv != 1 or Dk2 != Dk or block_table.shape[0] != B or cache_seqlens.shape[0] != B:
        raise ValueError("decode_paged_mtp shape mismatch")
    if out is None:
        out = torch.empty((B, sq, Hq, dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, sq, Hq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    with torch.cuda.device(q.device):
        need = int(library().attn_decode_paged_mtp_workspace_size(B, sq, Hq, dv, q.device.index))
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
        if not workspace.is_cuda or workspace.numel() * workspace.element_size() < need:
            raise ValueError("workspace too small")
        rc = library().attn_decode_paged_mtp(q.data_ptr(), kv_pages.data_ptr(), block_table.data_ptr(),
                                             cache_seqlens.data_ptr(), out.data_ptr(), lse.data_ptr(), B, sq, Hq, Dk,
                                             dv, page_size, num_pages, block_table.shape[1], float(scale),
                                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                             _stream_handle(q.device))
    _check(rc, "attn_decode_paged_mtp")
    return out, lse


def decode_paged_noalloc(q: torch.Tensor, kv_pages: torch.Tensor, block_table: torch.Tensor,
                         cache_seqlens: torch.Tensor, scale: float, dv: int = 512, out: torch.Tensor | None = None,
                         lse: torch.Tensor | None = None):
    """decode_paged for callers that cannot allocate a workspace: the library
    uses its own fixed scratch array (shared by all calls; calls that overlap
    on the GPU race).  Outputs are allocated here only when not given."""
    _need(q, "q", torch.bfloat16, 4)
    _need(kv_pages, "kv_pages", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    B, sq, Hq, Dk = q.shape
    num_pages, page_size, hkv, Dk2 = kv_pages.shape
    if sq != 1 or hkv != 1 or Dk2 != Dk or block_table.shape[0] != B or cache_seqlens.shape[0] != B:
        raise ValueError("decode_paged_noalloc shape mismatch")
    if out is None:
        out = torch.empty((B, 1, Hq, dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 2)
    with torch.cuda.device(q.device):
        rc = library().attn_decode_paged_noalloc(q.data_ptr(), kv_pages.data_ptr(), block_table.data_ptr(),
                                                 cache_seqlens.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq,
                                                 Dk, dv, page_size, num_pages, block_table.shape[1], float(scale),
                                                 _stream_handle(q.device))
    _check(rc, "attn_decode_paged_noalloc")
    return out, lse


def decode_gqa_workspace_size(B: int, Hq: int, Hkv: int, D: int, device=None) -> int:
    """Workspace bytes of decode_paged_gqa on `device` (0: unsupported shape or device)."""
    return int(library().attn_decode_paged_gqa_workspace_size(B, Hq, Hkv, D, _device_index(device)))


def decode_paged_gqa(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, block_table: torch.Tensor,
                     cache_seqlens: torch.Tensor, scale: float, out: torch.Tensor | None = None,
                     lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """GQA-path paged decode, one query token per sequence.

    q [B,1,Hq,D] bf16; k_pages, v_pages [num_pages,page_size,Hkv,D] bf16;
    block_table [B,max_pages] int32; cache_seqlens [B] int32.
    Returns (o [B,1,Hq,D] bf16, lse [B,Hq] fp32).
    """
    _need(q, "q", torch.bfloat16, 4)
    _need(k_pages, "k_pages", torch.bfloat16, 4)
    _need(v_pages, "v_pages", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    B, sq, Hq, D = q.shape
    num_pages, page_size, Hkv, D2 = k_pages.shape
    if (sq != 1 or D2 != D or tuple(v_pages.shape) != tuple(k_pages.shape) or block_table.shape[0] != B
            or cache_seqlens.shape[0] != B):
        raise ValueError("decode_paged_gqa shape mismatch")
    if out is None:
        out = torch.empty((B, 1, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 2)
    with torch.cuda.device(q.device):
        need = int(library().attn_decode_paged_gqa_workspace_size(B, Hq, Hkv, D, q.device.index))
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
        if not workspace.is_cuda or workspace.numel() * workspace.element_size() < need:
            raise ValueError("workspace too small")
        rc = library().attn_decode_paged_gqa(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                             block_table.data_ptr(), cache_seqlens.data_ptr(), out.data_ptr(),
                                             lse.data_ptr(), B, Hq, Hkv, D, page_size, num_pages,
                                             block_table.shape[1], float(scale), workspace.data_ptr(),
                                             workspace.numel() * workspace.element_size(),
                                             _stream_handle(q.device))
    _check(rc, "attn_decode_paged_gqa")
    return out, lse


def read_device_status(device: int = 0) -> int:
    """Status recorded by kernels on `device` (0 = ATTN_OK); resets it."""
    return int(library().attn_read_device_status(device))
