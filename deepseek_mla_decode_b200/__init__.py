"""B200-native weight-absorbed MLA decode.

Thin Python binding over the C ABI of ``libmla.so`` (``include/mla_decode.h``): it only
marshals torch tensors into pointers, sizes and the current CUDA stream.  Every step of
the computation runs in the library's CUDA kernels; there is no fallback path, and a
missing or unbuildable library raises ``RuntimeError``.

    meta = get_metadata(cache_seqlens, s_q, H)
    out, lse = decode(q_nope, q_pe, kv_cache, block_table, cache_seqlens,
                      softmax_scale, causal, meta)
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("MLA_LIBRARY") or os.path.join(_HERE, "libmla.so")

MLA_DEVICE_ERR_BLOCK_ID = 1
MLA_DEVICE_ERR_SEQLEN = 2
MLA_DEVICE_ERR_TIMEOUT = 4
MLA_DEVICE_ERR_METADATA = 8

EXPORTED_SYMBOLS = (
    "mla_status_string",
    "mla_metadata_size",
    "mla_get_metadata",
    "mla_workspace_size",
    "mla_decode",
    "mla_decode_ragged",
    "mla_decode_attention",
    "mla_decode_combine",
    "mla_decode_noalloc",
    "mla_device_sm_count",
    "mla_set_wait_timeout_ns",
    "mla_set_stall_injection",
    "mla_absorb_q",
    "mla_absorb_out",
    "mla_quantize_kv_fp8",
    "mla_decode_fp8",
    "mla_decode_fp8_attention",
    "mla_sage_workspace_size",
    "mla_sage_quantize",
    "mla_sage_attention",
    "mla_sage_prefill",
    "mla_get_metadata_tokens",
    "mla_decode_tokens",
    "mla_decode_fp8_tokens",
)

_lib = None


class MLAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmla.so (building it first if sources are newer) and declare signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path) or path == os.path.join(_HERE, "libmla.so"):
        try:
            from . import build as _build

            _build.build()
        except Exception as e:  # pragma: no cover - build errors are reported loudly
            if not os.path.exists(path):
                raise RuntimeError(f"libmla.so is missing and could not be built: {e}") from e
    L = ctypes.CDLL(path)
    c_int, c_size, c_vp, c_i64, c_f = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
    L.mla_status_string.restype = ctypes.c_char_p
    L.mla_status_string.argtypes = [c_int]
    L.mla_metadata_size.restype = c_int
    L.mla_metadata_size.argtypes = [c_int, c_int, c_int, ctypes.POINTER(c_size)]
    L.mla_workspace_size.restype = c_int
    L.mla_workspace_size.argtypes = [c_int, c_int, c_int, ctypes.POINTER(c_size)]
    L.mla_device_sm_count.restype = c_int
    L.mla_device_sm_count.argtypes = [ctypes.POINTER(c_int)]
    L.mla_set_wait_timeout_ns.restype = c_int
    L.mla_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    L.mla_set_stall_injection.restype = c_int
    L.mla_set_stall_injection.argtypes = [c_int]
    L.mla_get_metadata.restype = c_int
    L.mla_get_metadata.argtypes = [c_vp, c_int, c_int, c_int, c_vp, c_size, c_vp]
    dec_args = [c_vp, c_vp, c_vp, c_i64, c_vp, c_int, c_vp, c_int, c_int, c_int, c_f, c_int,
                c_vp, c_size, c_vp, c_size, c_vp, c_vp, c_vp, c_vp]
    for fn in (L.mla_decode, L.mla_decode_attention):
        fn.restype = c_int
        fn.argtypes = dec_args
    L.mla_get_metadata_tokens.restype = c_int
    L.mla_get_metadata_tokens.argtypes = [c_vp, c_vp, c_int, c_int, c_int, c_int, c_vp, c_size, c_vp]
    for fn in (L.mla_decode_ragged, L.mla_decode_fp8, L.mla_decode_fp8_attention, L.mla_decode_tokens,
               L.mla_decode_fp8_tokens):
        fn.restype = c_int
        fn.argtypes = dec_args[:7] + [c_vp] + dec_args[7:]
    for fn in (L.mla_absorb_q, L.mla_absorb_out):
        fn.restype = c_int
        fn.argtypes = [c_vp, c_vp, c_vp, c_int, c_int, c_vp]
    L.mla_quantize_kv_fp8.restype = c_int
    L.mla_quantize_kv_fp8.argtypes = [c_vp, c_vp, c_i64, c_vp]
    L.mla_sage_workspace_size.restype = c_int
    L.mla_sage_workspace_size.argtypes = [c_int, c_int, ctypes.POINTER(c_size)]
    L.mla_sage_quantize.restype = c_int
    L.mla_sage_quantize.argtypes = [c_vp, c_vp, c_vp, c_int, c_int, c_vp, c_size, c_vp]
    L.mla_sage_attention.restype = c_int
    L.mla_sage_attention.argtypes = [c_int, c_int, c_f, c_vp, c_size, c_vp, c_vp, c_vp, c_vp]
    L.mla_sage_prefill.restype = c_int
    L.mla_sage_prefill.argtypes = [c_vp, c_vp, c_vp, c_int, c_int, c_f, c_vp, c_size, c_vp, c_vp, c_vp, c_vp]
    L.mla_decode_noalloc.restype = c_int
    L.mla_decode_noalloc.argtypes = [c_vp, c_vp, c_vp, c_i64, c_vp, c_int, c_vp, c_int, c_int, c_int, c_f, c_int,
                                     c_vp, c_size, c_vp, c_vp, c_vp, c_vp]
    L.mla_decode_combine.restype = c_int
    L.mla_decode_combine.argtypes = [c_vp, c_int, c_int, c_int, c_int, c_vp, c_size, c_vp, c_size, c_vp, c_vp,
                                     c_vp, c_vp]
    _lib = L
    return L


def status_string(code: int) -> str:
    return load_library().mla_status_string(code).decode()


def _check(fn: str, code: int):
    if code != 0:
        raise MLAError(fn, code)


def metadata_size(B: int, s_q: int, H: int) -> int:
    n = ctypes.c_size_t()
    _check("mla_metadata_size", load_library().mla_metadata_size(B, s_q, H, ctypes.byref(n)))
    return n.value


def workspace_size(B: int, s_q: int, H: int) -> int:
    n = ctypes.c_size_t()
    _check("mla_workspace_size", load_library().mla_workspace_size(B, s_q, H, ctypes.byref(n)))
    return n.value


def device_sm_count() -> int:
    n = ctypes.c_int()
    _check("mla_device_sm_count", load_library().mla_device_sm_count(ctypes.byref(n)))
    return n.value


def set_wait_timeout_ns(ns: int) -> None:
    """Bound on the attention kernel's internal waits for later launches (0 = the
    default 1 s); see mla_set_wait_timeout_ns."""
    _check("mla_set_wait_timeout_ns", load_library().mla_set_wait_timeout_ns(int(ns)))


def set_stall_injection(enable: bool) -> None:
    """Test hook: make later launches' MMA warp wait on a barrier nothing completes,
    so the bounded waits run out (see mla_set_stall_injection)."""
    _check("mla_set_stall_injection", load_library().mla_set_stall_injection(int(bool(enable))))


def _stream_ptr(stream) -> int:
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def get_metadata(cache_seqlens, s_q: int, H: int, metadata=None, stream=None):
    """Split-KV schedule for one decode step (device int32 buffer)."""
    import torch

    B = cache_seqlens.shape[0]
    nbytes = metadata_size(B, s_q, H)
    if metadata is None:
        metadata = torch.empty((nbytes + 3) // 4, dtype=torch.int32, device=cache_seqlens.device)
    _check("mla_get_metadata", load_library().mla_get_metadata(
        cache_seqlens.data_ptr(), B, s_q, H, metadata.data_ptr(), metadata.numel() * metadata.element_size(),
        _stream_ptr(stream)))
    return metadata


def _decode_args(q_nope, q_pe, kv_cache, block_table, cache_seqlens, softmax_scale, causal, metadata, workspace,
                 out, lse, status, stream):
    B, s_q, H, _ = q_nope.shape
    for name, t in (("q_nope", q_nope), ("q_pe", q_pe), ("kv_cache", kv_cache), ("block_table", block_table),
                    ("cache_seqlens", cache_seqlens), ("out", out), ("lse", lse)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    return (q_nope.data_ptr(), q_pe.data_ptr(), kv_cache.data_ptr(), kv_cache.shape[0], block_table.data_ptr(),
            block_table.shape[1], cache_seqlens.data_ptr(), B, s_q, H, float(softmax_scale), int(bool(causal)),
            metadata.data_ptr(), metadata.numel() * metadata.element_size(), workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), out.data_ptr(), lse.data_ptr(),
            status.data_ptr() if status is not None else None, _stream_ptr(stream))


def _alloc_outputs(q_nope, workspace, out, lse):
    import torch

    B, s_q, H, _ = q_nope.shape
    if workspace is None:
        workspace = torch.empty(workspace_size(B, s_q, H), dtype=torch.uint8, device=q_nope.device)
    if out is None:
        out = torch.empty((B, s_q, H, 512), dtype=torch.bfloat16, device=q_nope.device)
    if lse is None:
        lse = torch.empty((B, s_q, H), dtype=torch.float32, device=q_nope.device)
    return workspace, out, lse


def decode(q_nope, q_pe, kv_cache, block_table, cache_seqlens, softmax_scale: float, causal: bool, metadata,
           workspace=None, out=None, lse=None, status=None, stream=None) -> Tuple[object, object]:
    """Weight-absorbed MLA decode; returns (out bf16 [B, s_q, H, 512], lse fp32 [B, s_q, H])."""
    workspace, out, lse = _alloc_outputs(q_nope, workspace, out, lse)
    _check("mla_decode", load_library().mla_decode(
        *_decode_args(q_nope, q_pe, kv_cache, block_table, cache_seqlens, softmax_scale, causal, metadata,
                      workspace, out, lse, status, stream)))
    return out, lse


def decode_ragged(q_nope, q_pe, kv_cache, block_table, cache_seqlens, q_lens, softmax_scale: float, causal: bool,
                  metadata, workspace=None, out=None, lse=None, status=None, stream=None) -> Tuple[object, object]:
    """mla_decode_ragged: the decode with q_lens[b] <= s_q query tokens for sequence b
    (padding tokens give out 0, lse -inf)."""
    workspace, out, lse = _alloc_outputs(q_nope, workspace, out, lse)
    if not q_lens.is_contiguous():
        raise ValueError("q_lens must be contiguous")
    args = _decode_args(q_nope, q_pe, kv_cache, block_table, cache_seqlens, softmax_scale, causal, metadata,
                        workspace, out, lse, status, stream)
    _check("mla_decode_ragged", load_library().mla_decode_ragged(*args[:7], q_lens.data_ptr(), *args[7:]))
    return out, lse


def decode_fp8(q_nope, q_pe, kv_fp8, block_table, cache_seqlens, softmax_scale: float, causal: bool, metadata,
               q_lens=None, workspace=None, out=None, lse=None, status=None, stream=None) -> Tuple[object, object]:
    """mla_decode_fp8: the decode over a packed FP8 cache [num_blocks, 64, 656] (uint8,
    as written by quantize_kv_fp8); q_lens as in decode_ragged, or None."""
    if kv_fp8.shape[-1] != 656:
        raise ValueError("packed FP8 cache [num_blocks, 64, 656] expected")
    workspace, out, lse = _alloc_outputs(q_nope, workspace, out, lse)
    if q_lens is not None and not q_lens.is_contiguous():
        raise ValueError("q_lens must be contiguous")
    args = _decode_args(q_nope, q_pe, kv_fp8, block_table, cache_seqlens, softmax_scale, causal, metadata,
                        workspace, out, lse, status, stream)
    _check("mla_decode_fp8", load_library().mla_decode_fp8(*args[:7], q_lens.data_ptr() if q_lens is not None
                                                           else None, *args[7:]))
    return out, lse


def get_metadata_tokens(cache_seqlens, q_lens, s_q: int, H: int, causal: bool, metadata=None, stream=None):
    """mla_get_metadata_tokens: the token schedule (an s_q = 1 schedule over B * s_q
    token sequences) for decode_tokens / decode_fp8_tokens; q_lens may be None."""
    import torch

    B = cache_seqlens.shape[0]
    nbytes = metadata_size(B * s_q, 1, H)
    if metadata is None:
        metadata = torch.empty((nbytes + 3) // 4, dtype=torch.int32, device=cache_seqlens.device)
    if q_lens is not None and not q_lens.is_contiguous():
        raise ValueError("q_lens must be contiguous")
    _check("mla_get_metadata_tokens", load_library().mla_get_metadata_tokens(
        cache_seqlens.data_ptr(), q_lens.data_ptr() if q_lens is not None else None, B, s_q, H, int(bool(causal)),
        metadata.data_ptr(), metadata.numel() * metadata.element_size(), _stream_ptr(stream)))
    return metadata


def _decode_tokens(fn, q_nope, q_pe, kv, block_table, cache_seqlens, q_lens, softmax_scale, causal, metadata,
                   workspace, out, lse, status, stream):
    import torch

    B, s_q, H, _ = q_nope.shape
    if workspace is None:
        workspace = torch.empty(workspace_size(B * s_q, 1, H), dtype=torch.uint8, device=q_nope.device)
    _, out, lse = _alloc_outputs(q_nope, workspace, out, lse)
    if q_lens is not None and not q_lens.is_contiguous():
        raise ValueError("q_lens must be contiguous")
    args = _decode_args(q_nope, q_pe, kv, block_table, cache_seqlens, softmax_scale, causal, metadata, workspace,
                        out, lse, status, stream)
    qptr = q_lens.data_ptr() if q_lens is not None else None
    _check(fn, getattr(load_library(), fn)(*args[:7], qptr, *args[7:]))
    return out, lse


def decode_tokens(q_nope, q_pe, kv_cache, block_table, cache_seqlens, q_lens, softmax_scale: float, causal: bool,
                  metadata, workspace=None, out=None, lse=None, status=None, stream=None) -> Tuple[object, object]:
    """mla_decode_tokens: decode_ragged balanced by the token schedule (metadata from
    get_metadata_tokens with the same q_lens and causal flag)."""
    return _decode_tokens("mla_decode_tokens", q_nope, q_pe, kv_cache, block_table, cache_seqlens, q_lens,
                          softmax_scale, causal, metadata, workspace, out, lse, status, stream)


def decode_fp8_tokens(q_nope, q_pe, kv_fp8, block_table, cache_seqlens, q_lens, softmax_scale: float, causal: bool,
                      metadata, workspace=None, out=None, lse=None, status=None, stream=None) -> Tuple[object, object]:
    """mla_decode_fp8_tokens: decode_fp8 with the token schedule."""
    if kv_fp8.shape[-1] != 656:
        raise ValueError("packed FP8 cache [num_blocks, 64, 656] expected")
    return _decode_tokens("mla_decode_fp8_tokens", q_nope, q_pe, kv_fp8, block_table, cache_seqlens, q_lens,
                          softmax_scale, causal, metadata, workspace, out, lse, status, stream)


def decode_fp8_attention(q_nope, q_pe, kv_fp8, block_table, cache_seqlens, softmax_scale: float, causal: bool,
                         metadata, workspace, out, lse, q_lens=None, status=None, stream=None):
    """The FP8 split-KV attention launch alone (see mla_decode_fp8_attention)."""
    args = _decode_args(q_nope, q_pe, kv_fp8, block_table, cache_seqlens, softmax_scale, causal, metadata,
                        workspace, out, lse, status, stream)
    _check("mla_decode_fp8_attention", load_library().mla_decode_fp8_attention(
        *args[:7], q_lens.data_ptr() if q_lens is not None else None, *args[7:]))


def sage_workspace_size(S: int, H: int) -> int:
    n = ctypes.c_size_t()
    _check("mla_sage_workspace_size", load_library().mla_sage_workspace_size(S, H, ctypes.byref(n)))
    return n.value


def _sage_check(q, k, v):
    S, H, dq = q.shape
    if dq != 192 or tuple(k.shape) != (S, H, 192) or tuple(v.shape) != (S, H, 128):
        raise ValueError("q, k [S, H, 192] and v [S, H, 128] expected")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    return S, H


def sage_quantize(q, k, v, workspace=None, stream=None):
    """mla_sage_quantize: the INT8 / FP8 codes and scales of q, k, v in a workspace
    (uint8 tensor; layout in include/mla_decode.h)."""
    import torch

    S, H = _sage_check(q, k, v)
    if workspace is None:
        workspace = torch.empty(sage_workspace_size(S, H), dtype=torch.uint8, device=q.device)
    _check("mla_sage_quantize", load_library().mla_sage_quantize(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), S, H, workspace.data_ptr(), workspace.numel(), _stream_ptr(stream)))
    return workspace


def sage_attention(S: int, H: int, softmax_scale: float, workspace, out=None, lse=None, status=None, stream=None):
    """mla_sage_attention over a filled workspace; returns (out bf16 [S, H, 128], lse fp32 [S, H])."""
    import torch

    if out is None:
        out = torch.empty((S, H, 128), dtype=torch.bfloat16, device=workspace.device)
    if lse is None:
        lse = torch.empty((S, H), dtype=torch.float32, device=workspace.device)
    _check("mla_sage_attention", load_library().mla_sage_attention(
        S, H, float(softmax_scale), workspace.data_ptr(), workspace.numel(), out.data_ptr(), lse.data_ptr(),
        status.data_ptr() if status is not None else None, _stream_ptr(stream)))
    return out, lse


def sage_prefill(q, k, v, softmax_scale: float, workspace=None, out=None, lse=None, status=None, stream=None):
    """mla_sage_prefill: quantised causal prefill attention (q, k [S, H, 192], v [S, H, 128],
    bf16); returns (out bf16 [S, H, 128], lse fp32 [S, H])."""
    import torch

    S, H = _sage_check(q, k, v)
    if workspace is None:
        workspace = torch.empty(sage_workspace_size(S, H), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((S, H, 128), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((S, H), dtype=torch.float32, device=q.device)
    _check("mla_sage_prefill", load_library().mla_sage_prefill(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), S, H, float(softmax_scale), workspace.data_ptr(), workspace.numel(),
        out.data_ptr(), lse.data_ptr(), status.data_ptr() if status is not None else None, _stream_ptr(stream)))
    return out, lse


def absorb_q(q_heads, w_uk, q_nope=None, stream=None):
    """mla_absorb_q: q_nope[..., h, :] = W_UK[h]^T q_heads[..., h, :] for q_heads
    [B, s_q, H, 128] and w_uk [H, 128, 512]; returns q_nope [B, s_q, H, 512] (bf16)."""
    import torch

    *lead, H, d = q_heads.shape
    if d != 128 or tuple(w_uk.shape) != (H, 128, 512):
        raise ValueError("q_heads [..., H, 128] and w_uk [H, 128, 512] expected")
    if not (q_heads.is_contiguous() and w_uk.is_contiguous()):
        raise ValueError("inputs must be contiguous")
    R = q_heads.numel() // (H * 128)
    if q_nope is None:
        q_nope = torch.empty((*lead, H, 512), dtype=torch.bfloat16, device=q_heads.device)
    _check("mla_absorb_q", load_library().mla_absorb_q(q_heads.data_ptr(), w_uk.data_ptr(), q_nope.data_ptr(), R, H,
                                                       _stream_ptr(stream)))
    return q_nope


def absorb_out(o_latent, w_uv, y=None, stream=None):
    """mla_absorb_out: y[..., h, :] = W_UV[h] o_latent[..., h, :] for o_latent
    [B, s_q, H, 512] and w_uv [H, 128, 512]; returns y [B, s_q, H, 128] (bf16)."""
    import torch

    *lead, H, d = o_latent.shape
    if d != 512 or tuple(w_uv.shape) != (H, 128, 512):
        raise ValueError("o_latent [..., H, 512] and w_uv [H, 128, 512] expected")
    if not (o_latent.is_contiguous() and w_uv.is_contiguous()):
        raise ValueError("inputs must be contiguous")
    R = o_latent.numel() // (H * 512)
    if y is None:
        y = torch.empty((*lead, H, 128), dtype=torch.bfloat16, device=o_latent.device)
    _check("mla_absorb_out", load_library().mla_absorb_out(o_latent.data_ptr(), w_uv.data_ptr(), y.data_ptr(), R, H,
                                                           _stream_ptr(stream)))
    return y


def quantize_kv_fp8(kv_cache, kv_fp8=None, stream=None):
    """mla_quantize_kv_fp8: bf16 cache [num_blocks, 64, 576] -> packed FP8 rows
    [num_blocks, 64, 656] (uint8)."""
    import torch

    if kv_cache.shape[-1] != 576 or not kv_cache.is_contiguous():
        raise ValueError("contiguous [..., 576] bf16 cache expected")
    rows = kv_cache.numel() // 576
    if kv_fp8 is None:
        kv_fp8 = torch.empty((*kv_cache.shape[:-1], 656), dtype=torch.uint8, device=kv_cache.device)
    _check("mla_quantize_kv_fp8", load_library().mla_quantize_kv_fp8(kv_cache.data_ptr(), kv_fp8.data_ptr(), rows,
                                                                     _stream_ptr(stream)))
    return kv_fp8


def decode_attention(q_nope, q_pe, kv_cache, block_table, cache_seqlens, softmax_scale: float, causal: bool,
                     metadata, workspace, out, lse, status=None, stream=None):
    """The split-KV attention launch alone (see mla_decode_attention)."""
    _check("mla_decode_attention", load_library().mla_decode_attention(
        *_decode_args(q_nope, q_pe, kv_cache, block_table, cache_seqlens, softmax_scale, causal, metadata,
                      workspace, out, lse, status, stream)))


def decode_combine(cache_seqlens, max_blocks: int, s_q: int, H: int, metadata, workspace, out, lse, status=None,
                   stream=None):
    """The LSE-combine launch alone (see mla_decode_combine)."""
    B = cache_seqlens.shape[0]
    _check("mla_decode_combine", load_library().mla_decode_combine(
        cache_seqlens.data_ptr(), int(max_blocks), B, s_q, H, metadata.data_ptr(),
        metadata.numel() * metadata.element_size(), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
        out.data_ptr(), lse.data_ptr(), status.data_ptr() if status is not None else None, _stream_ptr(stream)))


def decode_noalloc(q_nope, q_pe, kv_cache, block_table, cache_seqlens, softmax_scale: float, causal: bool,
                   metadata, out, lse, status=None, stream=None):
    """mla_decode_noalloc: the decode with the library's built-in 64 MiB scratch instead
    of a workspace, for callers that cannot allocate device memory.  ``out`` and ``lse``
    are caller-provided.  Raises MLAError(code 4) when the shape needs more scratch."""
    args = _decode_args(q_nope, q_pe, kv_cache, block_table, cache_seqlens, softmax_scale, causal, metadata,
                        metadata, out, lse, status, stream)
    # drop the workspace pointer / size (positions 14, 15) from the mla_decode argument list
    args = args[:14] + args[16:]
    _check("mla_decode_noalloc", load_library().mla_decode_noalloc(*args))
    return out, lse
