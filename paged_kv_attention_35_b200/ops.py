"""ctypes binding over ``libpagedattn.so`` -- argument marshalling only.

Every computation runs in the library's CUDA kernels; this module only turns
torch tensors into pointers, sizes and the current CUDA stream, allocates the
outputs (and the decode workspace) when the caller does not pass them, and
turns a non-OK status into ``RuntimeError``.  There is no fallback: importing
this module raises if the library is not built, and every call requires CUDA
tensors.  Names and semantics follow ``include/pagedattn.h``.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m paged_kv_attention_35_b200.build` (there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

PA_OK = 0
PA_BF16 = 0
FLAG_SLOT_OOB, FLAG_BLOCK_OOB, FLAG_LEN_OOB, FLAG_TIMEOUT, FLAG_SLOT_MISMATCH = 1, 2, 4, 8, 16
STATUS = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_WORKSPACE",
          4: "PA_ERR_CUDA"}

_p, _i32, _i64, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t

SIGNATURES = {
    "pa_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "pa_last_error_message": ([], ctypes.c_char_p),
    "pa_version": ([], ctypes.c_char_p),
    "pa_store_kvcache": ([_p, _p, _i64, _i64, _p, _p, _p, _i32, _i32, _i32, _i64, ctypes.c_int, _p, _p],
                         ctypes.c_int),
    "pa_decode_workspace_size": ([_i32, _i32, _i32, _i32, _i32, _i32], _sz),
    "pa_decode": ([_p, _p, _i64, _p, _p, _p, _i32, _p, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                   _f32, _i32, _p, _sz, ctypes.c_int, _p, _p], ctypes.c_int),
    "pa_decode_store": ([_p, _p, _i64, _p, _p, _i64, _i64, _p, _p, _p, _p, _i32, _p, _i32, _i32,
                         _i32, _i32, _i32, _i32, _i32, _f32, _i32, _p, _sz, ctypes.c_int, _p, _p],
                        ctypes.c_int),
    "pa_decode_noalloc": ([_p, _p, _i64, _p, _p, _p, _i32, _p, _i32, _i32, _i32, _i32, _i32, _i32,
                           _i32, _f32, _i32, ctypes.c_int, _p, _p], ctypes.c_int),
    "pa_prefill_varlen": ([_p, _p, _i64, _p, _p, _p, _p, _i32, _i32, _i32, _p, _i32, _i32, _i32, _i32,
                           _i32, _i32, _i32, _f32, ctypes.c_int, _p, _p], ctypes.c_int),
    "pa_prefill_store": ([_p, _p, _i64, _p, _p, _i64, _i64, _p, _p, _p, _p, _p, _i32, _i32, _i32,
                          _p, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32, ctypes.c_int, _p, _p],
                         ctypes.c_int),
    "pa_watchdog_read": ([ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
    "pa_selftest_wait_timeout": ([_p, ctypes.c_uint32, _p, _p], ctypes.c_int),
}
for _name, (_args, _res) in SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


def lib():
    return _lib


def version() -> str:
    return _lib.pa_version().decode()


def _check(status: int, what: str) -> None:
    if status != PA_OK:
        msg = _lib.pa_last_error_message().decode()
        raise RuntimeError(f"{what}: {_lib.pa_status_string(status).decode()}: {msg}")


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _need_cuda(**tensors) -> None:
    for name, t in tensors.items():
        if t is None:
            continue
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor (no CPU path)")


def _need_bf16(**tensors) -> None:
    for name, t in tensors.items():
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")


def _need_i32(**tensors) -> None:
    for name, t in tensors.items():
        if t.dtype != torch.int32 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous int32 tensor")


def _token_stride(t: torch.Tensor, name: str) -> int:
    """Rows of [N, H, D] may be strided; each row's H*D elements must be contiguous."""
    if t.dim() != 3:
        raise ValueError(f"{name} must be [N, H, D]")
    if t.stride(2) != 1 or t.stride(1) != t.shape[2]:
        raise ValueError(f"{name}: heads and head_dim must be contiguous within a token row")
    return t.stride(0)


def store_kvcache(key, value, k_cache, v_cache, slot_mapping, err_flag=None) -> None:
    """Scatter key/value [N, Hkv, D] into the pools [NB, bs, Hkv, D] at slot_mapping [N]."""
    _need_cuda(key=key, value=value, k_cache=k_cache, v_cache=v_cache, slot_mapping=slot_mapping,
               err_flag=err_flag)
    _need_bf16(key=key, value=value, k_cache=k_cache, v_cache=v_cache)
    _need_i32(slot_mapping=slot_mapping)
    if not (k_cache.is_contiguous() and v_cache.is_contiguous()):
        raise ValueError("pools must be contiguous")
    nb, bs, hkv, d = k_cache.shape
    n = key.shape[0]
    if slot_mapping.numel() != n or value.shape[0] != n:
        raise ValueError("key/value/slot_mapping lengths differ")
    if key.shape[1:] != (hkv, d) or value.shape[1:] != (hkv, d):
        raise ValueError("key/value rows do not match the pool's [Hkv, D]")
    _check(_lib.pa_store_kvcache(_ptr(key), _ptr(value), _token_stride(key, "key"),
                                 _token_stride(value, "value"), _ptr(k_cache), _ptr(v_cache),
                                 _ptr(slot_mapping), n, hkv, d, nb * bs, PA_BF16, _ptr(err_flag),
                                 _stream()), "pa_store_kvcache")


def decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                          partition_size=0) -> int:
    return int(_lib.pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                             max_context_len, partition_size))


def decode(q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale=None, out=None,
           workspace=None, partition_size=0, err_flag=None):
    """Paged decode attention; q [B, Hq, D] -> out [B, Hq, D] (bf16)."""
    _need_cuda(q=q, k_cache=k_cache, v_cache=v_cache, block_tables=block_tables,
               context_lens=context_lens, out=out, workspace=workspace, err_flag=err_flag)
    _need_bf16(q=q, k_cache=k_cache, v_cache=v_cache)
    _need_i32(block_tables=block_tables, context_lens=context_lens)
    nb, bs, hkv, d = k_cache.shape
    B, hq, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the pool's")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, hq, d), dtype=torch.bfloat16, device=q.device)
    ws_bytes = decode_workspace_size(B, hq, hkv, d, max_context_len, partition_size)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    _check(_lib.pa_decode(_ptr(out), _ptr(q), _token_stride(q, "q"), _ptr(k_cache), _ptr(v_cache),
                          _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), B,
                          int(max_context_len), hq, hkv, d, bs, nb, float(scale),
                          int(partition_size), _ptr(workspace),
                          0 if workspace is None else workspace.numel() * workspace.element_size(),
                          PA_BF16, _ptr(err_flag), _stream()), "pa_decode")
    return out


def decode_store(q, key, value, k_cache, v_cache, slot_mapping, block_tables, context_lens,
                 max_context_len, scale=None, out=None, workspace=None, partition_size=0,
                 err_flag=None):
    """One decode step's ``store_kvcache`` and ``decode`` in one launch (``pa_decode_store``):
    key/value [B, Hkv, D] rows go to ``slot_mapping`` (the slots of each sequence's newest
    position), then q [B, Hq, D] attends -> out [B, Hq, D] (bf16)."""
    _need_cuda(q=q, key=key, value=value, k_cache=k_cache, v_cache=v_cache,
               slot_mapping=slot_mapping, block_tables=block_tables, context_lens=context_lens,
               out=out, workspace=workspace, err_flag=err_flag)
    _need_bf16(q=q, key=key, value=value, k_cache=k_cache, v_cache=v_cache)
    _need_i32(slot_mapping=slot_mapping, block_tables=block_tables, context_lens=context_lens)
    nb, bs, hkv, d = k_cache.shape
    B, hq, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the pool's")
    if key.shape[0] != B or value.shape[0] != B or slot_mapping.numel() != B:
        raise ValueError("decode_store takes one new token per sequence")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, hq, d), dtype=torch.bfloat16, device=q.device)
    ws_bytes = decode_workspace_size(B, hq, hkv, d, max_context_len, partition_size)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    _check(_lib.pa_decode_store(_ptr(out), _ptr(q), _token_stride(q, "q"), _ptr(key), _ptr(value),
                                _token_stride(key, "key"), _token_stride(value, "value"),
                                _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache),
                                _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), B,
                                int(max_context_len), hq, hkv, d, bs, nb, float(scale),
                                int(partition_size), _ptr(workspace),
                                0 if workspace is None else workspace.numel() * workspace.element_size(),
                                PA_BF16, _ptr(err_flag), _stream()), "pa_decode_store")
    return out


NOALLOC_SCRATCH_BYTES = 16 << 20


def decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale=None,
                   out=None, partition_size=0, err_flag=None):
    """``decode`` through ``pa_decode_noalloc``: the split-K scratch is the library's
    fixed 16 MiB device array, so no workspace is allocated or passed (for callers
    that cannot allocate device memory).  Calls overlapping on the GPU race on it."""
    _need_cuda(q=q, k_cache=k_cache, v_cache=v_cache, block_tables=block_tables,
               context_lens=context_lens, out=out, err_flag=err_flag)
    _need_bf16(q=q, k_cache=k_cache, v_cache=v_cache)
    _need_i32(block_tables=block_tables, context_lens=context_lens)
    nb, bs, hkv, d = k_cache.shape
    B, hq, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the pool's")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, hq, d), dtype=torch.bfloat16, device=q.device)
    _check(_lib.pa_decode_noalloc(_ptr(out), _ptr(q), _token_stride(q, "q"), _ptr(k_cache),
                                  _ptr(v_cache), _ptr(block_tables), block_tables.shape[1],
                                  _ptr(context_lens), B, int(max_context_len), hq, hkv, d, bs, nb,
                                  float(scale), int(partition_size), PA_BF16, _ptr(err_flag),
                                  _stream()), "pa_decode_noalloc")
    return out


def prefill_varlen(q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                   block_tables, scale=None, out=None, err_flag=None):
    """Causal varlen prefill over the paged pool; q [total_q, Hq, D] -> out (bf16)."""
    _need_cuda(q=q, k_cache=k_cache, v_cache=v_cache, cu_seqlens_q=cu_seqlens_q,
               cu_seqlens_k=cu_seqlens_k, block_tables=block_tables, out=out, err_flag=err_flag)
    _need_bf16(q=q, k_cache=k_cache, v_cache=v_cache)
    _need_i32(cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k, block_tables=block_tables)
    nb, bs, hkv, d = k_cache.shape
    total_q, hq, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the pool's")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((total_q, hq, d), dtype=torch.bfloat16, device=q.device)
    num_seqs = cu_seqlens_q.numel() - 1
    _check(_lib.pa_prefill_varlen(_ptr(out), _ptr(q), _token_stride(q, "q"), _ptr(k_cache),
                                  _ptr(v_cache), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                                  int(max_seqlen_q), int(max_seqlen_k), total_q, _ptr(block_tables),
                                  block_tables.shape[1], num_seqs, hq, hkv, d, bs, nb, float(scale),
                                  PA_BF16, _ptr(err_flag), _stream()), "pa_prefill_varlen")
    return out


def prefill_store(q, key, value, k_cache, v_cache, slot_mapping, cu_seqlens_q, cu_seqlens_k,
                  max_seqlen_q, max_seqlen_k, block_tables, scale=None, out=None, err_flag=None):
    """One prefill step's ``store_kvcache`` and ``prefill_varlen`` in one launch
    (``pa_prefill_store``): key/value [total_q, Hkv, D] rows go to ``slot_mapping`` while
    q [total_q, Hq, D] attends over the cached prefix in the pool and the new rows -> out."""
    _need_cuda(q=q, key=key, value=value, k_cache=k_cache, v_cache=v_cache,
               slot_mapping=slot_mapping, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k,
               block_tables=block_tables, out=out, err_flag=err_flag)
    _need_bf16(q=q, key=key, value=value, k_cache=k_cache, v_cache=v_cache)
    _need_i32(slot_mapping=slot_mapping, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k,
              block_tables=block_tables)
    nb, bs, hkv, d = k_cache.shape
    total_q, hq, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the pool's")
    if (key.shape[0] != total_q or value.shape[0] != total_q or slot_mapping.numel() != total_q
            or tuple(key.shape[1:]) != (hkv, d) or tuple(value.shape[1:]) != (hkv, d)):
        raise ValueError("prefill_store takes one key/value row and slot per query token")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((total_q, hq, d), dtype=torch.bfloat16, device=q.device)
    num_seqs = cu_seqlens_q.numel() - 1
    _check(_lib.pa_prefill_store(_ptr(out), _ptr(q), _token_stride(q, "q"), _ptr(key), _ptr(value),
                                 _token_stride(key, "key"), _token_stride(value, "value"),
                                 _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache),
                                 _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(max_seqlen_q),
                                 int(max_seqlen_k), total_q, _ptr(block_tables),
                                 block_tables.shape[1], num_seqs, hq, hkv, d, bs, nb, float(scale),
                                 PA_BF16, _ptr(err_flag), _stream()), "pa_prefill_store")
    return out


def watchdog_read() -> int:
    v = ctypes.c_uint32(0)
    _check(_lib.pa_watchdog_read(ctypes.byref(v)), "pa_watchdog_read")
    return int(v.value)


def selftest_wait_timeout(limit_us: int = 50_000, err_flag=None, waited_ns=None) -> None:
    """Health check of the failure detection (``pa_selftest_wait_timeout``): a bounded
    wait that nothing completes gives up after ``limit_us`` and reports PA_FLAG_TIMEOUT
    in ``err_flag`` (device int32) and the watchdog word; ``waited_ns`` (device int64)
    receives the time it waited."""
    _need_cuda(err_flag=err_flag, waited_ns=waited_ns)
    _check(_lib.pa_selftest_wait_timeout(_ptr(err_flag), int(limit_us), _ptr(waited_ns), _stream()),
           "pa_selftest_wait_timeout")
