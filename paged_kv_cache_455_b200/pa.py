"""Python binding of libpa.so (argument marshalling only).

Every function here takes torch tensors, checks that their shapes, dtypes and
devices agree, derives the sizes the C ABI wants, and calls the C function of
the same name on the current CUDA stream.  All computation happens in the
library's CUDA kernels; there is no fallback.  If libpa.so is missing this
module fails to import.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} not found: build it with `python -m paged_kv_cache_455_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_WORKSPACE = range(5)
PA_DTYPE_F32, PA_DTYPE_BF16, PA_DTYPE_FP8_E4M3 = 0, 1, 2
PA_DEV_BAD_SLOT, PA_DEV_BAD_BLOCK, PA_DEV_BAD_CONTEXT, PA_DEV_WAIT_TIMEOUT = 1, 2, 4, 8

# Every symbol include/pa.h declares, with its C signature.
SIGNATURES = {
    "pa_reshape_and_cache": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I64, _I, _P, _P]),
    "pa_decode_attention": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I64, _F,
                                 _I, _P, _SZ, _P, _P]),
    "pa_decode_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "pa_num_partitions": (_I, [_I, _I]),
    "pa_splitk_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "pa_decode_splitk": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I64, _F, _I,
                              _I, _I, _P, _P, _P, _P, _P]),
    "pa_splitk_reduce": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "pa_decode_attention_static": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                                        _I64, _F, _I, _P, _P]),
    "pa_copy_blocks": (_I, [_P, _P, _P, _I, _I64, _I, _I, _I, _I, _P, _P]),
    "pa_swap_blocks": (_I, [_P, _P, _I64, _P, _P, _I64, _P, _I, _I, _I, _I, _I, _P, _P]),
    "pa_prefill_attention": (_I, [_P, _P, _P, _I, _I, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I,
                                  _I, _I64, _F, _I, _P, _P]),
    "pa_reshape_and_cache_fp8": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I64, _F, _F, _P, _P]),
    "pa_decode_attention_fp8": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I64, _F,
                                     _F, _F, _P, _SZ, _P, _P]),
    "pa_status_string": (ctypes.c_char_p, [_I]),
    "pa_launch_count": (ctypes.c_ulonglong, []),
    # include/pa_testing.h
    "pa_testing_set_wait_limit_ns": (None, [ctypes.c_ulonglong]),
    "pa_testing_withhold_copy": (None, [_I]),
}
for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.pa_status_string(status).decode()} (status {status})")


def _check(status: int, where: str) -> None:
    if status != PA_OK:
        raise PaError(status, where)


FP8_POOL_DTYPES = (torch.uint8, torch.float8_e4m3fn)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return PA_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return PA_DTYPE_BF16
    if t.dtype in FP8_POOL_DTYPES:
        return PA_DTYPE_FP8_E4M3
    raise ValueError(f"unsupported dtype {t.dtype}")


def _cuda(*tensors) -> None:
    for t in tensors:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def launch_count() -> int:
    return int(lib.pa_launch_count())


def testing_set_wait_limit_ns(ns: int) -> None:
    """Test hook: limit of the decode kernels' bounded waits (0: the default)."""
    lib.pa_testing_set_wait_limit_ns(int(ns))


def testing_withhold_copy(cta: int) -> None:
    """Test hook: CTA `cta` of later decode launches withholds the copies of its
    second tile, so its bounded waits run out (-1: off)."""
    lib.pa_testing_withhold_copy(int(cta))


def pa_decode_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int,
                              head_dim: int, max_context_len: int) -> int:
    return int(lib.pa_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                             max_context_len))


def pa_num_partitions(max_context_len: int, partition_size: int) -> int:
    return int(lib.pa_num_partitions(max_context_len, partition_size))


def pa_splitk_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int,
                              max_partitions: int) -> int:
    return int(lib.pa_splitk_workspace_bytes(num_seqs, num_q_heads, head_dim, max_partitions))


def pa_reshape_and_cache(key: torch.Tensor, value: torch.Tensor, k_pool: torch.Tensor,
                         v_pool: torch.Tensor, slot_mapping: torch.Tensor,
                         dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """key/value [T, Hkv, d]; pools [nb, bs, Hkv, d]; slot_mapping [T] int64."""
    _cuda(key, value, k_pool, v_pool, slot_mapping, dev_status)
    T, hkv, d = key.shape
    nb, bs = k_pool.shape[:2]
    if value.shape != key.shape or v_pool.shape != k_pool.shape or k_pool.shape[2:] != (hkv, d):
        raise ValueError("shape mismatch")
    if slot_mapping.dtype != torch.int64 or slot_mapping.shape != (T,):
        raise ValueError("slot_mapping must be int64 [T]")
    if not (key.dtype == value.dtype == k_pool.dtype == v_pool.dtype):
        raise ValueError("dtype mismatch")
    _check(lib.pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_pool), _ptr(v_pool),
                                    _ptr(slot_mapping), T, hkv, d, bs, nb, _dtype_code(key),
                                    _ptr(dev_status), _stream(stream)), "pa_reshape_and_cache")


def pa_reshape_and_cache_fp8(key: torch.Tensor, value: torch.Tensor, k_pool: torch.Tensor,
                             v_pool: torch.Tensor, slot_mapping: torch.Tensor, k_scale: float,
                             v_scale: float, dev_status: Optional[torch.Tensor] = None,
                             stream=None) -> None:
    """key/value [T, Hkv, d] bf16; pools [nb, bs, Hkv, d] of E4M3 codes (uint8 or
    float8_e4m3fn); slot_mapping [T] int64; per-tensor scales."""
    _cuda(key, value, k_pool, v_pool, slot_mapping, dev_status)
    T, hkv, d = key.shape
    nb, bs = k_pool.shape[:2]
    if value.shape != key.shape or v_pool.shape != k_pool.shape or k_pool.shape[2:] != (hkv, d):
        raise ValueError("shape mismatch")
    if slot_mapping.dtype != torch.int64 or slot_mapping.shape != (T,):
        raise ValueError("slot_mapping must be int64 [T]")
    if key.dtype != torch.bfloat16 or value.dtype != torch.bfloat16:
        raise ValueError("key and value must be bf16")
    if k_pool.dtype not in FP8_POOL_DTYPES or v_pool.dtype not in FP8_POOL_DTYPES:
        raise ValueError("pools must hold E4M3 codes (uint8 or float8_e4m3fn)")
    _check(lib.pa_reshape_and_cache_fp8(_ptr(key), _ptr(value), _ptr(k_pool), _ptr(v_pool),
                                        _ptr(slot_mapping), T, hkv, d, bs, nb, float(k_scale),
                                        float(v_scale), _ptr(dev_status), _stream(stream)),
           "pa_reshape_and_cache_fp8")


def pa_decode_attention_fp8(out: torch.Tensor, query: torch.Tensor, k_pool: torch.Tensor,
                            v_pool: torch.Tensor, block_tables: torch.Tensor,
                            context_lens: torch.Tensor, max_context_len: int, scale: float,
                            k_scale: float, v_scale: float,
                            workspace: Optional[torch.Tensor] = None,
                            dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """out, query [B, Hq, d] bf16; pools [nb, bs, Hkv, d] of E4M3 codes;
    block_tables [B, max_blocks] int32; context_lens [B] int32."""
    _cuda(out, query, k_pool, v_pool, block_tables, context_lens, workspace, dev_status)
    B, hq, d = query.shape
    nb, bs, hkv, d2 = k_pool.shape
    if out.shape != query.shape or v_pool.shape != k_pool.shape or d2 != d:
        raise ValueError("shape mismatch")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("block_tables must be int32 [B, max_blocks]")
    if context_lens.dtype != torch.int32 or context_lens.shape != (B,):
        raise ValueError("context_lens must be int32 [B]")
    if query.dtype != torch.bfloat16 or out.dtype != torch.bfloat16:
        raise ValueError("query and out must be bf16")
    if k_pool.dtype not in FP8_POOL_DTYPES or v_pool.dtype not in FP8_POOL_DTYPES:
        raise ValueError("pools must hold E4M3 codes (uint8 or float8_e4m3fn)")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_attention_fp8(_ptr(out), _ptr(query), _ptr(k_pool), _ptr(v_pool),
                                       _ptr(block_tables), block_tables.shape[1],
                                       _ptr(context_lens), B, int(max_context_len), hq, hkv, d,
                                       bs, nb, float(scale), float(k_scale), float(v_scale),
                                       _ptr(workspace), ws_bytes, _ptr(dev_status),
                                       _stream(stream)), "pa_decode_attention_fp8")


def pa_copy_blocks(k_pool: torch.Tensor, v_pool: torch.Tensor, block_mapping: torch.Tensor,
                   dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """pools [nb, bs, Hkv, d]; block_mapping [P, 2] int64 (source, destination)."""
    _cuda(k_pool, v_pool, block_mapping, dev_status)
    nb, bs, hkv, d = k_pool.shape
    if v_pool.shape != k_pool.shape or v_pool.dtype != k_pool.dtype:
        raise ValueError("pool mismatch")
    if block_mapping.dtype != torch.int64 or block_mapping.dim() != 2 or block_mapping.shape[1] != 2:
        raise ValueError("block_mapping must be int64 [P, 2]")
    _check(lib.pa_copy_blocks(_ptr(k_pool), _ptr(v_pool), _ptr(block_mapping),
                              block_mapping.shape[0], nb, bs, hkv, d, _dtype_code(k_pool),
                              _ptr(dev_status), _stream(stream)), "pa_copy_blocks")


def pa_swap_blocks(dst_k: torch.Tensor, dst_v: torch.Tensor, src_k: torch.Tensor,
                   src_v: torch.Tensor, block_mapping: torch.Tensor,
                   dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Copies block src -> dst for each (src, dst) row of block_mapping [P, 2]
    int64 from the source pools to the destination pools [nb, bs, Hkv, d];
    one side may be pinned host memory (paging blocks out and back in)."""
    for t in (dst_k, dst_v, src_k, src_v):
        if not t.is_contiguous() or not (t.is_cuda or t.is_pinned()):
            raise ValueError("pools must be contiguous CUDA or pinned host tensors")
    _cuda(block_mapping, dev_status)
    if dst_k.shape[1:] != src_k.shape[1:] or dst_v.shape != dst_k.shape or src_v.shape != src_k.shape:
        raise ValueError("pool shape mismatch")
    if not (dst_k.dtype == dst_v.dtype == src_k.dtype == src_v.dtype):
        raise ValueError("dtype mismatch")
    if block_mapping.dtype != torch.int64 or block_mapping.dim() != 2 or block_mapping.shape[1] != 2:
        raise ValueError("block_mapping must be int64 [P, 2]")
    _, bs, hkv, d = dst_k.shape
    _check(lib.pa_swap_blocks(_ptr(dst_k), _ptr(dst_v), dst_k.shape[0], _ptr(src_k), _ptr(src_v),
                              src_k.shape[0], _ptr(block_mapping), block_mapping.shape[0], bs,
                              hkv, d, _dtype_code(dst_k), _ptr(dev_status), _stream(stream)),
           "pa_swap_blocks")


def pa_prefill_attention(out: torch.Tensor, query: torch.Tensor, cu_q_lens: torch.Tensor,
                         max_q_len: int, k_pool: torch.Tensor, v_pool: torch.Tensor,
                         block_tables: torch.Tensor, context_lens: torch.Tensor,
                         max_context_len: int, scale: float,
                         dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """query/out [total_q, Hq, d] bf16; cu_q_lens [B + 1] int32; pools
    [nb, bs, Hkv, d]; block_tables [B, max_blocks] int32; context_lens [B] int32."""
    _cuda(out, query, cu_q_lens, k_pool, v_pool, block_tables, context_lens, dev_status)
    total_q, hq, d = query.shape
    nb, bs, hkv, d2 = k_pool.shape
    B = context_lens.shape[0]
    if out.shape != query.shape or v_pool.shape != k_pool.shape or d2 != d:
        raise ValueError("shape mismatch")
    if cu_q_lens.dtype != torch.int32 or cu_q_lens.shape != (B + 1,):
        raise ValueError("cu_q_lens must be int32 [B + 1]")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("block_tables must be int32 [B, max_blocks]")
    if context_lens.dtype != torch.int32:
        raise ValueError("context_lens must be int32 [B]")
    if not (out.dtype == query.dtype == k_pool.dtype == v_pool.dtype):
        raise ValueError("dtype mismatch")
    _check(lib.pa_prefill_attention(_ptr(out), _ptr(query), _ptr(cu_q_lens), total_q,
                                    int(max_q_len), _ptr(k_pool), _ptr(v_pool),
                                    _ptr(block_tables), block_tables.shape[1],
                                    _ptr(context_lens), B, int(max_context_len), hq, hkv, d, bs,
                                    nb, float(scale), _dtype_code(query), _ptr(dev_status),
                                    _stream(stream)), "pa_prefill_attention")


def _attn_sizes(out, query, k_pool, v_pool, block_tables, context_lens):
    _cuda(out, query, k_pool, v_pool, block_tables, context_lens)
    B, hq, d = query.shape
    nb, bs, hkv, d2 = k_pool.shape
    if out.shape != query.shape or v_pool.shape != k_pool.shape or d2 != d:
        raise ValueError("shape mismatch")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("block_tables must be int32 [B, max_blocks]")
    if context_lens.dtype != torch.int32 or context_lens.shape != (B,):
        raise ValueError("context_lens must be int32 [B]")
    if not (out.dtype == query.dtype == k_pool.dtype == v_pool.dtype):
        raise ValueError("dtype mismatch")
    return B, hq, hkv, d, bs, nb, block_tables.shape[1]


def pa_decode_attention(out: torch.Tensor, query: torch.Tensor, k_pool: torch.Tensor,
                        v_pool: torch.Tensor, block_tables: torch.Tensor,
                        context_lens: torch.Tensor, max_context_len: int, scale: float,
                        workspace: Optional[torch.Tensor] = None,
                        dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """out, query [B, Hq, d]; pools [nb, bs, Hkv, d]; block_tables [B, max_blocks]
    int32; context_lens [B] int32; workspace: any contiguous CUDA tensor (its
    bytes are used) or None."""
    B, hq, hkv, d, bs, nb, maxb = _attn_sizes(out, query, k_pool, v_pool, block_tables,
                                              context_lens)
    _cuda(workspace, dev_status)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_attention(_ptr(out), _ptr(query), _ptr(k_pool), _ptr(v_pool),
                                   _ptr(block_tables), maxb, _ptr(context_lens), B,
                                   int(max_context_len), hq, hkv, d, bs, nb, float(scale),
                                   _dtype_code(query), _ptr(workspace), ws_bytes,
                                   _ptr(dev_status), _stream(stream)), "pa_decode_attention")


PA_STATIC_SCRATCH_BYTES = 8 << 20


def pa_decode_attention_static(out: torch.Tensor, query: torch.Tensor, k_pool: torch.Tensor,
                               v_pool: torch.Tensor, block_tables: torch.Tensor,
                               context_lens: torch.Tensor, max_context_len: int, scale: float,
                               dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """pa_decode_attention without a workspace: the library's fixed device
    scratch array is used instead (for callers that cannot allocate)."""
    B, hq, hkv, d, bs, nb, maxb = _attn_sizes(out, query, k_pool, v_pool, block_tables,
                                              context_lens)
    _cuda(dev_status)
    _check(lib.pa_decode_attention_static(_ptr(out), _ptr(query), _ptr(k_pool), _ptr(v_pool),
                                          _ptr(block_tables), maxb, _ptr(context_lens), B,
                                          int(max_context_len), hq, hkv, d, bs, nb, float(scale),
                                          _dtype_code(query), _ptr(dev_status), _stream(stream)),
           "pa_decode_attention_static")


def pa_decode_splitk(out: torch.Tensor, query: torch.Tensor, k_pool: torch.Tensor,
                     v_pool: torch.Tensor, block_tables: torch.Tensor,
                     context_lens: torch.Tensor, max_context_len: int, scale: float,
                     partition_size: int, tmp_out: torch.Tensor, max_logits: torch.Tensor,
                     exp_sums: torch.Tensor, dev_status: Optional[torch.Tensor] = None,
                     stream=None) -> None:
    """tmp_out [B, Hq, P, d] fp32; max_logits, exp_sums [B, Hq, P] fp32."""
    B, hq, hkv, d, bs, nb, maxb = _attn_sizes(out, query, k_pool, v_pool, block_tables,
                                              context_lens)
    _cuda(tmp_out, max_logits, exp_sums, dev_status)
    P = tmp_out.shape[2]
    if tmp_out.shape != (B, hq, P, d) or max_logits.shape != (B, hq, P) or \
            exp_sums.shape != (B, hq, P):
        raise ValueError("split-K buffer shape mismatch")
    if not (tmp_out.dtype == max_logits.dtype == exp_sums.dtype == torch.float32):
        raise ValueError("split-K buffers must be float32")
    _check(lib.pa_decode_splitk(_ptr(out), _ptr(query), _ptr(k_pool), _ptr(v_pool),
                                _ptr(block_tables), maxb, _ptr(context_lens), B,
                                int(max_context_len), hq, hkv, d, bs, nb, float(scale),
                                _dtype_code(query), int(partition_size), P, _ptr(tmp_out),
                                _ptr(max_logits), _ptr(exp_sums), _ptr(dev_status),
                                _stream(stream)), "pa_decode_splitk")


def pa_splitk_reduce(out: torch.Tensor, tmp_out: torch.Tensor, max_logits: torch.Tensor,
                     exp_sums: torch.Tensor, context_lens: torch.Tensor, partition_size: int,
                     stream=None) -> None:
    _cuda(out, tmp_out, max_logits, exp_sums, context_lens)
    B, hq, P, d = tmp_out.shape
    if out.shape != (B, hq, d):
        raise ValueError("shape mismatch")
    _check(lib.pa_splitk_reduce(_ptr(out), _ptr(tmp_out), _ptr(max_logits), _ptr(exp_sums),
                                _ptr(context_lens), B, hq, d, int(partition_size), P,
                                _dtype_code(out), _stream(stream)), "pa_splitk_reduce")


__all__ = [
    "lib", "LIB_PATH", "SIGNATURES", "PaError", "launch_count",
    "pa_reshape_and_cache", "pa_reshape_and_cache_fp8", "pa_decode_attention_fp8",
    "testing_set_wait_limit_ns", "testing_withhold_copy", "pa_copy_blocks", "pa_swap_blocks", "pa_prefill_attention", "pa_decode_attention", "pa_decode_workspace_bytes",
    "pa_decode_attention_static", "PA_STATIC_SCRATCH_BYTES",
    "pa_num_partitions", "pa_splitk_workspace_bytes", "pa_decode_splitk", "pa_splitk_reduce",
    "PA_OK", "PA_ERR_INVALID_ARG", "PA_ERR_UNSUPPORTED", "PA_ERR_CUDA", "PA_ERR_WORKSPACE",
    "PA_DTYPE_F32", "PA_DTYPE_BF16", "PA_DTYPE_FP8_E4M3",
    "PA_DEV_BAD_SLOT", "PA_DEV_BAD_BLOCK", "PA_DEV_BAD_CONTEXT", "PA_DEV_WAIT_TIMEOUT",
]
