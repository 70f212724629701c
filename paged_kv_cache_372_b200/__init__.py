"""Python binding of libpa_b200 (include/pa.h): argument marshalling only.

Every function here forwards torch CUDA tensors' device pointers, sizes and the
current CUDA stream to the C ABI of the same name and raises on a non-zero
status. There is no other code path: without the built library, or with CPU
tensors, the calls raise. Build the library with
``python -m paged_kv_cache_372_b200.build`` (``__graft_entry__.build()`` does it).
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# PA_B200_LIB points the binding at another build of the same library.
LIB_PATH = os.environ.get("PA_B200_LIB") or os.path.join(HERE, "_lib", "libpa_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "pa.h")

PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_DEVICE_CHECK = range(5)
PA_F16, PA_BF16 = 0, 1
PA_KV_E4M3, PA_KV_INT8 = 0, 1
DEVERR_BLOCK_ID, DEVERR_CONTEXT, DEVERR_SLOT, DEVERR_PAIR, DEVERR_TIMEOUT, DEVERR_QRANGE = 1, 2, 4, 8, 16, 32

_DTYPES = {torch.float16: PA_F16, torch.bfloat16: PA_BF16}


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


_lib = None
_P, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libpa_b200 is not built ({LIB_PATH} missing); "
                               "run `python -m paged_kv_cache_372_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.pa_status_string.restype = ctypes.c_char_p
        L.pa_status_string.argtypes = [_I]
        L.pa_last_error.restype = ctypes.c_char_p
        L.pa_last_error.argtypes = []
        L.pa_decode.restype = _I
        L.pa_decode.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I,
                                _P, _SZ, _P]
        L.pa_decode_append.restype = _I
        L.pa_decode_append.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                                       _I, _P, _SZ, _P]
        L.pa_decode_shared.restype = _I
        L.pa_decode_shared.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                                       _I, _P, _SZ, _P]
        L.pa_decode_fp8_partition_size.restype = _I
        L.pa_decode_fp8_partition_size.argtypes = [_I] * 7
        L.pa_decode_fp8_workspace_size.restype = _SZ
        L.pa_decode_fp8_workspace_size.argtypes = [_I] * 7
        L.pa_decode_shared_partition_size.restype = _I
        L.pa_decode_shared_partition_size.argtypes = [_I] * 7
        L.pa_decode_shared_workspace_size.restype = _SZ
        L.pa_decode_shared_workspace_size.argtypes = [_I] * 7
        L.pa_decode_fp8.restype = _I
        L.pa_decode_fp8.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _F, _F, _I,
                                    _P, _SZ, _P]
        L.pa_reshape_and_cache_fp8.restype = _I
        L.pa_reshape_and_cache_fp8.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _F, _P]
        L.pa_decode_workspace_size.restype = _SZ
        L.pa_decode_workspace_size.argtypes = [_I] * 7
        L.pa_decode_partition_size.restype = _I
        L.pa_decode_partition_size.argtypes = [_I] * 7
        L.pa_reshape_and_cache.restype = _I
        L.pa_reshape_and_cache.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]
        L.pa_copy_blocks.restype = _I
        L.pa_copy_blocks.argtypes = [ctypes.POINTER(_P), _I, _P, _I, _SZ, _I, _P]
        L.pa_swap_blocks.restype = _I
        L.pa_swap_blocks.argtypes = [ctypes.POINTER(_P), ctypes.POINTER(_P), _I, _P, _I, _SZ, _I, _I, _P]
        L.pa_device_errors.restype = _I
        L.pa_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint), _I, _P]
        L.pa_num_sms.restype = _I
        L.pa_num_sms.argtypes = []
        L.pa_selftest_bounded_wait.restype = _I
        L.pa_selftest_bounded_wait.argtypes = [ctypes.c_ulonglong, _P]
        L.pa_reshape_and_cache_quant.restype = _I
        L.pa_reshape_and_cache_quant.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P]
        L.pa_reshape_and_cache_quant_blocks.restype = _I
        L.pa_reshape_and_cache_quant_blocks.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P]
        L.pa_decode_quant_blocks.restype = _I
        L.pa_decode_quant.restype = _I
        L.pa_decode_quant.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P, _P,
                                      _I, _P, _SZ, _P]
        L.pa_decode_quant_blocks.argtypes = L.pa_decode_quant.argtypes
        L.pa_decode_shared_quant_blocks.restype = _I
        L.pa_decode_shared_quant_blocks.argtypes = L.pa_decode_quant.argtypes
        L.pa_decode_shared_quant.restype = _I
        L.pa_decode_shared_quant.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I,
                                             _P, _P, _I, _P, _SZ, _P]
        L.pa_launch_count.restype = ctypes.c_ulonglong
        L.pa_launch_count.argtypes = []
        L.pa_decode_noalloc.restype = _I
        L.pa_decode_noalloc.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P]
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/pa.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def _check(status: int) -> None:
    if status != PA_OK:
        L = lib()
        name = L.pa_status_string(status).decode()
        detail = L.pa_last_error().decode()
        raise PagedAttentionError(status, f"{name}: {detail}")


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _cuda(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


def pa_decode_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                             partition_size=0) -> int:
    return int(lib().pa_decode_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                              max_context_len, partition_size))


def pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                             partition_size=0) -> int:
    n = int(lib().pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                           max_context_len, partition_size))
    if n == 0:
        raise PagedAttentionError(PA_ERR_INVALID, "unsupported shape or partition size")
    return n


def pa_decode_fp8_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                                 partition_size=0) -> int:
    return int(lib().pa_decode_fp8_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                  max_context_len, partition_size))


def pa_decode_fp8_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                                 partition_size=0) -> int:
    n = int(lib().pa_decode_fp8_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                               max_context_len, partition_size))
    if n == 0:
        raise PagedAttentionError(PA_ERR_INVALID, "unsupported shape or partition size")
    return n


def pa_decode_shared_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                                    partition_size=0) -> int:
    return int(lib().pa_decode_shared_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                     max_context_len, partition_size))


def pa_decode_shared_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                                    partition_size=0) -> int:
    n = int(lib().pa_decode_shared_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                  max_context_len, partition_size))
    if n == 0:
        raise PagedAttentionError(PA_ERR_INVALID, "unsupported shape or partition size")
    return n


def alloc_workspace(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                    partition_size=0, device=None, shared=False, fp8=False) -> torch.Tensor:
    """Workspace for pa_decode / pa_decode_append, or with shared=True for
    pa_decode_shared, or with fp8=True for pa_decode_fp8."""
    size = (pa_decode_shared_workspace_size if shared else pa_decode_fp8_workspace_size if fp8
            else pa_decode_workspace_size)
    n = size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len, partition_size)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def pa_decode(out, q, k_pool, v_pool, block_tables, context_lens, scale, max_context_len,
              partition_size=0, workspace=None, stream=None) -> torch.Tensor:
    """out[s][h] = softmax(scale * q[s][h] . K) V over sequence s's paged cache.

    q, out [B][H][D]; k_pool, v_pool [NB][Hkv][bs][D] (fp16 or bf16);
    block_tables int32 [B][W]; context_lens int32 [B]. Asynchronous on `stream`.
    """
    if q.dim() != 3 or k_pool.dim() != 4:
        raise ValueError("q must be [B][H][D] and the pools [NB][Hkv][bs][D]")
    B, H, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or tuple(v_pool.shape) != tuple(k_pool.shape) or tuple(out.shape) != (B, H, D):
        raise ValueError("shape mismatch between q, out and the pools")
    if q.dtype not in _DTYPES or k_pool.dtype != q.dtype or v_pool.dtype != q.dtype or out.dtype != q.dtype:
        raise ValueError("q, out and the pools must share one dtype, fp16 or bf16")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or tuple(context_lens.shape) != (B,):
        raise ValueError("block_tables must be [B][W] and context_lens [B]")
    if workspace is None:
        workspace = alloc_workspace(B, H, Hkv, D, bs, max_context_len, partition_size, q.device)
    _check(lib().pa_decode(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(block_tables, "block_tables", torch.int32), _cuda(context_lens, "context_lens", torch.int32),
        B, H, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len), float(scale), _DTYPES[q.dtype],
        int(partition_size), _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return out


def pa_decode_append(out, q, k_new, v_new, k_pool, v_pool, block_tables, context_lens, scale, max_context_len,
                     partition_size=0, workspace=None, stream=None) -> torch.Tensor:
    """Write k_new/v_new [B][Hkv][D] at each sequence's last position, then pa_decode."""
    B, H, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    if tuple(k_new.shape) != (B, Hkv, D) or tuple(v_new.shape) != (B, Hkv, D):
        raise ValueError("k_new and v_new must be [B][Hkv][D]")
    if k_new.dtype != q.dtype or v_new.dtype != q.dtype or k_pool.dtype != q.dtype or v_pool.dtype != q.dtype:
        raise ValueError("q, k_new, v_new and the pools must share one dtype")
    if workspace is None:
        workspace = alloc_workspace(B, H, Hkv, D, bs, max_context_len, partition_size, q.device)
    _check(lib().pa_decode_append(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k_new, "k_new"), _cuda(v_new, "v_new"), _cuda(k_pool, "k_pool"),
        _cuda(v_pool, "v_pool"), _cuda(block_tables, "block_tables", torch.int32),
        _cuda(context_lens, "context_lens", torch.int32), B, H, Hkv, D, bs, block_tables.shape[1], NB,
        int(max_context_len), float(scale), _DTYPES[q.dtype], int(partition_size), _cuda(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def pa_decode_shared(out, q, k_pool, v_pool, block_tables, context_lens, scale, max_context_len,
                     partition_size=0, workspace=None, stream=None, k_new=None, v_new=None) -> torch.Tensor:
    """pa_decode (or, with k_new/v_new, pa_decode_append) that streams blocks
    shared by the leading parts of several sequences' tables once per group."""
    B, H, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or tuple(v_pool.shape) != tuple(k_pool.shape) or tuple(out.shape) != (B, H, D):
        raise ValueError("shape mismatch between q, out and the pools")
    if q.dtype not in _DTYPES or k_pool.dtype != q.dtype or v_pool.dtype != q.dtype or out.dtype != q.dtype:
        raise ValueError("q, out and the pools must share one dtype, fp16 or bf16")
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    if k_new is not None:
        if tuple(k_new.shape) != (B, Hkv, D) or tuple(v_new.shape) != (B, Hkv, D):
            raise ValueError("k_new and v_new must be [B][Hkv][D]")
        if k_new.dtype != q.dtype or v_new.dtype != q.dtype:
            raise ValueError("k_new and v_new must have q's dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or tuple(context_lens.shape) != (B,):
        raise ValueError("block_tables must be [B][W] and context_lens [B]")
    if workspace is None:
        workspace = alloc_workspace(B, H, Hkv, D, bs, max_context_len, partition_size, q.device, shared=True)
    _check(lib().pa_decode_shared(
        _cuda(out, "out"), _cuda(q, "q"), None if k_new is None else _cuda(k_new, "k_new"),
        None if v_new is None else _cuda(v_new, "v_new"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(block_tables, "block_tables", torch.int32), _cuda(context_lens, "context_lens", torch.int32),
        B, H, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len), float(scale), _DTYPES[q.dtype],
        int(partition_size), _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return out


def pa_decode_fp8(out, q, k_pool, v_pool, block_tables, context_lens, scale, max_context_len, k_scale, v_scale,
                  partition_size=0, workspace=None, stream=None) -> torch.Tensor:
    """pa_decode over an E4M3 cache: k_pool, v_pool uint8 codes [NB][Hkv][bs][D];
    element = scale * code (k_scale for keys, v_scale for values)."""
    B, H, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or tuple(v_pool.shape) != tuple(k_pool.shape) or tuple(out.shape) != (B, H, D):
        raise ValueError("shape mismatch between q, out and the pools")
    if k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise ValueError("fp8 pools must be uint8 tensors of E4M3 codes")
    if q.dtype not in _DTYPES or out.dtype != q.dtype:
        raise ValueError("q and out must share one dtype, fp16 or bf16")
    if workspace is None:
        workspace = alloc_workspace(B, H, Hkv, D, bs, max_context_len, partition_size, q.device, fp8=True)
    _check(lib().pa_decode_fp8(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(block_tables, "block_tables", torch.int32), _cuda(context_lens, "context_lens", torch.int32),
        B, H, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len), float(scale), _DTYPES[q.dtype],
        float(k_scale), float(v_scale), int(partition_size), _cuda(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def pa_reshape_and_cache_fp8(k, v, k_pool, v_pool, slot_mapping, k_scale, v_scale, stream=None) -> None:
    """Quantising write: k_pool[slot] = E4M3(k[t] / k_scale) (and v) for t with slot >= 0."""
    T, Hkv, D = k.shape
    NB, Hkv2, bs, D2 = k_pool.shape
    if (Hkv2, D2) != (Hkv, D) or tuple(v.shape) != tuple(k.shape) or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("shape mismatch between k, v and the pools")
    if k.dtype not in _DTYPES or v.dtype != k.dtype or k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise ValueError("k, v fp16/bf16; pools uint8")
    _check(lib().pa_reshape_and_cache_fp8(
        _cuda(k, "k"), _cuda(v, "v"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(slot_mapping, "slot_mapping", torch.int64), T, Hkv, D, bs, NB, _DTYPES[k.dtype], float(k_scale),
        float(v_scale), _stream(stream)))


KV_FORMATS = {"e4m3": PA_KV_E4M3, "int8": PA_KV_INT8}


def _scales(t, name, n, blocks=None):
    shape = (n,) if blocks is None else (blocks, n)
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.float32 or tuple(t.shape) != shape:
        what = "[num_kv_heads]" if blocks is None else "[num_blocks][num_kv_heads]"
        raise ValueError(f"{name} must be a float32 CUDA tensor of shape {what}")
    return _cuda(t, name)


def pa_reshape_and_cache_quant(k, v, k_pool, v_pool, slot_mapping, kv_format, k_scales, v_scales,
                               stream=None) -> None:
    """Quantising write into an 8-bit cache ("e4m3" or "int8" codes) with one
    scale per KV head: k_pool[slot] = encode(k[t] / k_scales[h]) (and v)."""
    T, Hkv, D = k.shape
    NB, Hkv2, bs, D2 = k_pool.shape
    if (Hkv2, D2) != (Hkv, D) or tuple(v.shape) != tuple(k.shape) or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("shape mismatch between k, v and the pools")
    if k.dtype not in _DTYPES or v.dtype != k.dtype or k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise ValueError("k, v fp16/bf16; pools uint8")
    _check(lib().pa_reshape_and_cache_quant(
        _cuda(k, "k"), _cuda(v, "v"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(slot_mapping, "slot_mapping", torch.int64), T, Hkv, D, bs, NB, _DTYPES[k.dtype],
        KV_FORMATS[kv_format], _scales(k_scales, "k_scales", Hkv), _scales(v_scales, "v_scales", Hkv),
        _stream(stream)))


def pa_decode_quant(out, q, k_pool, v_pool, block_tables, context_lens, scale, max_context_len, kv_format,
                    k_scales, v_scales, partition_size=0, workspace=None, stream=None) -> torch.Tensor:
    """pa_decode over an 8-bit cache ("e4m3" or "int8" uint8 codes [NB][Hkv][bs][D])
    with one scale per KV head (float32 CUDA tensors [Hkv])."""
    B, H, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or tuple(v_pool.shape) != tuple(k_pool.shape) or tuple(out.shape) != (B, H, D):
        raise ValueError("shape mismatch between q, out and the pools")
    if k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise ValueError("8-bit pools must be uint8 tensors of codes")
    if q.dtype not in _DTYPES or out.dtype != q.dtype:
        raise ValueError("q and out must share one dtype, fp16 or bf16")
    if workspace is None:
        workspace = alloc_workspace(B, H, Hkv, D, bs, max_context_len, partition_size, q.device, fp8=True)
    _check(lib().pa_decode_quant(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(block_tables, "block_tables", torch.int32), _cuda(context_lens, "context_lens", torch.int32),
        B, H, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len), float(scale), _DTYPES[q.dtype],
        KV_FORMATS[kv_format], _scales(k_scales, "k_scales", Hkv), _scales(v_scales, "v_scales", Hkv),
        int(partition_size), _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return out


def pa_reshape_and_cache_quant_blocks(k, v, k_pool, v_pool, slot_mapping, kv_format, k_scales, v_scales,
                                      stream=None) -> None:
    """pa_reshape_and_cache_quant with one scale per (physical block, KV head):
    k_scales, v_scales float32 CUDA tensors [NB][Hkv]."""
    T, Hkv, D = k.shape
    NB, Hkv2, bs, D2 = k_pool.shape
    if (Hkv2, D2) != (Hkv, D) or tuple(v.shape) != tuple(k.shape) or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("shape mismatch between k, v and the pools")
    if k.dtype not in _DTYPES or v.dtype != k.dtype or k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise ValueError("k, v fp16/bf16; pools uint8")
    _check(lib().pa_reshape_and_cache_quant_blocks(
        _cuda(k, "k"), _cuda(v, "v"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(slot_mapping, "slot_mapping", torch.int64), T, Hkv, D, bs, NB, _DTYPES[k.dtype],
        KV_FORMATS[kv_format], _scales(k_scales, "k_scales", Hkv, NB), _scales(v_scales, "v_scales", Hkv, NB),
        _stream(stream)))


def pa_decode_quant_blocks(out, q, k_pool, v_pool, block_tables, context_lens, scale, max_context_len, kv_format,
                           k_scales, v_scales, partition_size=0, workspace=None, stream=None) -> torch.Tensor:
    """pa_decode_quant with one scale per (physical block, KV head): k_scales,
    v_scales float32 CUDA tensors [NB][Hkv]."""
    B, H, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or tuple(v_pool.shape) != tuple(k_pool.shape) or tuple(out.shape) != (B, H, D):
        raise ValueError("shape mismatch between q, out and the pools")
    if k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise ValueError("8-bit pools must be uint8 tensors of codes")
    if q.dtype not in _DTYPES or out.dtype != q.dtype:
        raise ValueError("q and out must share one dtype, fp16 or bf16")
    if workspace is None:
        workspace = alloc_workspace(B, H, Hkv, D, bs, max_context_len, partition_size, q.device, fp8=True)
    _check(lib().pa_decode_quant_blocks(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(block_tables, "block_tables", torch.int32), _cuda(context_lens, "context_lens", torch.int32),
        B, H, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len), float(scale), _DTYPES[q.dtype],
        KV_FORMATS[kv_format], _scales(k_scales, "k_scales", Hkv, NB), _scales(v_scales, "v_scales", Hkv, NB),
        int(partition_size), _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return out


def pa_decode_shared_quant(out, q, k_pool, v_pool, block_tables, context_lens, scale, max_context_len, kv_format,
                           k_scales, v_scales, partition_size=0, workspace=None, stream=None) -> torch.Tensor:
    """pa_decode_shared over an 8-bit cache ("e4m3" or "int8" codes) with one
    scale per KV head (float32 CUDA tensors [Hkv])."""
    B, H, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or tuple(v_pool.shape) != tuple(k_pool.shape) or tuple(out.shape) != (B, H, D):
        raise ValueError("shape mismatch between q, out and the pools")
    if k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise ValueError("8-bit pools must be uint8 tensors of codes")
    if q.dtype not in _DTYPES or out.dtype != q.dtype:
        raise ValueError("q and out must share one dtype, fp16 or bf16")
    if workspace is None:
        workspace = alloc_workspace(B, H, Hkv, D, bs, max_context_len, partition_size, q.device, shared=True)
    _check(lib().pa_decode_shared_quant(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(block_tables, "block_tables", torch.int32), _cuda(context_lens, "context_lens", torch.int32),
        B, H, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len), float(scale), _DTYPES[q.dtype],
        KV_FORMATS[kv_format], _scales(k_scales, "k_scales", Hkv), _scales(v_scales, "v_scales", Hkv),
        int(partition_size), _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return out


def pa_decode_shared_quant_blocks(out, q, k_pool, v_pool, block_tables, context_lens, scale, max_context_len,
                                  kv_format, k_scales, v_scales, partition_size=0, workspace=None,
                                  stream=None) -> torch.Tensor:
    """pa_decode_shared_quant with one scale per (physical block, KV head):
    k_scales, v_scales float32 CUDA tensors [NB][Hkv]."""
    B, H, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or tuple(v_pool.shape) != tuple(k_pool.shape) or tuple(out.shape) != (B, H, D):
        raise ValueError("shape mismatch between q, out and the pools")
    if k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise ValueError("8-bit pools must be uint8 tensors of codes")
    if q.dtype not in _DTYPES or out.dtype != q.dtype:
        raise ValueError("q and out must share one dtype, fp16 or bf16")
    if workspace is None:
        workspace = alloc_workspace(B, H, Hkv, D, bs, max_context_len, partition_size, q.device, shared=True)
    _check(lib().pa_decode_shared_quant_blocks(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(block_tables, "block_tables", torch.int32), _cuda(context_lens, "context_lens", torch.int32),
        B, H, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len), float(scale), _DTYPES[q.dtype],
        KV_FORMATS[kv_format], _scales(k_scales, "k_scales", Hkv, NB), _scales(v_scales, "v_scales", Hkv, NB),
        int(partition_size), _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return out


def pa_reshape_and_cache(k, v, k_pool, v_pool, slot_mapping, stream=None) -> None:
    """k_pool[slot // bs][h][slot % bs] = k[t][h] (and v) for every t with slot >= 0."""
    T, Hkv, D = k.shape
    NB, Hkv2, bs, D2 = k_pool.shape
    if (Hkv2, D2) != (Hkv, D) or tuple(v.shape) != tuple(k.shape) or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("shape mismatch between k, v and the pools")
    if k.dtype not in _DTYPES or any(x.dtype != k.dtype for x in (v, k_pool, v_pool)):
        raise ValueError("k, v and the pools must share one dtype, fp16 or bf16")
    if tuple(slot_mapping.shape) != (T,):
        raise ValueError("slot_mapping must be [num_tokens]")
    _check(lib().pa_reshape_and_cache(
        _cuda(k, "k"), _cuda(v, "v"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(slot_mapping, "slot_mapping", torch.int64), T, Hkv, D, bs, NB, _DTYPES[k.dtype],
        _stream(stream)))


def pa_copy_blocks(pools, src_dst_pairs, stream=None) -> None:
    """For each (src, dst) row of src_dst_pairs (int64 CUDA [P][2]): pool[dst] = pool[src], every pool."""
    pools = list(pools)
    if not pools:
        return
    nb = pools[0].shape[0]
    block_bytes = pools[0][0].numel() * pools[0].element_size()
    for t in pools:
        if t.shape[0] != nb or t[0].numel() * t.element_size() != block_bytes:
            raise ValueError("all pools must have the same number and size of blocks")
    pairs = src_dst_pairs
    if pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [P][2]")
    ptrs = (_P * len(pools))(*[_cuda(t, "pool") for t in pools])
    _check(lib().pa_copy_blocks(ptrs, len(pools), _cuda(pairs, "src_dst_pairs", torch.int64),
                                pairs.shape[0], block_bytes, nb, _stream(stream)))


def pa_swap_blocks(dst_pools, src_pools, src_dst_pairs, stream=None) -> None:
    """dst_pools[i][dst] = src_pools[i][src] for each (src, dst) row of src_dst_pairs.

    Pools are CUDA tensors or page-locked CPU tensors (``pin_memory()``) with the
    same block size; src_dst_pairs is an int64 [P][2] CUDA or page-locked tensor.
    """
    dst_pools, src_pools = list(dst_pools), list(src_pools)
    if len(dst_pools) != len(src_pools):
        raise ValueError("dst_pools and src_pools differ in length")
    if not dst_pools:
        return
    block_bytes = dst_pools[0][0].numel() * dst_pools[0].element_size()

    def ptr(t, name):
        if not isinstance(t, torch.Tensor) or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous tensor")
        if not t.is_cuda and not t.is_pinned():
            raise ValueError(f"{name} must be a CUDA tensor or page-locked (pin_memory) CPU tensor")
        return t.data_ptr()

    for t in dst_pools + src_pools:
        if t[0].numel() * t.element_size() != block_bytes:
            raise ValueError("all pools must have the same block size")
    pairs = src_dst_pairs
    if pairs.dim() != 2 or pairs.shape[1] != 2 or pairs.dtype != torch.int64:
        raise ValueError("src_dst_pairs must be int64 [P][2]")
    dp = (_P * len(dst_pools))(*[ptr(t, "dst pool") for t in dst_pools])
    sp = (_P * len(src_pools))(*[ptr(t, "src pool") for t in src_pools])
    _check(lib().pa_swap_blocks(dp, sp, len(dst_pools), ptr(pairs, "src_dst_pairs"), pairs.shape[0],
                                block_bytes, src_pools[0].shape[0], dst_pools[0].shape[0], _stream(stream)))


def pa_launch_count() -> int:
    """Kernels the library has launched from the calling thread so far (all
    entry points); the difference around a region is that region's count."""
    return int(lib().pa_launch_count())


def pa_device_errors(clear: bool = True, stream=None) -> int:
    """Synchronise the stream and return (optionally clear) the device error bits."""
    flags = ctypes.c_uint(0)
    st = lib().pa_device_errors(ctypes.byref(flags), int(bool(clear)), _stream(stream))
    if st not in (PA_OK, PA_ERR_DEVICE_CHECK):
        _check(st)
    return int(flags.value)


def pa_num_sms() -> int:
    return int(lib().pa_num_sms())


def pa_selftest_bounded_wait(limit_ns: int, stream=None) -> None:
    """Run the bounded-wait self-test kernel (sets DEVERR_TIMEOUT when it ends)."""
    _check(lib().pa_selftest_bounded_wait(int(limit_ns), _stream(stream)))


NOALLOC_SCRATCH_BYTES = 16 << 20


def pa_decode_noalloc(out, q, k_pool, v_pool, block_tables, context_lens, scale, max_context_len,
                      partition_size=0, stream=None) -> torch.Tensor:
    """pa_decode with the library's fixed scratch array instead of a workspace
    (for callers that cannot allocate at decode time; see include/pa.h)."""
    B, H, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    _check(lib().pa_decode_noalloc(
        _cuda(out, "out"), _cuda(q, "q"), _cuda(k_pool, "k_pool"), _cuda(v_pool, "v_pool"),
        _cuda(block_tables, "block_tables", torch.int32), _cuda(context_lens, "context_lens", torch.int32),
        B, H, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len), float(scale), _DTYPES[q.dtype],
        int(partition_size), _stream(stream)))
    return out
