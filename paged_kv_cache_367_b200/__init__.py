"""B200-native paged KV append and PagedAttention decode.

A thin ctypes binding over ``libpagedkv.so`` (C ABI in include/pagedkv.h). It
only marshals arguments: every step of the path runs in the library's CUDA
kernels. PyTorch tensors supply device memory and the current CUDA stream.
There is no fallback: if the library is missing, every call raises.

Build the library with ``python -m paged_kv_cache_367_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["paged_kv_append", "paged_attention_decode", "paged_attention_workspace_size",
           "paged_attention_decode_static", "paged_kv_copy_blocks", "paged_kv_swap_blocks",
           "paged_attention_prefill", "append_args", "decode_args",
           "pkv_device_status", "pkv_selftest_expired_wait", "pkv_status_string", "pkv_version",
           "load_library", "PagedKVError",
           "PKV_F32", "PKV_F16", "PKV_BF16", "PKV_FP8_E4M3", "PKV_DECODE_FORCE_SIMT",
           "PKV_DECODE_ZEROED_WORKSPACE", "PKV_DECODE_EARLY_START", "PKV_DECODE_TENSOR_CORES",
           "PKV_DECODE_CUDA_CORES", "PKV_PREFILL_MMA_SYNC",
           "LIB_PATH", "EXPORTED_SYMBOLS"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedkv.so")

PKV_F32, PKV_F16, PKV_BF16, PKV_FP8_E4M3 = 0, 1, 2, 3
PKV_DECODE_FORCE_SIMT = 1
PKV_DECODE_ZEROED_WORKSPACE = 2
PKV_DECODE_EARLY_START = 4
PKV_DECODE_TENSOR_CORES = 8
PKV_DECODE_CUDA_CORES = 16
PKV_PREFILL_MMA_SYNC = 1

EXPORTED_SYMBOLS = ("paged_kv_append", "paged_attention_workspace_size",
                    "paged_attention_decode", "paged_attention_decode_static",
                    "paged_attention_prefill", "pkv_device_status", "pkv_selftest_expired_wait",
                    "pkv_status_string", "pkv_version",
                    # include/pagedkv_blocks.h
                    "pkv_bm_create", "pkv_bm_destroy", "pkv_bm_num_free", "pkv_bm_num_free_host",
                    "pkv_bm_can_allocate", "pkv_bm_allocate", "pkv_bm_can_append",
                    "pkv_bm_append_slot", "pkv_bm_append_slots", "pkv_bm_fork", "pkv_bm_free", "pkv_bm_swap_out",
                    "pkv_bm_swap_in", "pkv_bm_block_tables", "pkv_bm_seq_len", "pkv_bm_refcount",
                    "pkv_bm_usage", "pkv_bm_check", "paged_kv_copy_blocks", "paged_kv_swap_blocks")

_DTYPE_CODES = {torch.float32: PKV_F32, torch.float16: PKV_F16, torch.bfloat16: PKV_BF16,
                torch.uint8: PKV_FP8_E4M3, torch.float8_e4m3fn: PKV_FP8_E4M3}

_lib = None


class PagedKVError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: status {status} ({pkv_status_string(status)})")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libpagedkv.so once; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m paged_kv_cache_367_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, I64, F, U, SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                           ctypes.c_uint, ctypes.c_size_t)
    lib.paged_kv_append.argtypes = [P, P, P, P, P, I, I, I, I, I64, I, I, P, P, P]
    lib.paged_kv_append.restype = I
    lib.paged_attention_workspace_size.argtypes = [I, I, I, I, I, I]
    lib.paged_attention_workspace_size.restype = SZ
    lib.paged_attention_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I64, I, F, I, I,
                                           P, P, I, I, U, P, SZ, P]
    lib.paged_attention_decode.restype = I
    lib.pkv_status_string.argtypes = [I]
    lib.pkv_status_string.restype = ctypes.c_char_p
    lib.pkv_version.argtypes = []
    lib.pkv_version.restype = I
    lib.pkv_device_status.argtypes = [I]
    lib.pkv_device_status.restype = I
    lib.pkv_selftest_expired_wait.argtypes = [I64, I, P]
    lib.pkv_selftest_expired_wait.restype = I
    lib.paged_attention_decode_static.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I64, I, F,
                                                  I, I, P, P, I, I, U, P]
    lib.paged_attention_decode_static.restype = I
    lib.paged_attention_prefill.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I64, F,
                                            I, I, P, P, U, P]
    lib.paged_attention_prefill.restype = I
    # Block manager and block copies (include/pagedkv_blocks.h).
    lib.pkv_bm_create.argtypes = [I64, I64, I, I]
    lib.pkv_bm_create.restype = P
    lib.pkv_bm_destroy.argtypes = [P]
    lib.pkv_bm_destroy.restype = None
    for name in ("pkv_bm_num_free", "pkv_bm_num_free_host"):
        getattr(lib, name).argtypes = [P]
        getattr(lib, name).restype = I64
    lib.pkv_bm_can_allocate.argtypes = [P, I64]
    lib.pkv_bm_can_allocate.restype = I
    lib.pkv_bm_allocate.argtypes = [P, I64, P, I64, P, P]
    lib.pkv_bm_allocate.restype = I
    lib.pkv_bm_can_append.argtypes = [P, I64]
    lib.pkv_bm_can_append.restype = I
    lib.pkv_bm_append_slot.argtypes = [P, I64, ctypes.c_int32, P, P, P]
    lib.pkv_bm_append_slot.restype = I
    lib.pkv_bm_append_slots.argtypes = [P, P, P, I, P, P, P]
    lib.pkv_bm_append_slots.restype = I
    lib.pkv_bm_fork.argtypes = [P, I64, I64]
    lib.pkv_bm_fork.restype = I
    lib.pkv_bm_free.argtypes = [P, I64]
    lib.pkv_bm_free.restype = I
    for name in ("pkv_bm_swap_out", "pkv_bm_swap_in"):
        getattr(lib, name).argtypes = [P, P, I, P, I64, P]
        getattr(lib, name).restype = I
    lib.pkv_bm_block_tables.argtypes = [P, P, I, I, P, P]
    lib.pkv_bm_block_tables.restype = I
    lib.pkv_bm_seq_len.argtypes = [P, I64]
    lib.pkv_bm_seq_len.restype = I64
    lib.pkv_bm_refcount.argtypes = [P, ctypes.c_int32]
    lib.pkv_bm_refcount.restype = I
    lib.pkv_bm_usage.argtypes = [P, P]
    lib.pkv_bm_usage.restype = I
    lib.pkv_bm_check.argtypes = [P]
    lib.pkv_bm_check.restype = I
    lib.paged_kv_copy_blocks.argtypes = [P, P, P, I, I64, I64, P]
    lib.paged_kv_copy_blocks.restype = I
    lib.paged_kv_swap_blocks.argtypes = [P, P, P, P, P, I, I64, I64, I64, P]
    lib.paged_kv_swap_blocks.restype = I
    _lib = lib
    return lib


def pkv_status_string(status: int) -> str:
    return load_library().pkv_status_string(int(status)).decode()


def pkv_version() -> int:
    return load_library().pkv_version()


def pkv_device_status(clear: bool = False) -> int:
    """Health word since the last clear: 0 healthy; | 1 a bounded wait inside a
    kernel expired; | 2 a block-table entry outside the pool was read."""
    return load_library().pkv_device_status(1 if clear else 0)


def pkv_selftest_expired_wait(limit_cycles: int = 1 << 20, note_out_of_pool: bool = True) -> None:
    """Enqueue the health word's fault-free self-test (a bounded wait on a barrier
    nothing completes) on the current stream."""
    st = load_library().pkv_selftest_expired_wait(int(limit_cycles), 1 if note_out_of_pool else 0,
                                                  _stream(None))
    if st != 0:
        raise PagedKVError("pkv_selftest_expired_wait", st)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _DTYPE_CODES[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def append_args(key, value, k_cache, v_cache, slot_mapping, *, k_scale=None, v_scale=None,
                stream=None) -> tuple:
    """The arguments of the C call paged_kv_append for these tensors (pointers,
    sizes, dtype codes, stream), in its order: a caller that repeats the call on
    the same buffers can marshal them once."""
    T, Hkv, D = key.shape
    nb, bs = k_cache.shape[0], k_cache.shape[1]
    return (_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), T, Hkv, D,
            bs, nb, _dtype_code(key), _dtype_code(k_cache), _ptr(k_scale), _ptr(v_scale),
            _stream(stream))


def paged_kv_append(key, value, k_cache, v_cache, slot_mapping, *, k_scale=None, v_scale=None,
                    stream=None) -> None:
    """Write key/value [T, Hkv, D] into the pool [num_blocks, bs, Hkv, D] at
    slot_mapping [T] (int64); see paged_kv_append in include/pagedkv.h."""
    st = load_library().paged_kv_append(*append_args(key, value, k_cache, v_cache, slot_mapping,
                                                     k_scale=k_scale, v_scale=v_scale,
                                                     stream=stream))
    if st != 0:
        raise PagedKVError("paged_kv_append", st)


def paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_seq_len,
                                   partition_size) -> int:
    return load_library().paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads,
                                                         head_dim, max_seq_len, partition_size)


def decode_args(out, query, k_cache, v_cache, block_table, seq_lens, *, max_seq_len, scale,
                partition_size=0, workspace=None, k_scale=None, v_scale=None, max_ctas=0,
                flags=0, stream=None) -> tuple:
    """The arguments of the C call paged_attention_decode for these tensors, in
    its order (see append_args)."""
    S, Hq, D = query.shape
    nb, bs, Hkv, _ = k_cache.shape
    mbps = block_table.shape[1]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return (_ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
            _ptr(seq_lens), S, Hq, Hkv, D, bs, mbps, nb, int(max_seq_len), float(scale),
            _dtype_code(query), _dtype_code(k_cache), _ptr(k_scale), _ptr(v_scale),
            int(partition_size), int(max_ctas), int(flags), _ptr(workspace), ws_bytes,
            _stream(stream))


def paged_attention_decode(out, query, k_cache, v_cache, block_table, seq_lens, *, max_seq_len,
                           scale, partition_size=0, workspace=None, k_scale=None, v_scale=None,
                           max_ctas=0, flags=0, stream=None) -> None:
    """out[i, j] = softmax attention of query[i, j] over sequence i's paged K/V;
    see paged_attention_decode in include/pagedkv.h."""
    st = load_library().paged_attention_decode(*decode_args(
        out, query, k_cache, v_cache, block_table, seq_lens, max_seq_len=max_seq_len, scale=scale,
        partition_size=partition_size, workspace=workspace, k_scale=k_scale, v_scale=v_scale,
        max_ctas=max_ctas, flags=flags, stream=stream))
    if st != 0:
        raise PagedKVError("paged_attention_decode", st)


def paged_attention_decode_static(out, query, k_cache, v_cache, block_table, seq_lens, *,
                                  max_seq_len, scale, partition_size=0, k_scale=None,
                                  v_scale=None, max_ctas=0, flags=0, stream=None) -> None:
    """paged_attention_decode with the library's own fixed scratch instead of a
    caller workspace, for callers that cannot allocate device memory; see
    paged_attention_decode_static in include/pagedkv.h (16 MiB limit, calls that
    overlap on the GPU race)."""
    lib = load_library()
    S, Hq, D = query.shape
    nb, bs, Hkv, _ = k_cache.shape
    mbps = block_table.shape[1]
    st = lib.paged_attention_decode_static(_ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache),
                                           _ptr(block_table), _ptr(seq_lens), S, Hq, Hkv, D, bs,
                                           mbps, nb, int(max_seq_len), float(scale),
                                           _dtype_code(query), _dtype_code(k_cache),
                                           _ptr(k_scale), _ptr(v_scale), int(partition_size),
                                           int(max_ctas), int(flags), _stream(stream))
    if st != 0:
        raise PagedKVError("paged_attention_decode_static", st)


def paged_attention_prefill(out, query, k_cache, v_cache, block_table, seq_lens, query_start, *,
                            max_q_len, scale, k_scale=None, v_scale=None, flags=0,
                            stream=None) -> None:
    """Causal attention of multi-token queries (chunked prefill, the uncached
    rest of a prefix-cache hit) over the paged cache; see
    paged_attention_prefill in include/pagedkv.h."""
    lib = load_library()
    T, Hq, D = query.shape
    nb, bs, Hkv, _ = k_cache.shape
    S = seq_lens.shape[0]
    st = lib.paged_attention_prefill(_ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache),
                                     _ptr(block_table), _ptr(seq_lens), _ptr(query_start), S, T,
                                     int(max_q_len), Hq, Hkv, D, bs, block_table.shape[1], nb,
                                     float(scale), _dtype_code(query), _dtype_code(k_cache),
                                     _ptr(k_scale), _ptr(v_scale), int(flags), _stream(stream))
    if st != 0:
        raise PagedKVError("paged_attention_prefill", st)


def _block_bytes(pool) -> int:
    return pool[0].numel() * pool.element_size() if pool.shape[0] else \
        int(torch.Size(pool.shape[1:]).numel()) * pool.element_size()


def paged_kv_copy_blocks(k_cache, v_cache, block_mapping, *, stream=None) -> None:
    """Copy-on-write copies inside one pool: for each row (src, dst) of
    block_mapping ([n, 2] int64, device), K[src] -> K[dst] and V[src] -> V[dst];
    see paged_kv_copy_blocks in include/pagedkv_blocks.h."""
    lib = load_library()
    n = block_mapping.shape[0]
    st = lib.paged_kv_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_mapping), n,
                                  _block_bytes(k_cache), k_cache.shape[0], _stream(stream))
    if st != 0:
        raise PagedKVError("paged_kv_copy_blocks", st)


def paged_kv_swap_blocks(src_k, src_v, dst_k, dst_v, block_mapping, *, stream=None) -> None:
    """Block copies between two pools of the same block shape, either of which
    may be pinned host memory (swap-out / swap-in); see paged_kv_swap_blocks in
    include/pagedkv_blocks.h."""
    lib = load_library()
    bb = _block_bytes(src_k)
    if _block_bytes(dst_k) != bb:
        raise ValueError("source and destination pools have different block shapes")
    n = block_mapping.shape[0]
    st = lib.paged_kv_swap_blocks(_ptr(src_k), _ptr(src_v), _ptr(dst_k), _ptr(dst_v),
                                  _ptr(block_mapping), n, bb, src_k.shape[0], dst_k.shape[0],
                                  _stream(stream))
    if st != 0:
        raise PagedKVError("paged_kv_swap_blocks", st)
