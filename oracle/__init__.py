"""CPU oracle for paged KV append and PagedAttention decode (TEST INFRASTRUCTURE).

A plain fp64 restatement of what the paged decode path computes, written in C
(``pagedkv_oracle.c``) and loaded here through ctypes. Only the test suite,
``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
this package; the product library never does, and the two share no code.

Pages followed (title, address, section):
  * "vLLM 推理引擎源码级拆解" (chenxutan.com/d/5333) §2.2 block-table figure and
    append into the last block, §2.3 PagedAttention kernel (per-token block-table
    walk, dot(q, k) * scale, softmax, write back; GQA/MQA).
  * "vLLM 深度实战" (chenxutan.com/d/3332) §1.2 Block / Block Table.
  * "vLLM 0.5 深度拆解" (chenxutan.com/d/4924) §4.2 FP8 KV cache, §2.3 chunked
    prefill (multi-token queries over the paged cache, causal).

Storage conventions of the arrays passed in (raw element storage, C order):
  f32 -> numpy float32, f16 -> numpy float16, bf16 -> numpy uint16 bit
  patterns, e4m3 -> numpy uint8 codes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pagedkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

DTYPE_CODES = {"f32": 0, "f16": 1, "bf16": 2, "e4m3": 3}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2, "e4m3": 1}

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into liboracle.so next to its source (gcc, OpenMP)."""
    stale = force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-std=c11", "-Wall", "-shared",
                               "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, I64, D, F = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                           ctypes.c_double, ctypes.c_float)
        lib.orc_e4m3_encode.argtypes = [F]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_value.restype = D
        lib.orc_e4m3_encode_array.argtypes = [P, P, I64]
        lib.orc_e4m3_encode_array.restype = None
        lib.orc_values_array.argtypes = [P, I, P, I64]
        lib.orc_values_array.restype = None
        lib.orc_num_blocks.argtypes = [I64, I]
        lib.orc_num_blocks.restype = I64
        lib.orc_slot_of_token.argtypes = [P, I64, I]
        lib.orc_slot_of_token.restype = I64
        lib.orc_append.argtypes = [P, P, P, P, P, I, I, I, I, I64, I, I, F, F]
        lib.orc_append.restype = I
        lib.orc_decode_items.argtypes = [P, P, I64, P, P, P, P, P, I, I, I, I, I, I64, D,
                                         I, I, D, D, I]
        lib.orc_decode_items.restype = I
        lib.orc_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I64, D, I, I, D, D, I]
        lib.orc_decode.restype = I
        lib.orc_prefill_items.argtypes = [P, P, I64, P, P, P, P, P, P, I, I, I, I, I, I, I64,
                                          D, I, I, D, D, I]
        lib.orc_prefill_items.restype = I
        _lib = lib
    return _lib


def _c(a: np.ndarray) -> np.ndarray:
    if not a.flags["C_CONTIGUOUS"]:
        raise ValueError("oracle arrays must be C-contiguous")
    return a


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(_c(a).ctypes.data)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """E4M3 codes of binary32 values: nearest-even, saturating to +-448, NaN -> 0x7F."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    _load().orc_e4m3_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def values(raw: np.ndarray, dtype: str) -> np.ndarray:
    """Exact fp64 values of raw element storage of the given dtype."""
    raw = np.ascontiguousarray(raw)
    n = raw.nbytes // ELEM_BYTES[dtype]
    out = np.empty(n, dtype=np.float64)
    _load().orc_values_array(_ptr(raw), DTYPE_CODES[dtype], _ptr(out), n)
    return out.reshape(raw.shape) if raw.size == n else out


def num_blocks_for(seq_len: int, block_size: int) -> int:
    """Blocks occupied by a sequence: ceil(seq_len / block_size)."""
    return int(_load().orc_num_blocks(seq_len, block_size))


def slot_of_token(block_table_row: np.ndarray, tok: int, block_size: int) -> int:
    """physical_block * block_size + offset for token `tok` of one sequence."""
    row = np.ascontiguousarray(block_table_row, dtype=np.int32)
    return int(_load().orc_slot_of_token(_ptr(row), tok, block_size))


def append(key, value, k_cache, v_cache, slot_mapping, *, num_kv_heads, head_dim,
           block_size, num_blocks, src_dtype, cache_dtype, k_scale=1.0, v_scale=1.0):
    """Write each token's K/V row into its slot of the host caches (in place)."""
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    r = _load().orc_append(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                           _ptr(slot_mapping), len(slot_mapping), num_kv_heads, head_dim,
                           block_size, num_blocks, DTYPE_CODES[src_dtype],
                           DTYPE_CODES[cache_dtype], float(k_scale), float(v_scale))
    if r != 0:
        raise ValueError("oracle append: unsupported dtype pair")


def decode(query, k_cache, v_cache, block_table, seq_lens, *, num_heads, num_kv_heads,
           head_dim, block_size, scale, q_dtype, cache_dtype, k_scale=1.0, v_scale=1.0,
           items=None, threads=0, num_blocks=None):
    """fp64 paged decode attention.

    `scale`, `k_scale` and `v_scale` are rounded to binary32 first, as the
    library receives them. Returns (out, threads_used). Without `items`, out is [num_seqs, num_heads,
    head_dim]; with `items` (an [n, 2] array of (sequence, query head)), out is
    [n, head_dim] in item order.
    """
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    # The library takes the softmax and KV scales as binary32; so does the oracle.
    scale, k_scale, v_scale = (float(np.float32(x)) for x in (scale, k_scale, v_scale))
    S, mbps = block_table.shape
    nb = num_blocks if num_blocks is not None else k_cache.shape[0]
    lib = _load()
    common = (_ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens))
    if items is None:
        out = np.empty((S, num_heads, head_dim), dtype=np.float64)
        used = lib.orc_decode(_ptr(out), *common, S, num_heads, num_kv_heads, head_dim,
                              block_size, mbps, nb, float(scale), DTYPE_CODES[q_dtype],
                              DTYPE_CODES[cache_dtype], float(k_scale), float(v_scale),
                              int(threads))
    else:
        items = np.ascontiguousarray(items, dtype=np.int32).reshape(-1, 2)
        out = np.empty((len(items), head_dim), dtype=np.float64)
        used = lib.orc_decode_items(_ptr(out), _ptr(items), len(items), *common, num_heads,
                                    num_kv_heads, head_dim, block_size, mbps, nb, float(scale),
                                    DTYPE_CODES[q_dtype], DTYPE_CODES[cache_dtype],
                                    float(k_scale), float(v_scale), int(threads))
    if used < 0:
        raise ValueError("oracle decode: num_heads must be a multiple of num_kv_heads")
    return out, used


def prefill(query, k_cache, v_cache, block_table, seq_lens, query_start, *, num_heads,
            num_kv_heads, head_dim, block_size, scale, q_dtype, cache_dtype, k_scale=1.0,
            v_scale=1.0, items=None, threads=0, num_blocks=None):
    """fp64 causal attention of multi-token queries over the paged cache.

    query is [num_q_tokens, num_heads, head_dim]; rows query_start[i] ..
    query_start[i+1]-1 are the last tokens of sequence i (whose seq_lens[i]
    cached tokens include them), and each attends over the tokens up to its own
    position. Returns (out, threads_used): out is [num_q_tokens, num_heads,
    head_dim], or [n, head_dim] for `items` (an [n, 2] array of (row, query head)).
    """
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    query_start = np.ascontiguousarray(query_start, dtype=np.int32)
    scale, k_scale, v_scale = (float(np.float32(x)) for x in (scale, k_scale, v_scale))
    S, mbps = block_table.shape
    T = int(query_start[-1])
    nb = num_blocks if num_blocks is not None else k_cache.shape[0]
    if items is None:
        items = np.stack(np.meshgrid(np.arange(T), np.arange(num_heads), indexing="ij"),
                         -1).reshape(-1, 2)
        shape = (T, num_heads, head_dim)
    else:
        shape = (len(items), head_dim)
    items = np.ascontiguousarray(items, dtype=np.int32).reshape(-1, 2)
    out = np.empty((len(items), head_dim), dtype=np.float64)
    used = _load().orc_prefill_items(
        _ptr(out), _ptr(items), len(items), _ptr(query), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_table), _ptr(seq_lens), _ptr(query_start), S, num_heads, num_kv_heads,
        head_dim, block_size, mbps, nb, float(scale), DTYPE_CODES[q_dtype],
        DTYPE_CODES[cache_dtype], float(k_scale), float(v_scale), int(threads))
    if used < 0:
        raise ValueError("oracle prefill: num_heads must be a multiple of num_kv_heads")
    return out.reshape(shape), used
