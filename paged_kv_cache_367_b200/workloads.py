"""Seeded synthetic inputs for paged decode (shared by the tests and the benchmark).

This module only draws inputs: sequence lengths, a shuffled physical block pool
with per-sequence block tables, the slot each sequence's new token goes to, and
random Q/K/V data already cast to its storage dtype. It performs none of the
attention arithmetic. The CUDA library and the CPU oracle both take its output.

Workload shapes follow the pages' examples: Llama-2-13B (40 layers x 40 KV
heads x 128, fp16) from the KV-bytes formula in "vLLM 推理引擎源码级拆解"
(chenxutan.com/d/5333) §1, 16-token blocks and shuffled physical blocks from its
§2.1-2.2 figure, block sizes 8/16/32 from its §7, and FP8 KV from "vLLM 0.5 深度
拆解" (chenxutan.com/d/4924) §4.2.

Recipe:
  * lengths: numpy PCG64 seeded with the config seed; uniform integers, or
    lognormal round(exp(N(ln median, sigma))) clipped to [lo, hi];
  * pool: enough blocks for every sequence plus 10% spare (or a fixed pool
    size); physical ids are a seeded permutation of the pool; unused
    block-table entries are -1; a shared prefix uses the same physical blocks
    at the head of every sequence's table;
  * data: torch.Generator seeded with the config seed; Q, K pool, V pool, new K,
    new V drawn N(0, 1) in fp32 and cast (round to nearest even) to the storage
    dtype. FP8 pools are drawn in the code domain, N(0, (448/5)^2) clipped to
    +-448 and cast to E4M3, with k_scale = v_scale = 5/448, so the dequantised
    values are about N(0, 1);
  * poison (parity runs): spare blocks, slots past each sequence's length, and
    the slot of the token appended this step hold NaN, so a stray read or a
    missing append shows up in the output.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import numpy as np
import torch

TORCH_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16,
                "e4m3": torch.uint8}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2, "e4m3": 1}
FP8_CODE_SIGMA = 448.0 / 5.0
FP8_SCALE = 5.0 / 448.0


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    q_dtype: str
    cache_dtype: str
    lens: tuple
    partition_size: int = 0
    pool_blocks: int = 0
    prefix_len: int = 0
    seed: int = 1000

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def replace(self, **kw) -> "DecodeConfig":
        return dataclasses.replace(self, **kw)


# The five workloads. Sizes are the pages' model shapes (see module docstring).
CONFIGS = {
    "tiny": DecodeConfig("tiny", 4, 8, 8, 64, 16, "f32", "f32", ("uniform", 1, 100),
                         partition_size=0, pool_blocks=64, seed=1001),
    "llama2_13b_mha": DecodeConfig("llama2_13b_mha", 64, 40, 40, 128, 16, "f16", "f16",
                                   ("uniform", 128, 2048), partition_size=512, seed=1002),
    "gqa70b": DecodeConfig("gqa70b", 128, 64, 8, 128, 16, "bf16", "bf16",
                           ("lognormal", 1024, 0.8, 16, 8192), partition_size=256, seed=1003),
    "long_splitk": DecodeConfig("long_splitk", 8, 32, 8, 128, 32, "bf16", "bf16",
                                ("uniform", 32768, 131072), partition_size=512, seed=1004),
    "fp8_prefix": DecodeConfig("fp8_prefix", 64, 32, 8, 128, 16, "bf16", "e4m3",
                               ("uniform", 16, 512), partition_size=256, prefix_len=1024,
                               seed=1005),
}


def draw_seq_lens(cfg: DecodeConfig, rng: np.random.Generator) -> np.ndarray:
    kind = cfg.lens[0]
    if kind == "uniform":
        lo, hi = cfg.lens[1], cfg.lens[2]
        lens = rng.integers(lo, hi + 1, size=cfg.num_seqs)
    elif kind == "lognormal":
        median, sigma, lo, hi = cfg.lens[1:]
        lens = np.clip(np.rint(np.exp(rng.normal(math.log(median), sigma, cfg.num_seqs))), lo, hi)
    elif kind == "fixed":
        lens = np.asarray(cfg.lens[1], dtype=np.int64).reshape(-1)
        assert len(lens) == cfg.num_seqs
    else:
        raise ValueError(kind)
    return (lens + cfg.prefix_len).astype(np.int32)


@dataclass
class Workload:
    cfg: DecodeConfig
    seq_lens: np.ndarray        # [S] int32
    block_table: np.ndarray     # [S, max_blocks_per_seq] int32, -1 = unused
    slot_mapping: np.ndarray    # [S] int64: slot of each sequence's newest token
    num_blocks: int
    query: torch.Tensor         # [S, Hq, D]
    k_cache: torch.Tensor       # [num_blocks, bs, Hkv, D]
    v_cache: torch.Tensor
    new_key: torch.Tensor       # [S, Hkv, D], query dtype
    new_value: torch.Tensor
    k_scale: float
    v_scale: float

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max()) if len(self.seq_lens) else 0

    @property
    def max_blocks_per_seq(self) -> int:
        return self.block_table.shape[1]


def host(t: torch.Tensor) -> np.ndarray:
    """Raw element storage of a tensor as a numpy array (bf16 as uint16 bits)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _alloc_tables(cfg: DecodeConfig, lens: np.ndarray, rng: np.random.Generator):
    bs = cfg.block_size
    nbs = [-(-int(L) // bs) for L in lens]
    prefix_blocks = cfg.prefix_len // bs
    assert cfg.prefix_len % bs == 0
    needed = prefix_blocks + sum(n - prefix_blocks for n in nbs)
    num_blocks = cfg.pool_blocks or (needed + max(1, needed // 10))
    assert num_blocks >= needed, "pool too small"
    ids = rng.permutation(num_blocks).astype(np.int32)
    mbps = max(nbs) if nbs else 1
    table = np.full((cfg.num_seqs, max(mbps, 1)), -1, dtype=np.int32)
    shared = ids[:prefix_blocks]
    nxt = prefix_blocks
    for i, n in enumerate(nbs):
        table[i, :prefix_blocks] = shared
        own = n - prefix_blocks
        table[i, prefix_blocks:n] = ids[nxt:nxt + own]
        nxt += own
    slots = np.array([int(table[i, (L - 1) // bs]) * bs + (L - 1) % bs if L > 0 else -1
                      for i, L in enumerate(lens)], dtype=np.int64)
    return table, slots, num_blocks, ids[nxt:]


def _randn(shape, dtype: str, gen: torch.Generator, device) -> torch.Tensor:
    """N(0,1) fp32 cast to the storage dtype; drawn in chunks over dim 0."""
    out = torch.empty(shape, dtype=TORCH_DTYPES[dtype], device=device)
    rows = shape[0]
    per_row = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    step = max(1, (1 << 26) // max(per_row, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        x = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen, device=device,
                        dtype=torch.float32)
        if dtype == "e4m3":
            x = (x * FP8_CODE_SIGMA).clamp_(-448.0, 448.0)
            out[r0:r1] = x.to(torch.float8_e4m3fn).view(torch.uint8)
        else:
            out[r0:r1] = x.to(TORCH_DTYPES[dtype])
    return out


def _nan_fill(t: torch.Tensor, dtype: str):
    if dtype == "e4m3":
        t.fill_(0x7F)
    else:
        t.fill_(float("nan"))


def make_workload(cfg: DecodeConfig, device="cpu", poison: bool = False,
                  seq_lens=None) -> Workload:
    """Draw one workload. `seq_lens` (optional) overrides the drawn lengths."""
    rng = np.random.default_rng(cfg.seed)
    lens = draw_seq_lens(cfg, rng)
    if seq_lens is not None:
        lens = np.asarray(seq_lens, dtype=np.int32).reshape(-1)
        cfg = cfg.replace(num_seqs=len(lens))
    table, slots, num_blocks, spare = _alloc_tables(cfg, lens, rng)
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed)
    S, Hq, Hkv, D, bs = cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    query = _randn((S, Hq, D), cfg.q_dtype, gen, device)
    k_cache = _randn((num_blocks, bs, Hkv, D), cfg.cache_dtype, gen, device)
    v_cache = _randn((num_blocks, bs, Hkv, D), cfg.cache_dtype, gen, device)
    new_key = _randn((S, Hkv, D), cfg.q_dtype, gen, device)
    new_value = _randn((S, Hkv, D), cfg.q_dtype, gen, device)
    scale8 = FP8_SCALE if cfg.cache_dtype == "e4m3" else 1.0
    if poison:
        flat_k = k_cache.view(num_blocks * bs, Hkv, D)
        flat_v = v_cache.view(num_blocks * bs, Hkv, D)
        bad = []
        for blk in spare.tolist():
            bad.extend(range(blk * bs, blk * bs + bs))
        for i, L in enumerate(lens.tolist()):
            if L <= 0:
                continue
            last = int(table[i, (L - 1) // bs])
            bad.extend(last * bs + off for off in range((L - 1) % bs + 1, bs))
            bad.append(int(slots[i]))
        if bad:
            idx = torch.as_tensor(sorted(set(bad)), dtype=torch.long, device=device)
            pk = flat_k[idx]
            _nan_fill(pk, cfg.cache_dtype)
            flat_k[idx] = pk
            flat_v[idx] = pk
    return Workload(cfg, lens, table, slots, num_blocks, query, k_cache, v_cache,
                    new_key, new_value, scale8, scale8)
