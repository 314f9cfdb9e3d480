"""paged_attention_decode (after paged_kv_append) through the C ABI vs the fp64
oracle on the five workloads, at sizes the oracle finishes in seconds (several
tiles and ragged tails), plus invariants and edge cases on the GPU."""
import numpy as np
import pytest
import torch

import paged_kv_cache_367_b200 as pkv
from paged_kv_cache_367_b200 import workloads as W
from parity import (assert_close, gpu_step, host_pools, oracle_append, oracle_decode, to_f64,
                    tolerance)

pytestmark = pytest.mark.gpu

C = W.CONFIGS
SMALL = {
    "tiny": C["tiny"],
    "llama2_13b_mha": C["llama2_13b_mha"].replace(num_seqs=6, lens=("uniform", 128, 700)),
    "gqa70b": C["gqa70b"].replace(num_seqs=10, lens=("lognormal", 600, 0.8, 16, 1500)),
    "long_splitk": C["long_splitk"].replace(num_seqs=2, lens=("uniform", 4096, 9000)),
    "fp8_prefix": C["fp8_prefix"].replace(num_seqs=8),
}
FLAGS = [0, pkv.PKV_DECODE_FORCE_SIMT]


def _check(cfg, dev, **kw):
    wl = W.make_workload(cfg, device=dev, poison=True)
    kc, vc = host_pools(wl)
    oracle_append(wl, kc, vc)
    out = gpu_step(wl, dev, **kw)
    # The append left the pool byte-identical to the oracle's.
    assert np.array_equal(W.host(wl.k_cache).view(np.uint8), kc.view(np.uint8))
    assert np.array_equal(W.host(wl.v_cache).view(np.uint8), vc.view(np.uint8))
    want = oracle_decode(wl, kc, vc)
    return assert_close(to_f64(out), want, cfg, cfg.name)


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("flags", FLAGS)
def test_workload_parity(cuda_dev, name, flags):
    _check(SMALL[name], cuda_dev, flags=flags)


@pytest.mark.parametrize("name", ["llama2_13b_mha", "gqa70b", "long_splitk"])
@pytest.mark.parametrize("partition_size,max_ctas", [(0, 0), (32, 0), (512, 3), (64, 1), (256, 1000)])
def test_split_and_grid_variants(cuda_dev, name, partition_size, max_ctas):
    cfg = SMALL[name]
    if partition_size % cfg.block_size:
        partition_size = cfg.block_size * max(1, partition_size // cfg.block_size)
    _check(cfg, cuda_dev, partition_size=partition_size, max_ctas=max_ctas)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_fp8_prefix_block_sizes(cuda_dev, bs):
    _check(SMALL["fp8_prefix"].replace(block_size=bs), cuda_dev)


@pytest.mark.parametrize("bs", [8, 32])
@pytest.mark.parametrize("flags", FLAGS)
def test_bf16_block_sizes(cuda_dev, bs, flags):
    _check(SMALL["gqa70b"].replace(block_size=bs), cuda_dev, flags=flags)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 4), (24, 2), (16, 1), (32, 2)])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_group_sizes(cuda_dev, Hq, Hkv, dt):
    cfg = C["gqa70b"].replace(num_seqs=5, num_heads=Hq, num_kv_heads=Hkv, q_dtype=dt,
                              cache_dtype=dt, lens=("uniform", 1, 300), head_dim=64,
                              partition_size=64, seed=77)
    _check(cfg, cuda_dev)


@pytest.mark.parametrize("S", [150, 192, 193, 256, 257, 600])
@pytest.mark.parametrize("flags", FLAGS)
def test_many_sequences(cuda_dev, S, flags):
    # Batches larger than a CTA (one sequence per thread) take the multi-pass
    # schedule set-up; zero lengths are mixed in.
    cfg = C["gqa70b"].replace(num_seqs=S, lens=("uniform", 0, 200), partition_size=64, seed=S)
    _check(cfg, cuda_dev, flags=flags)


@pytest.mark.parametrize("L,P", [(40000, 64), (9000, 32), (3000, 16)])
@pytest.mark.parametrize("flags", FLAGS)
def test_unit_split_into_many_pieces(cuda_dev, L, P, flags):
    # One sequence with one KV head spread over every CTA: the merge of its
    # partials takes more pieces than a warp has lanes.
    cfg = C["gqa70b"].replace(num_seqs=1, num_heads=8, num_kv_heads=1, lens=("fixed", [L]),
                              partition_size=P, seed=5)
    _check(cfg, cuda_dev, flags=flags)


def test_permutation_of_physical_blocks_is_bit_identical(cuda_dev):
    cfg = SMALL["gqa70b"]
    wl = W.make_workload(cfg, device=cuda_dev)
    out1 = gpu_step(wl, cuda_dev)
    perm = torch.randperm(wl.num_blocks, generator=torch.Generator().manual_seed(3))
    kc2 = torch.empty_like(wl.k_cache)
    vc2 = torch.empty_like(wl.v_cache)
    kc2[perm.to(cuda_dev)] = wl.k_cache
    vc2[perm.to(cuda_dev)] = wl.v_cache
    bt2 = np.where(wl.block_table >= 0, perm.numpy()[np.maximum(wl.block_table, 0)], -1)
    wl.k_cache, wl.v_cache = kc2, vc2
    out2 = gpu_step(wl, cuda_dev, append=False, block_table=bt2.astype(np.int32))
    assert torch.equal(out1, out2)


def test_shared_prefix_equals_duplicated_blocks_bit_identical(cuda_dev):
    cfg = SMALL["fp8_prefix"].replace(cache_dtype="bf16")
    wl = W.make_workload(cfg, device=cuda_dev)
    out1 = gpu_step(wl, cuda_dev)
    pre = cfg.prefix_len // cfg.block_size
    shared = wl.block_table[0, :pre].copy()
    extra = cfg.num_seqs * pre
    nb2 = wl.num_blocks + extra
    kc2 = torch.empty((nb2,) + tuple(wl.k_cache.shape[1:]), dtype=wl.k_cache.dtype, device=cuda_dev)
    vc2 = torch.empty_like(kc2)
    kc2[:wl.num_blocks] = wl.k_cache
    vc2[:wl.num_blocks] = wl.v_cache
    bt2 = wl.block_table.copy()
    for i in range(cfg.num_seqs):
        ids = np.arange(wl.num_blocks + i * pre, wl.num_blocks + (i + 1) * pre)
        kc2[torch.from_numpy(ids).to(cuda_dev)] = wl.k_cache[torch.from_numpy(shared).long().to(cuda_dev)]
        vc2[torch.from_numpy(ids).to(cuda_dev)] = wl.v_cache[torch.from_numpy(shared).long().to(cuda_dev)]
        bt2[i, :pre] = ids
    wl.k_cache, wl.v_cache = kc2, vc2
    out2 = gpu_step(wl, cuda_dev, append=False, block_table=bt2)
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("dt", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("flags", FLAGS)
def test_single_token_returns_the_v_row_exactly(cuda_dev, dt, flags):
    cfg = C["gqa70b"].replace(num_seqs=3, q_dtype=dt, cache_dtype=dt, lens=("fixed", [1, 1, 1]),
                              seed=21)
    wl = W.make_workload(cfg, device=cuda_dev)
    out = gpu_step(wl, cuda_dev, flags=flags)
    g = cfg.num_heads // cfg.num_kv_heads
    want = wl.new_value.repeat_interleave(g, dim=1)
    assert torch.equal(out, want)


def test_zero_length_sequences_give_zeros(cuda_dev):
    cfg = SMALL["gqa70b"].replace(num_seqs=4, lens=("fixed", [0, 40, 0, 3]))
    wl = W.make_workload(cfg, device=cuda_dev, poison=True)
    kc, vc = host_pools(wl)
    sl = wl.slot_mapping.copy()
    wl.slot_mapping = sl
    oracle_append(wl, kc, vc)
    out = gpu_step(wl, cuda_dev)
    assert torch.all(out[0] == 0) and torch.all(out[2] == 0)
    want = oracle_decode(wl, kc, vc)
    assert_close(to_f64(out), want, cfg)


def test_all_sequences_empty(cuda_dev):
    cfg = SMALL["gqa70b"].replace(num_seqs=3, lens=("fixed", [0, 0, 0]))
    wl = W.make_workload(cfg, device=cuda_dev)
    out = gpu_step(wl, cuda_dev, append=False, max_seq_len=16)
    assert torch.all(out == 0)


def test_seq_lens_are_clamped_to_the_table(cuda_dev):
    cfg = SMALL["gqa70b"].replace(num_seqs=4, lens=("fixed", [40, 17, 64, 5]))
    wl = W.make_workload(cfg, device=cuda_dev)
    kc, vc = host_pools(wl)
    oracle_append(wl, kc, vc)
    gpu_step(wl, cuda_dev)                          # append once
    big = wl.seq_lens.copy()
    big[1] = 10_000                                  # past max_blocks_per_seq * bs
    big[3] = -5
    out = gpu_step(wl, cuda_dev, append=False, seq_lens=big, max_seq_len=10_000)
    clamped = np.clip(big, 0, wl.max_blocks_per_seq * cfg.block_size).astype(np.int32)
    want = oracle_decode(wl, kc, vc, seq_lens=clamped)
    assert_close(to_f64(out), want, cfg)
    # The clamped length reaches the table's unused (-1) entries: reported.
    assert pkv.pkv_device_status(clear=True) == 2


def test_block_ids_outside_the_pool_read_as_zeros(cuda_dev):
    cfg = SMALL["gqa70b"].replace(num_seqs=3, lens=("fixed", [50, 33, 70]))
    wl = W.make_workload(cfg, device=cuda_dev)
    kc, vc = host_pools(wl)
    oracle_append(wl, kc, vc)
    gpu_step(wl, cuda_dev)
    bt = wl.block_table.copy()
    bt[0, 1] = wl.num_blocks + 3
    bt[2, 0] = -9
    for flags in FLAGS:
        out = gpu_step(wl, cuda_dev, append=False, block_table=bt, flags=flags)
        want = oracle_decode(wl, kc, vc, block_table=bt)
        assert_close(to_f64(out), want, cfg)
        assert pkv.pkv_device_status(clear=True) == 2  # the corrupt entries are reported


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (32, 8), (64, 8), (16, 1)])
@pytest.mark.parametrize("qdt", ["bf16", "f16"])
@pytest.mark.parametrize("flags", FLAGS)
def test_fp8_cache_group_sizes(cuda_dev, Hq, Hkv, qdt, flags):
    cfg = C["fp8_prefix"].replace(num_seqs=5, num_heads=Hq, num_kv_heads=Hkv, q_dtype=qdt,
                                  lens=("uniform", 1, 400), prefix_len=0, partition_size=64,
                                  seed=91)
    _check(cfg, cuda_dev, flags=flags)


@pytest.mark.parametrize("qdt", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("flags", FLAGS)
def test_fp8_cache_head_dims_and_query_dtypes(cuda_dev, qdt, D, flags):
    # head_dim 64 over an E4M3 cache runs the CUDA-core kernel; so does an fp32
    # query over an E4M3 cache (the new tokens are quantised from fp32 too).
    cfg = C["fp8_prefix"].replace(num_seqs=6, num_heads=32, num_kv_heads=8, head_dim=D,
                                  q_dtype=qdt, lens=("uniform", 1, 500), prefix_len=0,
                                  partition_size=64, seed=93 + D)
    _check(cfg, cuda_dev, flags=flags)


PRODUCTS = [pkv.PKV_DECODE_TENSOR_CORES, pkv.PKV_DECODE_CUDA_CORES]


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 8), (12, 4), (16, 4), (32, 4), (16, 16)])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("flags", PRODUCTS)
def test_products_on_tensor_or_cuda_cores(cuda_dev, Hq, Hkv, D, dt, flags):
    # The TMA-fed kernel with its products on the tensor cores (mma.sync) or on
    # the CUDA cores (groups of up to 4 heads; wider ones stay on the tensor
    # cores), split and unsplit sequences, ragged tails.
    cfg = C["gqa70b"].replace(num_seqs=7, num_heads=Hq, num_kv_heads=Hkv, head_dim=D, q_dtype=dt,
                              cache_dtype=dt, lens=("uniform", 1, 700), partition_size=128,
                              seed=Hq * 3 + Hkv + D)
    _check(cfg, cuda_dev, flags=flags)


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("flags", PRODUCTS)
def test_mha_products_block_sizes(cuda_dev, bs, flags):
    _check(SMALL["llama2_13b_mha"].replace(block_size=bs), cuda_dev, flags=flags)


@pytest.mark.parametrize("flags", PRODUCTS)
def test_mha_products_single_token_exact(cuda_dev, flags):
    cfg = C["llama2_13b_mha"].replace(num_seqs=3, lens=("fixed", [1, 1, 1]), seed=22)
    wl = W.make_workload(cfg, device=cuda_dev)
    out = gpu_step(wl, cuda_dev, flags=flags)
    assert torch.equal(out, wl.new_value)
