"""paged_kv_append through the C ABI vs the oracle: the whole pool must be
byte-identical after the append (bit-exact slot writes)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_367_b200 as pkv
from paged_kv_cache_367_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = [("f32", "f32", 64), ("f16", "f16", 128), ("bf16", "bf16", 128), ("bf16", "e4m3", 128),
         ("f16", "e4m3", 64), ("f32", "e4m3", 128), ("bf16", "bf16", 72)]


@pytest.mark.parametrize("src,cache,D", CASES)
def test_append_pool_bytes_match_oracle(cuda_dev, src, cache, D):
    rng = np.random.default_rng(hash((src, cache, D)) % 2**32)
    nb, bs, Hkv, T = 37, 16, 3, 50
    gen = torch.Generator(device=cuda_dev)
    gen.manual_seed(5)
    kc = W._randn((nb, bs, Hkv, D), cache, gen, cuda_dev)
    vc = W._randn((nb, bs, Hkv, D), cache, gen, cuda_dev)
    key = W._randn((T, Hkv, D), src, gen, cuda_dev)
    val = W._randn((T, Hkv, D), src, gen, cuda_dev)
    slots = rng.choice(nb * bs, T, replace=False).astype(np.int64)
    slots[::7] = -1                      # padding entries
    slots[3] = nb * bs + 5               # past the pool: ignored
    ks = float(key.float().abs().amax()) / 448.0
    vs = float(val.float().abs().amax()) / 448.0
    kc_h, vc_h = W.host(kc).copy(), W.host(vc).copy()
    oracle.append(W.host(key), W.host(val), kc_h, vc_h, slots, num_kv_heads=Hkv, head_dim=D,
                  block_size=bs, num_blocks=nb, src_dtype=src, cache_dtype=cache,
                  k_scale=ks, v_scale=vs)
    kst = torch.tensor([ks], dtype=torch.float32, device=cuda_dev)
    vst = torch.tensor([vs], dtype=torch.float32, device=cuda_dev)
    pkv.paged_kv_append(key, val, kc, vc, torch.from_numpy(slots).to(cuda_dev),
                        k_scale=kst, v_scale=vst)
    torch.cuda.synchronize()
    assert np.array_equal(W.host(kc).view(np.uint8), kc_h.view(np.uint8))
    assert np.array_equal(W.host(vc).view(np.uint8), vc_h.view(np.uint8))


def test_append_fp8_saturates_and_keeps_sign(cuda_dev):
    Hkv, D, nb, bs = 1, 64, 2, 8
    key = torch.zeros((1, Hkv, D), dtype=torch.float32, device=cuda_dev)
    key[0, 0, :8] = torch.tensor([1e6, -1e6, 448.0, 460.0, 470.0, -0.0, 1e-9, 2.0 ** -9])
    kc = torch.zeros((nb, bs, Hkv, D), dtype=torch.uint8, device=cuda_dev)
    vc = torch.zeros_like(kc)
    one = torch.ones(1, dtype=torch.float32, device=cuda_dev)
    pkv.paged_kv_append(key, key, kc, vc, torch.tensor([3], device=cuda_dev), k_scale=one,
                        v_scale=one)
    torch.cuda.synchronize()
    got = kc.view(-1, D)[3, :8].cpu().numpy()
    want = oracle.e4m3_encode(key[0, 0, :8].cpu().numpy())
    assert np.array_equal(got, want)
    assert got[0] == 0x7E and got[1] == 0xFE


def test_append_zero_tokens_is_a_no_op(cuda_dev):
    kc = torch.zeros((2, 8, 1, 64), dtype=torch.bfloat16, device=cuda_dev)
    key = torch.zeros((0, 1, 64), dtype=torch.bfloat16, device=cuda_dev)
    pkv.paged_kv_append(key, key, kc, kc, torch.zeros(0, dtype=torch.int64, device=cuda_dev))
    torch.cuda.synchronize()
    assert kc.abs().sum().item() == 0
