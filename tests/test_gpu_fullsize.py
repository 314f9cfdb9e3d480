"""The five decode workloads at their stated sizes, in the launch configuration
bench.py times, against the fp64 oracle element by element.

Each workload is drawn whole (no reduced copy) with spare blocks, tail slots
and this step's slots poisoned with NaN. One step is run as the benchmark runs
it: paged_kv_append of every sequence's new token, then paged_attention_decode
with the workload's partition size and a full wave of CTAs. The first decode
call zeroes the workspace counters; a second step then runs with the serving
flags (PKV_DECODE_ZEROED_WORKSPACE | PKV_DECODE_EARLY_START, the decode started
behind the append). After the append the whole pool must equal the oracle's
byte for byte; both decode outputs must be within the workload's tolerance of
the oracle over every (sequence, query head, dimension). The FP8 workload runs
at block sizes 8, 16 and 32. Errors are reported in the session summary."""
import numpy as np
import pytest
import torch

import paged_kv_cache_367_b200 as pkv
from paged_kv_cache_367_b200 import workloads as W
from parity import (assert_close, device_tables, host_pools, oracle_append, oracle_decode, scales,
                    to_f64)

pytestmark = pytest.mark.gpu

CASES = [("tiny", None), ("llama2_13b_mha", None), ("gqa70b", None), ("long_splitk", None),
         ("fp8_prefix", 8), ("fp8_prefix", 16), ("fp8_prefix", 32)]
SERVING = pkv.PKV_DECODE_ZEROED_WORKSPACE | pkv.PKV_DECODE_EARLY_START


@pytest.mark.parametrize("name,bs", CASES)
def test_stated_size_workload_matches_oracle(cuda_dev, name, bs, parity_report):
    cfg = W.CONFIGS[name]
    if bs is not None:
        cfg = cfg.replace(block_size=bs)
    wl = W.make_workload(cfg, device=cuda_dev, poison=True)
    c = wl.cfg
    kc, vc = host_pools(wl)
    oracle_append(wl, kc, vc)
    want = oracle_decode(wl, kc, vc)

    bt, lens, slots = device_tables(wl, cuda_dev)
    ks, vs = scales(wl, cuda_dev)
    P = c.partition_size
    nbytes = pkv.paged_attention_workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads,
                                                c.head_dim, wl.max_seq_len, P)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=cuda_dev) if nbytes else None
    outs = []
    for flags in (0, SERVING):
        out = torch.full(wl.query.shape, float("nan"), dtype=wl.query.dtype, device=cuda_dev)
        pkv.paged_kv_append(wl.new_key, wl.new_value, wl.k_cache, wl.v_cache, slots,
                            k_scale=ks, v_scale=vs)
        pkv.paged_attention_decode(out, wl.query, wl.k_cache, wl.v_cache, bt, lens,
                                   max_seq_len=wl.max_seq_len, scale=c.scale, partition_size=P,
                                   workspace=ws, k_scale=ks, v_scale=vs, flags=flags)
        torch.cuda.synchronize()
        outs.append(out)
        if flags == 0:
            assert np.array_equal(W.host(wl.k_cache).view(np.uint8), kc.view(np.uint8))
            assert np.array_equal(W.host(wl.v_cache).view(np.uint8), vc.view(np.uint8))
    label = f"{name} bs {c.block_size}: {c.num_seqs} seqs, {int(wl.seq_lens.sum())} tokens"
    for flags, out in zip(("plain", "serving flags"), outs):
        mx, mean = assert_close(to_f64(out), want, c, f"{label} ({flags})")
        parity_report.append(f"{label} ({flags}): max abs err {mx:.3e}, mean abs err {mean:.3e}")
