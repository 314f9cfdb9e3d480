"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
binding and the CPU oracle on the same seeded workload, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_367_b200 as pkv
from paged_kv_cache_367_b200 import workloads as W

# Tolerances against the fp64 oracle (max abs, mean abs).
TOL = {"f32": (1e-4, 1e-5), "f16": (1e-2, 1e-3), "bf16": (1e-2, 1e-3), "e4m3": (3e-2, 3e-3)}


def tolerance(cfg):
    return TOL["e4m3"] if cfg.cache_dtype == "e4m3" else TOL[cfg.q_dtype]


def device_tables(wl, dev):
    bt = torch.from_numpy(wl.block_table).to(dev)
    lens = torch.from_numpy(wl.seq_lens).to(dev)
    slots = torch.from_numpy(wl.slot_mapping).to(dev)
    return bt, lens, slots


def scales(wl, dev):
    if wl.cfg.cache_dtype != "e4m3":
        return None, None
    return (torch.tensor([wl.k_scale], dtype=torch.float32, device=dev),
            torch.tensor([wl.v_scale], dtype=torch.float32, device=dev))


def gpu_step(wl, dev, *, partition_size=None, max_ctas=0, flags=0, append=True,
             seq_lens=None, max_seq_len=None, block_table=None):
    """Append each sequence's new token (optional), then decode. Returns out (device)."""
    cfg = wl.cfg
    bt, lens, slots = device_tables(wl, dev)
    if block_table is not None:
        bt = torch.as_tensor(block_table, dtype=torch.int32).to(dev)
    if seq_lens is not None:
        lens = torch.as_tensor(seq_lens, dtype=torch.int32).to(dev)
    ks, vs = scales(wl, dev)
    if append:
        pkv.paged_kv_append(wl.new_key, wl.new_value, wl.k_cache, wl.v_cache, slots,
                            k_scale=ks, v_scale=vs)
    P = cfg.partition_size if partition_size is None else partition_size
    msl = wl.max_seq_len if max_seq_len is None else max_seq_len
    ws_bytes = pkv.paged_attention_workspace_size(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads,
                                                  cfg.head_dim, msl, P)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    out = torch.full(wl.query.shape, float("nan"), dtype=wl.query.dtype, device=dev)
    pkv.paged_attention_decode(out, wl.query, wl.k_cache, wl.v_cache, bt, lens,
                               max_seq_len=msl, scale=cfg.scale, partition_size=P,
                               workspace=ws if ws_bytes else None, k_scale=ks, v_scale=vs,
                               max_ctas=max_ctas, flags=flags)
    torch.cuda.synchronize()
    return out


def host_pools(wl):
    return W.host(wl.k_cache).copy(), W.host(wl.v_cache).copy()


def oracle_append(wl, kc, vc):
    cfg = wl.cfg
    oracle.append(W.host(wl.new_key), W.host(wl.new_value), kc, vc, wl.slot_mapping,
                  num_kv_heads=cfg.num_kv_heads, head_dim=cfg.head_dim,
                  block_size=cfg.block_size, num_blocks=wl.num_blocks, src_dtype=cfg.q_dtype,
                  cache_dtype=cfg.cache_dtype, k_scale=wl.k_scale, v_scale=wl.v_scale)


def oracle_decode(wl, kc, vc, items=None, seq_lens=None, block_table=None):
    cfg = wl.cfg
    out, _ = oracle.decode(W.host(wl.query), kc, vc,
                           wl.block_table if block_table is None else block_table,
                           wl.seq_lens if seq_lens is None else seq_lens,
                           num_heads=cfg.num_heads, num_kv_heads=cfg.num_kv_heads,
                           head_dim=cfg.head_dim, block_size=cfg.block_size, scale=cfg.scale,
                           q_dtype=cfg.q_dtype, cache_dtype=cfg.cache_dtype,
                           k_scale=wl.k_scale, v_scale=wl.v_scale, items=items)
    return out


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, want: np.ndarray):
    err = np.abs(got - want)
    return float(np.max(err)) if err.size else 0.0, float(np.mean(err)) if err.size else 0.0


def assert_close(got: np.ndarray, want: np.ndarray, cfg, what=""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, mean = errors(got, want)
    tmax, tmean = tolerance(cfg)
    assert mx <= tmax and mean <= tmean, f"{what}: max {mx:.3g} (tol {tmax}), mean {mean:.3g} (tol {tmean})"
    return mx, mean
