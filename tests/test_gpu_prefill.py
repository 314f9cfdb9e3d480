"""paged_attention_prefill (causal multi-token queries over the paged cache)
through the C ABI against the fp64 oracle: full prefills, chunks continuing a
cached context, GQA/MQA group sizes, head dims, block sizes, dtypes, and the
edge cases (poisoned slots past the range, out-of-pool ids, chunks longer than
max_q_len, chunks longer than their context)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_367_b200 as pkv
from paged_kv_cache_367_b200 import workloads as W
from parity import TOL

pytestmark = pytest.mark.gpu

TORCH = {"bf16": torch.bfloat16, "f16": torch.float16}


def make_case(lens, qlens, Hq, Hkv, D, bs, dt, dev, seed=0, spare=5, cache=None):
    """Pools for the given lengths (cache: None = the query dtype, or "e4m3":
    codes drawn as in workloads.py with k_scale = v_scale = 5/448)."""
    rng = np.random.default_rng(seed)
    gen = torch.Generator().manual_seed(seed)
    nbs = [-(-L // bs) for L in lens]
    nb = sum(nbs) + spare
    ids = rng.permutation(nb)
    mbps = max(nbs + [1])
    bt = np.full((len(lens), mbps), -1, np.int32)
    n = 0
    for i, k in enumerate(nbs):
        bt[i, :k] = ids[n:n + k]
        n += k
    cache = cache or dt
    if cache == "e4m3":
        def codes():
            x = (torch.randn((nb, bs, Hkv, D), generator=gen) * W.FP8_CODE_SIGMA).clamp(-448, 448)
            return x.to(torch.float8_e4m3fn).view(torch.uint8)
        kc, vc = codes(), codes()
    else:
        kc = torch.randn((nb, bs, Hkv, D), generator=gen).to(TORCH[dt])
        vc = torch.randn((nb, bs, Hkv, D), generator=gen).to(TORCH[dt])
    # Slots past every sequence's length hold NaN: they must never reach the output.
    used = np.zeros((nb, bs), bool)
    for i, L in enumerate(lens):
        for t in range(L):
            used[bt[i, t // bs], t % bs] = True
    mask = torch.from_numpy(~used)
    nan = 0x7F if cache == "e4m3" else float("nan")
    kc[mask] = nan
    vc[mask] = nan
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = torch.randn((int(qs[-1]), Hq, D), generator=gen).to(TORCH[dt])
    sc = W.FP8_SCALE if cache == "e4m3" else 1.0
    return dict(kc=kc.to(dev), vc=vc.to(dev), bt=bt, lens=np.asarray(lens, np.int32), qs=qs,
                q=q.to(dev), Hq=Hq, Hkv=Hkv, D=D, bs=bs, dt=dt, dev=dev, cache=cache, sc=sc)


def run_gpu(c, max_q_len=None, bt=None, fill=float("nan"), status=0, flags=0):
    dev = c["dev"]
    out = torch.full(tuple(c["q"].shape), fill, dtype=c["q"].dtype, device=dev)
    bt = c["bt"] if bt is None else bt
    mq = int(np.diff(c["qs"]).max()) if max_q_len is None else max_q_len
    ks = vs = None
    if c["cache"] == "e4m3":
        ks = torch.tensor([c["sc"]], dtype=torch.float32, device=dev)
        vs = torch.tensor([c["sc"]], dtype=torch.float32, device=dev)
    pkv.paged_attention_prefill(out, c["q"], c["kc"], c["vc"], torch.from_numpy(bt).to(dev),
                                torch.from_numpy(c["lens"]).to(dev),
                                torch.from_numpy(c["qs"]).to(dev), max_q_len=mq,
                                scale=c["D"] ** -0.5, k_scale=ks, v_scale=vs, flags=flags)
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(clear=True) == status
    return out


def run_oracle(c, bt=None):
    bt = c["bt"] if bt is None else bt
    want, _ = oracle.prefill(W.host(c["q"]), W.host(c["kc"]), W.host(c["vc"]), bt, c["lens"],
                             c["qs"], num_heads=c["Hq"], num_kv_heads=c["Hkv"], head_dim=c["D"],
                             block_size=c["bs"], scale=c["D"] ** -0.5, q_dtype=c["dt"],
                             cache_dtype=c["cache"], k_scale=c["sc"], v_scale=c["sc"])
    return want


def check(got, want, dt, rows=None):
    g = got.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        g, want = g[rows], want[rows]
    err = np.abs(g - want)
    assert np.all(np.isfinite(g))
    assert err.max() <= TOL[dt][0] and err.mean() <= TOL[dt][1], (err.max(), err.mean())


CASES = {
    "full prefills": ([1, 17, 64, 100, 300], [1, 17, 64, 100, 300]),
    "chunks over a cached context": ([500, 130, 64, 1000], [128, 3, 64, 37]),
    "single tokens": ([1, 50, 777], [1, 1, 1]),
}


KERNELS = [0, pkv.PKV_PREFILL_MMA_SYNC]  # tcgen05 (default), mma.sync


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (32, 8), (16, 1), (12, 2), (6, 2), (64, 4)])
@pytest.mark.parametrize("flags", KERNELS)
def test_prefill_parity_group_sizes(cuda_dev, case, Hq, Hkv, flags):
    lens, qlens = CASES[case]
    c = make_case(lens, qlens, Hq, Hkv, 128, 16, "bf16", cuda_dev, seed=Hq + Hkv)
    check(run_gpu(c, flags=flags), run_oracle(c), "bf16")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("flags", KERNELS)
def test_prefill_parity_dims_blocks_dtypes(cuda_dev, D, bs, dt, flags):
    c = make_case([400, 90, 33], [200, 90, 5], 16, 4, D, bs, dt, cuda_dev, seed=D + bs)
    check(run_gpu(c, flags=flags), run_oracle(c), dt)


def test_prefill_large_score_range_forces_rescaling(cuda_dev):
    # Keys aligned with the queries and growing along the sequence give scores
    # whose running maximum rises by more than 2^8 several times (the tcgen05
    # kernel then rescales O in tensor memory). Both kernels must meet the
    # tolerance and agree with each other to within the rounding of P.
    c = make_case([700, 300], [700, 40], 8, 2, 128, 16, "bf16", cuda_dev, seed=31)
    L = 700
    ramp = torch.linspace(0.2, 3.0, L).to(torch.bfloat16)
    q = c["q"].float()
    kc, bt = c["kc"].float(), c["bt"]
    for t in range(L):  # sequence 0: key t = the mean of its position's query group, scaled
        kc[bt[0, t // 16], t % 16] = q[t].view(2, 4, 128).mean(1) * ramp[t]
    c["kc"] = kc.to(torch.bfloat16)
    want = run_oracle(c)
    tc5 = run_gpu(c)
    mma = run_gpu(c, flags=pkv.PKV_PREFILL_MMA_SYNC)
    check(tc5, want, "bf16")
    check(mma, want, "bf16")
    # (outputs are rounded to bf16 once: allow a unit or two in the last place)
    a, b = tc5.float(), mma.float()
    assert torch.all((a - b).abs() <= 2 ** -7 * b.abs() + 2e-3)


@pytest.mark.parametrize("flags", KERNELS)
def test_prefill_long_chunk_many_tiles(cuda_dev, flags):
    c = make_case([3000, 2100], [1024, 2100], 32, 8, 128, 16, "bf16", cuda_dev, seed=9)
    got = run_gpu(c, flags=flags)
    # Sampled rows (the oracle is slow at this size): every 37th row and the last ones.
    T = int(c["qs"][-1])
    rows = np.unique(np.concatenate([np.arange(0, T, 37), np.arange(T - 5, T)]))
    items = np.stack(np.meshgrid(rows, np.arange(32), indexing="ij"), -1).reshape(-1, 2)
    want, _ = oracle.prefill(W.host(c["q"]), W.host(c["kc"]), W.host(c["vc"]), c["bt"],
                             c["lens"], c["qs"], num_heads=32, num_kv_heads=8, head_dim=128,
                             block_size=16, scale=128 ** -0.5, q_dtype="bf16",
                             cache_dtype="bf16", items=items)
    g = got.float().cpu().numpy()[items[:, 0], items[:, 1]].astype(np.float64)
    err = np.abs(g - want)
    assert err.max() <= TOL["bf16"][0] and err.mean() <= TOL["bf16"][1]


def test_single_token_rows_match_decode(cuda_dev):
    c = make_case([1, 50, 777, 64], [1, 1, 1, 1], 32, 8, 128, 16, "bf16", cuda_dev, seed=4)
    got = run_gpu(c)
    out = torch.empty_like(c["q"])
    S = 4
    ws = torch.empty(pkv.paged_attention_workspace_size(S, 32, 8, 128, 777, 0) + 1,
                     dtype=torch.uint8, device=cuda_dev)
    pkv.paged_attention_decode(out, c["q"], c["kc"], c["vc"], torch.from_numpy(c["bt"]).to(cuda_dev),
                               torch.from_numpy(c["lens"]).to(cuda_dev), max_seq_len=777,
                               scale=128 ** -0.5, workspace=ws)
    torch.cuda.synchronize()
    assert (got.float() - out.float()).abs().max().item() <= 2 * TOL["bf16"][0]


def test_chunk_longer_than_max_q_len_computes_its_last_rows(cuda_dev):
    c = make_case([200, 100], [150, 100], 8, 2, 64, 16, "bf16", cuda_dev, seed=12)
    got = run_gpu(c, max_q_len=64, fill=0.0)
    want = run_oracle(c)
    rows = np.r_[150 - 64:150, 250 - 64:250]
    check(got, want, "bf16", rows=rows)
    skipped = np.r_[0:150 - 64, 150:250 - 64]
    assert torch.all(got[torch.from_numpy(skipped).to(cuda_dev)] == 0)


@pytest.mark.parametrize("flags", KERNELS)
def test_chunk_longer_than_its_context_gives_zero_rows(cuda_dev, flags):
    # 10 query tokens over a 6-token context: the first 4 sit before position 0.
    c = make_case([6, 40], [10, 8], 8, 8, 64, 8, "bf16", cuda_dev, seed=2)
    got = run_gpu(c, flags=flags)
    want = run_oracle(c)
    assert np.all(want[:4] == 0)
    check(got, want, "bf16")


@pytest.mark.parametrize("flags", KERNELS)
def test_block_ids_outside_the_pool_read_as_zeros(cuda_dev, flags):
    c = make_case([70, 33], [20, 33], 16, 4, 128, 16, "bf16", cuda_dev, seed=6)
    bt = c["bt"].copy()
    nb = c["kc"].shape[0]
    bt[0, 1] = nb + 7
    bt[1, 0] = -3
    check(run_gpu(c, bt=bt, status=2, flags=flags), run_oracle(c, bt=bt), "bf16")  # reported


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (32, 8), (16, 1), (12, 2)])
@pytest.mark.parametrize("D", [64, 128])
def test_prefill_fp8_cache_parity(cuda_dev, case, Hq, Hkv, D):
    # E4M3 caches on the tcgen05 kernel: codes widened to f16 in shared memory,
    # k_scale folded into the scores, v_scale into the output.
    lens, qlens = CASES[case]
    c = make_case(lens, qlens, Hq, Hkv, D, 16, "bf16", cuda_dev, seed=Hq + D, cache="e4m3")
    check(run_gpu(c), run_oracle(c), "e4m3")


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("flags", KERNELS)
def test_prefill_fp8_cache_blocks_dtypes(cuda_dev, bs, dt, D, flags):
    # Both kernels over an E4M3 cache: tcgen05 (codes widened in shared memory)
    # and mma.sync (codes widened in registers).
    c = make_case([400, 90, 33], [200, 90, 5], 16, 4, D, bs, dt, cuda_dev, seed=D + bs + 1,
                  cache="e4m3")
    check(run_gpu(c, flags=flags), run_oracle(c), "e4m3")


def test_prefill_fp8_out_of_pool_and_prefix_hit_matches_decode(cuda_dev):
    # Out-of-pool ids read as zeros and are reported; a one-token chunk over an
    # FP8 cache equals the FP8 decode of the same token.
    c = make_case([70, 33, 500], [20, 33, 1], 16, 4, 128, 16, "bf16", cuda_dev, seed=8,
                  cache="e4m3")
    bt = c["bt"].copy()
    bt[0, 1] = c["kc"].shape[0] + 7
    check(run_gpu(c, bt=bt, status=2), run_oracle(c, bt=bt), "e4m3")
    got = run_gpu(c)
    last = int(c["qs"][-1]) - 1
    q1 = c["q"][last:last + 1]
    out = torch.empty_like(q1)
    sc = torch.tensor([c["sc"]], dtype=torch.float32, device=cuda_dev)
    pkv.paged_attention_decode(out, q1, c["kc"], c["vc"],
                               torch.from_numpy(c["bt"][2:3].copy()).to(cuda_dev),
                               torch.from_numpy(c["lens"][2:3].copy()).to(cuda_dev),
                               max_seq_len=500, scale=128 ** -0.5, k_scale=sc, v_scale=sc)
    torch.cuda.synchronize()
    assert (got[last:last + 1].float() - out.float()).abs().max().item() <= 2 * TOL["e4m3"][0]


def _device_args(c):
    dev = c["dev"]
    return (torch.from_numpy(c["bt"]).to(dev), torch.from_numpy(c["lens"]).to(dev),
            torch.from_numpy(c["qs"]).to(dev), int(np.diff(c["qs"]).max()))


def test_prefill_repeated_calls_and_graph_replays_reuse_work_counters(cuda_dev):
    # The tcgen05 kernel is persistent: its CTAs take items from a work counter
    # that each call takes from a ring of 64 and that the call's last CTA puts
    # back to zero. More calls than the ring holds, and replays of a captured
    # graph (which keeps its calls' counters), must all compute every item.
    c = make_case([300, 257, 64, 500, 33, 129], [300, 100, 64, 200, 33, 1], 32, 8, 128, 16,
                  "bf16", cuda_dev, seed=5)
    bt, lens, qs, mq = _device_args(c)
    want = run_oracle(c)
    outs = [torch.full(tuple(c["q"].shape), float("nan"), dtype=c["q"].dtype, device=cuda_dev)
            for _ in range(3)]

    def call(out):
        pkv.paged_attention_prefill(out, c["q"], c["kc"], c["vc"], bt, lens, qs, max_q_len=mq,
                                    scale=c["D"] ** -0.5)

    call(outs[0])
    torch.cuda.synchronize()
    first = outs[0].clone()
    check(first, want, "bf16")
    for _ in range(70):
        call(outs[0])
    torch.cuda.synchronize()
    assert torch.equal(outs[0], first)
    for o in outs:
        o.fill_(float("nan"))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        call(outs[0])  # warm-up outside the capture
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for o in outs:
                pkv.paged_attention_prefill(o, c["q"], c["kc"], c["vc"], bt, lens, qs,
                                            max_q_len=mq, scale=c["D"] ** -0.5, stream=s)
    for _ in range(5):
        for o in outs:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for o in outs:
            assert torch.equal(o, first)
    assert pkv.pkv_device_status(clear=True) == 0


def test_prefill_concurrent_calls_on_two_streams(cuda_dev):
    # Calls in flight at the same time on different streams use different work
    # counters and must not take each other's items.
    a = make_case([700, 300, 90], [700, 40, 90], 16, 2, 128, 16, "bf16", cuda_dev, seed=21)
    b = make_case([200, 1000, 64, 64], [200, 128, 1, 64], 64, 8, 64, 32, "f16", cuda_dev,
                  seed=22)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for c, s in zip((a, b), streams):
        bt, lens, qs, mq = _device_args(c)
        o = [torch.full(tuple(c["q"].shape), float("nan"), dtype=c["q"].dtype, device=cuda_dev)
             for _ in range(4)]
        outs.append((c, bt, lens, qs, mq, s, o))
    torch.cuda.synchronize()
    for k in range(4):  # interleaved launches, no synchronisation between the streams
        for c, bt, lens, qs, mq, s, o in outs:
            pkv.paged_attention_prefill(o[k], c["q"], c["kc"], c["vc"], bt, lens, qs,
                                        max_q_len=mq, scale=c["D"] ** -0.5, stream=s)
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(clear=True) == 0
    for c, bt, lens, qs, mq, s, o in outs:
        want = run_oracle(c)
        for k in range(4):
            check(o[k], want, c["dt"])


def test_prefill_many_one_chunk_items(cuda_dev):
    # 300 short sequences give a few thousand one-chunk items: each CTA of the
    # persistent kernel takes many more than its ring of item records holds.
    rng = np.random.default_rng(9)
    lens = [int(x) for x in rng.integers(1, 60, size=300)]
    qlens = [int(min(L, q)) for L, q in zip(lens, rng.integers(1, 4, size=300))]
    c = make_case(lens, qlens, 32, 8, 128, 16, "bf16", cuda_dev, seed=9)
    check(run_gpu(c), run_oracle(c), "bf16")


BENCH_SHAPES = {  # the prefill workloads bench.py times: 64 query / 8 KV heads, D 128, block 16
    "1024-token chunks after 2048 cached": ([3072] * 8, [1024] * 8),
    "4096-token prompts": ([4096] * 4, [4096] * 4),
    "512-token prompts": ([512] * 16, [512] * 16),
}


@pytest.mark.parametrize("shape", list(BENCH_SHAPES))
@pytest.mark.parametrize("cache", ["bf16", "e4m3"])
def test_prefill_bench_workloads_at_full_size_sampled(cuda_dev, shape, cache):
    # The workloads the benchmark times, at their full sizes, on the default
    # kernel as it launches there; the fp64 oracle computes 1,536 sampled
    # (row, query head) outputs: the first and last rows of every chunk and of
    # every 256-row item boundary in the first sequence, and random ones.
    lens, qlens = BENCH_SHAPES[shape]
    c = make_case(lens, qlens, 64, 8, 128, 16, "bf16", cuda_dev, seed=len(lens),
                  cache=None if cache == "bf16" else cache)
    got = run_gpu(c)
    T = int(c["qs"][-1])
    rng = np.random.default_rng(5)
    rows = set(int(x) for x in c["qs"][:-1]) | set(int(x) - 1 for x in c["qs"][1:])
    rows |= set(range(0, min(T, qlens[0]), 32)) | set(range(31, min(T, qlens[0]), 32))
    rows = sorted(rows)
    items = [(r, int(h)) for r in rows for h in rng.choice(64, 2, replace=False)]
    items += [(int(r), int(h)) for r, h in zip(rng.integers(0, T, 1536 - len(items)),
                                                rng.integers(0, 64, 1536 - len(items)))]
    items = np.asarray(items[:1536], np.int32)
    want, _ = oracle.prefill(W.host(c["q"]), W.host(c["kc"]), W.host(c["vc"]), c["bt"],
                             c["lens"], c["qs"], num_heads=64, num_kv_heads=8, head_dim=128,
                             block_size=16, scale=128 ** -0.5, q_dtype="bf16",
                             cache_dtype=c["cache"], k_scale=c["sc"], v_scale=c["sc"],
                             items=items)
    g = got[items[:, 0], items[:, 1]].float().cpu().numpy().astype(np.float64)
    err = np.abs(g - want)
    tol = TOL["e4m3" if cache == "e4m3" else "bf16"]
    assert np.all(np.isfinite(g))
    assert err.max() <= tol[0] and err.mean() <= tol[1], (err.max(), err.mean())


@pytest.mark.parametrize("D", [64, 128])
def test_prefill_output_only_16_byte_aligned(cuda_dev, D):
    # The epilogue stores 32 bytes at a time when the output is 32-byte aligned
    # and 16 at a time otherwise: an output 16 bytes past an aligned allocation
    # takes the second path.
    c = make_case([400, 90, 33], [200, 90, 5], 16, 4, D, 16, "bf16", cuda_dev, seed=D + 3)
    n = int(c["q"].numel())
    buf = torch.full((n + 8,), float("nan"), dtype=c["q"].dtype, device=cuda_dev)
    out = buf[8:].view(c["q"].shape)
    assert out.data_ptr() % 32 == 16
    pkv.paged_attention_prefill(out, c["q"], c["kc"], c["vc"], torch.from_numpy(c["bt"]).to(cuda_dev),
                                torch.from_numpy(c["lens"]).to(cuda_dev),
                                torch.from_numpy(c["qs"]).to(cuda_dev),
                                max_q_len=int(np.diff(c["qs"]).max()), scale=D ** -0.5)
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(clear=True) == 0
    assert torch.isnan(buf[:8].float()).all()  # nothing written before the output
    check(out, run_oracle(c), "bf16")
