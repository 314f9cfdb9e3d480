"""Pins for the CPU oracle: values the pages fix, closed forms, invariants and
brute force on tiny inputs. None of these re-types the oracle's own code; each
is chosen so that a plausible slip in it (a wrong index, a dropped scale, a
transposed operand, a mis-rounded FP8 code) fails at least one test.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from paged_kv_cache_367_b200 import workloads as W


# ---------------------------------------------------------------- helpers ----

def brute_attention(q, K, V, scale):
    """Unpaged softmax attention of one query over contiguous K/V (numpy fp64)."""
    s = scale * (K @ q)
    w = np.exp(s - s.max())
    return (w[:, None] * V).sum(0) / w.sum()


def scatter_into_pool(per_seq, block_table, block_size, pool_shape, fill=np.nan):
    """Test-side paging: place token t of sequence i at pool[bt[i][t//bs], t%bs]."""
    pool = np.full(pool_shape, fill, dtype=np.float64)
    for i, X in enumerate(per_seq):
        for t in range(X.shape[0]):
            pool[block_table[i][t // block_size], t % block_size] = X[t]
    return pool


def f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def oracle_f32(orc, q, kc, vc, bt, lens, Hq, Hkv, D, bs, scale, **kw):
    out, _ = orc.decode(f32(q), f32(kc), f32(vc), np.asarray(bt, np.int32),
                        np.asarray(lens, np.int32), num_heads=Hq, num_kv_heads=Hkv,
                        head_dim=D, block_size=bs, scale=scale, q_dtype="f32",
                        cache_dtype="f32", **kw)
    return out


# ------------------------------------------------------- element formats ----

def test_e4m3_decode_all_codes_match_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ours = orc.values(codes, "e4m3")
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert set(np.flatnonzero(nan).tolist()) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_e4m3_encode_all_bf16_values_match_torch(orc):
    bits = np.arange(65536, dtype=np.uint32) << 16
    x = bits.view(np.float32)
    ours = orc.e4m3_encode(x)
    finite = np.isfinite(x) & (np.abs(x) < 464.0)   # torch turns |x| >= 464 into NaN
    ref = torch.from_numpy(x[finite]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours[finite], ref)
    big = np.isfinite(x) & (np.abs(x) >= 448.0)
    assert np.all((ours[big] & 0x7F) == 0x7E)          # saturation to +-448
    assert np.all((ours[np.isinf(x)] & 0x7F) == 0x7E)
    assert np.all((ours[np.isnan(x)] & 0x7F) == 0x7F)


def test_e4m3_encode_rounding_boundaries_match_torch(orc):
    vals = orc.values(np.arange(256, dtype=np.uint8), "e4m3")
    pos = np.unique(vals[np.isfinite(vals) & (vals >= 0)])
    mids = (pos[:-1] + pos[1:]) / 2                      # exact ties
    cand = np.concatenate([pos, mids]).astype(np.float32)
    ulp_up = np.nextafter(cand, np.float32(np.inf))
    ulp_dn = np.nextafter(cand, np.float32(-np.inf))
    x = np.concatenate([cand, ulp_up, ulp_dn])
    x = np.concatenate([x, -x])
    rng = np.random.default_rng(7)
    x = np.concatenate([x, rng.standard_normal(200000).astype(np.float32) * 100,
                        rng.standard_normal(200000).astype(np.float32) * 0.01])
    x = x[np.abs(x) < 464.0]
    ours = orc.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_16bit_decoders_exact(orc):
    allbits = np.arange(65536, dtype=np.uint16)
    bf = orc.values(allbits, "bf16")
    ref_bf = torch.from_numpy(allbits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    ok = ~np.isnan(ref_bf)
    assert np.array_equal(np.isnan(bf), ~ok) and np.array_equal(bf[ok], ref_bf[ok])
    h = orc.values(allbits.view(np.float16), "f16")
    ref_h = allbits.view(np.float16).astype(np.float64)
    ok = ~np.isnan(ref_h)
    assert np.array_equal(np.isnan(h), ~ok) and np.array_equal(h[ok], ref_h[ok])


# ---------------------------------------------------- block-table arithmetic ----

def test_blocks_per_sequence_from_the_page(orc):
    g = read_golden("blocks_per_seq.txt")
    for n_tok, n_blk in zip(g["tokens"], g["blocks"]):
        assert orc.num_blocks_for(n_tok, g["block_size"]) == n_blk


def test_block_table_figure_slots(orc):
    g = read_golden("block_table_figure.txt")
    bt = np.array(g["block_table"], np.int32)
    got = [orc.slot_of_token(bt, t, g["block_size"]) for t in range(len(g["slots"]))]
    assert got == g["slots"]


@pytest.mark.parametrize("L", [7, 8])
def test_block_table_figure_decode_reads_exactly_those_slots(orc, L):
    """Uniform scores (K = 0) make the output the mean of the gathered V rows; a
    one-hot V row per slot reveals which slots were read. Every other slot is NaN."""
    g = read_golden("block_table_figure.txt")
    bs, nb, D = g["block_size"], 8, 64
    kc = np.full((nb, bs, 1, D), np.nan)
    vc = np.full((nb, bs, 1, D), np.nan)
    expected = g["slots"][:L]
    for s in expected:
        kc[s // bs, s % bs, 0] = 0.0
        vc[s // bs, s % bs, 0] = 0.0
        vc[s // bs, s % bs, 0, s] = 1.0
    q = np.ones((1, 1, D))
    bt = np.array([g["block_table"]], np.int32)
    out = oracle_f32(orc, q, kc, vc, bt, [L], 1, 1, D, bs, 0.125)
    want = np.zeros(D)
    want[expected] = 1.0 / L
    assert np.array_equal(out[0, 0], want)


def test_kv_head_index_and_gqa_grouping(orc):
    """Pool [blocks, bs, Hkv, D]: KV head h holds value h+1; query heads j use
    KV head j // (Hq/Hkv) (consecutive grouping)."""
    Hq, Hkv, D, bs = 6, 3, 8, 4
    kc = np.zeros((2, bs, Hkv, D))
    vc = np.zeros((2, bs, Hkv, D))
    for h in range(Hkv):
        vc[:, :, h, :] = h + 1.0
    q = np.random.default_rng(0).standard_normal((1, Hq, D))
    out = oracle_f32(orc, q, kc, vc, [[1, 0]], [6], Hq, Hkv, D, bs, 1.0)
    for j in range(Hq):
        assert np.all(out[0, j] == j // 2 + 1.0)


# ------------------------------------------------------------- brute force ----

@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 2), (4, 1)])
def test_oracle_matches_unpaged_brute_force(orc, Hq, Hkv):
    rng = np.random.default_rng(11)
    S, D, bs, nb = 4, 64, 16, 64
    lens = [1, 17, 64, 100]
    scale = 1 / 8
    per_k = [rng.standard_normal((L, Hkv, D)) for L in lens]
    per_v = [rng.standard_normal((L, Hkv, D)) for L in lens]
    ids = rng.permutation(nb)
    bt = np.full((S, 7), -1, np.int32)
    n = 0
    for i, L in enumerate(lens):
        k = -(-L // bs)
        bt[i, :k] = ids[n:n + k]
        n += k
    kc = scatter_into_pool(per_k, bt, bs, (nb, bs, Hkv, D))
    vc = scatter_into_pool(per_v, bt, bs, (nb, bs, Hkv, D))
    q = rng.standard_normal((S, Hq, D))
    out = oracle_f32(orc, q.astype(np.float32), kc, vc, bt, lens, Hq, Hkv, D, bs, scale)
    g = Hq // Hkv
    for i in range(S):
        for j in range(Hq):
            K = per_k[i][:, j // g].astype(np.float32).astype(np.float64)
            V = per_v[i][:, j // g].astype(np.float32).astype(np.float64)
            want = brute_attention(q[i, j].astype(np.float32).astype(np.float64), K, V, scale)
            assert np.max(np.abs(out[i, j] - want)) <= 1e-12


def test_tiny_workload_matches_brute_force(orc):
    """The tiny configuration exactly (fp32, 4 seqs, 8 heads, D 64, bs 16, 64 blocks)."""
    wl = W.make_workload(W.CONFIGS["tiny"], device="cpu", poison=True)
    c = wl.cfg
    kc, vc = W.host(wl.k_cache).copy(), W.host(wl.v_cache).copy()
    # Fill the newest slot as the append would, so the pool is complete.
    nk, nv = W.host(wl.new_key), W.host(wl.new_value)
    for i, s in enumerate(wl.slot_mapping):
        kc[s // c.block_size, s % c.block_size] = nk[i]
        vc[s // c.block_size, s % c.block_size] = nv[i]
    q = W.host(wl.query)
    out = oracle_f32(orc, q, kc, vc, wl.block_table, wl.seq_lens, c.num_heads,
                     c.num_kv_heads, c.head_dim, c.block_size, c.scale)
    assert np.all(np.isfinite(out))
    for i, L in enumerate(wl.seq_lens):
        toks = [(wl.block_table[i][t // c.block_size], t % c.block_size) for t in range(L)]
        for j in range(c.num_heads):
            K = np.array([kc[b, o, j] for b, o in toks], np.float64)
            V = np.array([vc[b, o, j] for b, o in toks], np.float64)
            want = brute_attention(q[i, j].astype(np.float64), K, V, c.scale)
            assert np.max(np.abs(out[i, j] - want)) <= 1e-12


# ------------------------------------------------------------ special cases ----

def _one_seq(rng, L, D=32, bs=8, nb=None):
    nb = nb or (-(-L // bs) + 3)
    ids = rng.permutation(nb)[: -(-L // bs)]
    return np.array([ids], np.int32), nb


def test_single_token_returns_v_row(orc):
    rng = np.random.default_rng(1)
    D, bs = 32, 8
    bt, nb = _one_seq(rng, 1, D, bs)
    kc = rng.standard_normal((nb, bs, 1, D))
    vc = rng.standard_normal((nb, bs, 1, D))
    q = rng.standard_normal((1, 1, D))
    out = oracle_f32(orc, q, kc, vc, bt, [1], 1, 1, D, bs, 0.3)
    assert np.array_equal(out[0, 0], f32(vc[bt[0, 0], 0, 0]).astype(np.float64))


@pytest.mark.parametrize("case", ["const_k", "zero_q"])
def test_uniform_scores_give_mean_of_v(orc, case):
    rng = np.random.default_rng(2)
    L, D, bs = 37, 32, 8
    bt, nb = _one_seq(rng, L, D, bs)
    kc = rng.standard_normal((nb, bs, 1, D))
    q = rng.standard_normal((1, 1, D))
    if case == "const_k":
        kc[:] = rng.standard_normal(D)
    else:
        q[:] = 0.0
    vc = rng.standard_normal((nb, bs, 1, D))
    out = oracle_f32(orc, q, kc, vc, bt, [L], 1, 1, D, bs, 0.2)
    rows = np.array([f32(vc[bt[0, t // bs], t % bs, 0]) for t in range(L)], np.float64)
    assert np.max(np.abs(out[0, 0] - rows.mean(0))) <= 1e-12


def test_constant_v_gives_that_constant(orc):
    rng = np.random.default_rng(3)
    L, D, bs = 50, 32, 16
    bt, nb = _one_seq(rng, L, D, bs)
    kc = rng.standard_normal((nb, bs, 1, D)) * 3
    c = f32(rng.standard_normal(D)).astype(np.float64)
    vc = np.broadcast_to(c, (nb, bs, 1, D)).copy()
    out = oracle_f32(orc, rng.standard_normal((1, 1, D)), kc, vc, bt, [L], 1, 1, D, bs, 0.5)
    assert np.max(np.abs(out[0, 0] - c)) <= 1e-12


def test_dominant_key_selects_its_value(orc):
    rng = np.random.default_rng(4)
    L, D, bs, tstar = 40, 32, 8, 23
    bt, nb = _one_seq(rng, L, D, bs)
    kc = rng.standard_normal((nb, bs, 1, D)) * 0.01
    q = np.zeros((1, 1, D))
    q[0, 0, 3] = 1.0
    kc[bt[0, tstar // bs], tstar % bs, 0] = 1000.0 * q[0, 0]
    vc = rng.standard_normal((nb, bs, 1, D))
    out = oracle_f32(orc, q, kc, vc, bt, [L], 1, 1, D, bs, 1.0)
    want = f32(vc[bt[0, tstar // bs], tstar % bs, 0]).astype(np.float64)
    assert np.max(np.abs(out[0, 0] - want)) <= 1e-12


def test_zero_length_gives_zeros(orc):
    kc = np.full((2, 8, 1, 16), np.nan)
    out = oracle_f32(orc, np.ones((1, 1, 16)), kc, kc, [[-1]], [0], 1, 1, 16, 8, 1.0)
    assert np.array_equal(out[0, 0], np.zeros(16))


# --------------------------------------------------------------- invariants ----

def _random_problem(rng, S=3, Hq=4, Hkv=2, D=32, bs=8, lens=(9, 40, 64)):
    nbs = [-(-L // bs) for L in lens]
    nb = sum(nbs) + 5
    ids = rng.permutation(nb)
    bt = np.full((S, max(nbs)), -1, np.int32)
    n = 0
    for i, k in enumerate(nbs):
        bt[i, :k] = ids[n:n + k]
        n += k
    kc = rng.standard_normal((nb, bs, Hkv, D))
    vc = rng.standard_normal((nb, bs, Hkv, D))
    q = rng.standard_normal((S, Hq, D))
    return q, kc, vc, bt, list(lens), (Hq, Hkv, D, bs)


def test_physical_block_permutation_is_bit_identical(orc):
    rng = np.random.default_rng(5)
    q, kc, vc, bt, lens, (Hq, Hkv, D, bs) = _random_problem(rng)
    out1 = oracle_f32(orc, q, kc, vc, bt, lens, Hq, Hkv, D, bs, 0.25)
    perm = rng.permutation(kc.shape[0])          # new id of old block b is perm[b]
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    out2 = oracle_f32(orc, q, kc2, vc2, bt2, lens, Hq, Hkv, D, bs, 0.25)
    assert np.array_equal(out1, out2)


def test_shared_prefix_equals_duplicated_blocks(orc):
    rng = np.random.default_rng(6)
    S, Hq, Hkv, D, bs, P = 3, 4, 2, 32, 8, 16    # 2 shared prefix blocks
    lens = [16 + 3, 16 + 5, 16 + 8]
    nb = 2 + 2 * S
    kc = rng.standard_normal((nb, bs, Hkv, D))
    vc = rng.standard_normal((nb, bs, Hkv, D))
    shared = [0, 1]
    bt_shared = np.array([shared + [2 + i, -1] for i in range(S)], np.int32)
    # duplicated: copy the prefix blocks into private blocks 2+S+2i, 2+S+2i+1
    kc_d = np.concatenate([kc, np.zeros((2 * S, bs, Hkv, D))])
    vc_d = np.concatenate([vc, np.zeros((2 * S, bs, Hkv, D))])
    bt_dup = np.zeros((S, 4), np.int32) - 1
    for i in range(S):
        a, b = nb + 2 * i, nb + 2 * i + 1
        kc_d[a], kc_d[b], vc_d[a], vc_d[b] = kc[0], kc[1], vc[0], vc[1]
        bt_dup[i, :3] = [a, b, 2 + i]
    q = rng.standard_normal((S, Hq, D))
    o1 = oracle_f32(orc, q, kc, vc, bt_shared, lens, Hq, Hkv, D, bs, 0.3)
    o2 = oracle_f32(orc, q, kc_d, vc_d, bt_dup, lens, Hq, Hkv, D, bs, 0.3)
    assert np.array_equal(o1, o2)


def test_linearity_in_v(orc):
    rng = np.random.default_rng(8)
    q, kc, vc, bt, lens, (Hq, Hkv, D, bs) = _random_problem(rng)
    v2 = rng.standard_normal(vc.shape)
    a = oracle_f32(orc, q, kc, f32(vc), bt, lens, Hq, Hkv, D, bs, 0.25)
    b = oracle_f32(orc, q, kc, f32(v2), bt, lens, Hq, Hkv, D, bs, 0.25)
    c = oracle_f32(orc, q, kc, f32(vc).astype(np.float64) + f32(v2), bt, lens, Hq, Hkv, D, bs, 0.25)
    # f32(v1)+f32(v2) is rounded to f32 on the way in; allow that rounding.
    assert np.max(np.abs(c - (a + b))) <= 1e-6


def test_partition_merge_identity():
    """LSE merge of per-partition results equals the unsplit softmax (fp64):
    lse_p = m_p + ln l_p, out = sum_p exp(lse_p - M) o_p / sum_p exp(lse_p - M)."""
    rng = np.random.default_rng(9)
    L, D = 1300, 16
    K, V, q = rng.standard_normal((L, D)), rng.standard_normal((L, D)), rng.standard_normal(D)
    full = brute_attention(q, K, V, 0.3)
    for P in (1, 7, 512, 2000):
        os_, ls = [], []
        for p0 in range(0, L, P):
            s = 0.3 * (K[p0:p0 + P] @ q)
            m = s.max()
            w = np.exp(s - m)
            os_.append((w[:, None] * V[p0:p0 + P]).sum(0) / w.sum())
            ls.append(m + math.log(w.sum()))
        ls = np.array(ls)
        M = ls.max()
        wp = np.exp(ls - M)
        merged = (wp[:, None] * np.array(os_)).sum(0) / wp.sum()
        assert np.max(np.abs(merged - full)) <= 1e-12


# ---------------------------------------------------------------------- FP8 ----

def test_fp8_decode_uses_scaled_codes(orc):
    rng = np.random.default_rng(10)
    L, D, bs, Hkv, Hq = 45, 32, 16, 2, 4
    nb = 5
    bt = np.array([[3, 0, 4]], np.int32)
    kcodes = rng.integers(0, 256, (nb, bs, Hkv, D), dtype=np.uint8)
    vcodes = rng.integers(0, 256, (nb, bs, Hkv, D), dtype=np.uint8)
    kcodes[(kcodes & 0x7F) == 0x7F] = 0x10    # keep the used slots finite
    vcodes[(vcodes & 0x7F) == 0x7F] = 0x22
    ks, vs = 0.0123, 0.0456
    q = f32(rng.standard_normal((1, Hq, D)))
    out, _ = orc.decode(q, kcodes, vcodes, bt, np.array([L], np.int32), num_heads=Hq,
                        num_kv_heads=Hkv, head_dim=D, block_size=bs, scale=0.2,
                        q_dtype="f32", cache_dtype="e4m3", k_scale=ks, v_scale=vs)
    kt = torch.from_numpy(kcodes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    vt = torch.from_numpy(vcodes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for j in range(Hq):
        h = j // 2
        K = np.array([kt[bt[0, t // bs], t % bs, h] for t in range(L)]) * np.float64(np.float32(ks))
        V = np.array([vt[bt[0, t // bs], t % bs, h] for t in range(L)]) * np.float64(np.float32(vs))
        want = brute_attention(q[0, j].astype(np.float64), K, V, np.float64(np.float32(0.2)))
        assert np.max(np.abs(out[0, j] - want)) <= 1e-12


# ------------------------------------------------------------------- append ----

def test_append_writes_only_the_figure_slot(orc):
    """Append the 8th token of the figure's request (block size 4, table [7, 2]):
    it lands at physical block 2, offset 3, and nothing else changes."""
    g = read_golden("block_table_figure.txt")
    bs, nb, Hkv, D = g["block_size"], 8, 2, 16
    rng = np.random.default_rng(12)
    kc = f32(rng.standard_normal((nb, bs, Hkv, D)))
    vc = f32(rng.standard_normal((nb, bs, Hkv, D)))
    k0, v0 = kc.copy(), vc.copy()
    key = f32(rng.standard_normal((1, Hkv, D)))
    val = f32(rng.standard_normal((1, Hkv, D)))
    slot = g["slots"][7]
    orc.append(key, val, kc, vc, np.array([slot]), num_kv_heads=Hkv, head_dim=D,
               block_size=bs, num_blocks=nb, src_dtype="f32", cache_dtype="f32")
    assert np.array_equal(kc[2, 3], key[0]) and np.array_equal(vc[2, 3], val[0])
    mask = np.ones((nb, bs), bool)
    mask[2, 3] = False
    assert np.array_equal(kc[mask], k0[mask]) and np.array_equal(vc[mask], v0[mask])


def test_append_skips_negative_and_out_of_range_slots(orc):
    rng = np.random.default_rng(13)
    nb, bs, Hkv, D = 4, 8, 1, 8
    kc = f32(rng.standard_normal((nb, bs, Hkv, D)))
    k0 = kc.copy()
    vc = kc.copy()
    key = f32(rng.standard_normal((3, Hkv, D)))
    orc.append(key, key, kc, vc, np.array([-1, nb * bs, -7]), num_kv_heads=Hkv, head_dim=D,
               block_size=bs, num_blocks=nb, src_dtype="f32", cache_dtype="f32")
    assert np.array_equal(kc, k0) and np.array_equal(vc, k0)


def test_append_bf16_copy_is_byte_exact(orc):
    rng = np.random.default_rng(14)
    nb, bs, Hkv, D, T = 6, 16, 2, 64, 5
    kc = rng.integers(0, 65536, (nb, bs, Hkv, D), dtype=np.uint16)
    vc = kc.copy()
    key = rng.integers(0, 65536, (T, Hkv, D), dtype=np.uint16)
    val = rng.integers(0, 65536, (T, Hkv, D), dtype=np.uint16)
    slots = rng.choice(nb * bs, T, replace=False)
    orc.append(key, val, kc, vc, slots, num_kv_heads=Hkv, head_dim=D, block_size=bs,
               num_blocks=nb, src_dtype="bf16", cache_dtype="bf16")
    flat_k, flat_v = kc.reshape(nb * bs, Hkv, D), vc.reshape(nb * bs, Hkv, D)
    for t, s in enumerate(slots):
        assert np.array_equal(flat_k[s], key[t]) and np.array_equal(flat_v[s], val[t])


def test_append_fp8_matches_torch_quantisation(orc):
    rng = np.random.default_rng(15)
    nb, bs, Hkv, D, T = 4, 16, 2, 64, 6
    key_f = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).to(torch.bfloat16)
    val_f = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32) * 3).to(torch.bfloat16)
    ks = float(key_f.float().abs().amax()) / 448.0
    vs = float(val_f.float().abs().amax()) / 448.0
    kc = np.zeros((nb, bs, Hkv, D), np.uint8)
    vc = np.zeros((nb, bs, Hkv, D), np.uint8)
    slots = rng.choice(nb * bs, T, replace=False)
    orc.append(W.host(key_f), W.host(val_f), kc, vc, slots, num_kv_heads=Hkv, head_dim=D,
               block_size=bs, num_blocks=nb, src_dtype="bf16", cache_dtype="e4m3",
               k_scale=ks, v_scale=vs)
    ks32 = torch.tensor(ks, dtype=torch.float32)
    vs32 = torch.tensor(vs, dtype=torch.float32)
    kq = (key_f.float() / ks32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    vq = (val_f.float() / vs32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    fk, fv = kc.reshape(nb * bs, Hkv, D), vc.reshape(nb * bs, Hkv, D)
    for t, s in enumerate(slots):
        assert np.array_equal(fk[s], kq[t]) and np.array_equal(fv[s], vq[t])


def test_block_id_outside_pool_reads_as_zero_row(orc):
    """Reading adopted for corrupt tables: an id outside [0, num_blocks) is a zero row."""
    rng = np.random.default_rng(16)
    nb, bs, D = 3, 8, 16
    kc = rng.standard_normal((nb, bs, 1, D))
    vc = rng.standard_normal((nb, bs, 1, D))
    q = rng.standard_normal((1, 1, D))
    out = oracle_f32(orc, q, kc, vc, [[1, 99]], [12], 1, 1, D, bs, 0.5)
    K = np.concatenate([f32(kc[1, :, 0]), np.zeros((4, D))]).astype(np.float64)
    V = np.concatenate([f32(vc[1, :, 0]), np.zeros((4, D))]).astype(np.float64)
    want = brute_attention(f32(q[0, 0]).astype(np.float64), K, V, 0.5)
    assert np.max(np.abs(out[0, 0] - want)) <= 1e-12
