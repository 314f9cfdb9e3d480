"""Pins for the oracle's multi-token (causal) attention over the paged cache:
brute force with a full masked score matrix on contiguous K/V, closed forms,
causality and agreement with the pinned decode at one query token."""
import numpy as np
import pytest

from test_oracle_pins import f32, oracle_f32, scatter_into_pool


def _layout(rng, lens, bs, spare=3):
    nbs = [-(-L // bs) for L in lens]
    nb = sum(nbs) + spare
    ids = rng.permutation(nb)
    bt = np.full((len(lens), max(nbs)), -1, np.int32)
    n = 0
    for i, k in enumerate(nbs):
        bt[i, :k] = ids[n:n + k]
        n += k
    return bt, nb


def brute_causal(Q, K, V, positions, scale):
    """Full-matrix causal attention: S = scale Q K^T masked to t <= pos, row softmax, P V."""
    S = scale * (Q @ K.T)
    mask = np.arange(K.shape[0])[None, :] <= np.asarray(positions)[:, None]
    S = np.where(mask, S, -np.inf)
    P = np.exp(S - S.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    return P @ V


def run_prefill(orc, q, kc, vc, bt, lens, qs, Hq, Hkv, D, bs, scale):
    out, _ = orc.prefill(f32(q), f32(kc), f32(vc), bt, np.asarray(lens, np.int32),
                         np.asarray(qs, np.int32), num_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                         block_size=bs, scale=scale, q_dtype="f32", cache_dtype="f32")
    return out


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (4, 1)])
def test_prefill_matches_masked_matrix_brute_force(orc, Hq, Hkv):
    rng = np.random.default_rng(5)
    D, bs, scale = 32, 8, 0.25          # exact in binary32, as the oracle takes it
    lens = [37, 20, 64, 1, 9]            # cached tokens, the query chunk included
    qlens = [37, 5, 16, 1, 1]            # full prefill, chunks, single tokens
    qs = np.concatenate([[0], np.cumsum(qlens)])
    bt, nb = _layout(rng, lens, bs)
    per_k = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lens]
    per_v = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lens]
    kc = scatter_into_pool(per_k, bt, bs, (nb, bs, Hkv, D))
    vc = scatter_into_pool(per_v, bt, bs, (nb, bs, Hkv, D))
    q = rng.standard_normal((qs[-1], Hq, D)).astype(np.float32)
    out = run_prefill(orc, q, kc, vc, bt, lens, qs, Hq, Hkv, D, bs, scale)
    g = Hq // Hkv
    for i, (L, n) in enumerate(zip(lens, qlens)):
        pos = np.arange(L - n, L)
        for j in range(Hq):
            want = brute_causal(q[qs[i]:qs[i + 1], j].astype(np.float64),
                                per_k[i][:, j // g].astype(np.float64),
                                per_v[i][:, j // g].astype(np.float64), pos, scale)
            assert np.max(np.abs(out[qs[i]:qs[i + 1], j] - want)) <= 1e-12


def test_constant_keys_give_prefix_means(orc):
    rng = np.random.default_rng(2)
    D, bs, L = 16, 8, 29
    bt, nb = _layout(rng, [L], bs)
    k = np.tile(rng.standard_normal((1, 1, D)), (L, 1, 1))
    v = rng.standard_normal((L, 1, D))
    kc = scatter_into_pool([k], bt, bs, (nb, bs, 1, D))
    vc = scatter_into_pool([v], bt, bs, (nb, bs, 1, D))
    q = rng.standard_normal((L, 1, D))
    out = run_prefill(orc, q, kc, vc, bt, [L], [0, L], 1, 1, D, bs, 0.3)
    vf = v.astype(np.float32).astype(np.float64)[:, 0]
    want = np.cumsum(vf, 0) / np.arange(1, L + 1)[:, None]
    assert np.max(np.abs(out[:, 0] - want)) <= 1e-12
    assert np.array_equal(out[0, 0], vf[0])          # position 0 sees only itself


def test_rows_ignore_later_tokens(orc):
    rng = np.random.default_rng(3)
    D, bs, L, n = 16, 8, 40, 12
    bt, nb = _layout(rng, [L], bs)
    k = rng.standard_normal((L, 2, D))
    v = rng.standard_normal((L, 2, D))
    q = rng.standard_normal((n, 4, D))
    out1 = run_prefill(orc, q, scatter_into_pool([k], bt, bs, (nb, bs, 2, D)),
                       scatter_into_pool([v], bt, bs, (nb, bs, 2, D)), bt, [L], [0, n], 4, 2,
                       D, bs, 0.25)
    k2, v2 = k.copy(), v.copy()
    k2[L - 5:] += 3.0                                  # change the last 5 tokens only
    v2[L - 5:] -= 1.0
    out2 = run_prefill(orc, q, scatter_into_pool([k2], bt, bs, (nb, bs, 2, D)),
                       scatter_into_pool([v2], bt, bs, (nb, bs, 2, D)), bt, [L], [0, n], 4, 2,
                       D, bs, 0.25)
    first_changed = n - 5                              # rows at positions >= L - 5
    assert np.array_equal(out1[:first_changed], out2[:first_changed])
    assert not np.allclose(out1[first_changed:], out2[first_changed:])


def test_single_token_chunks_equal_decode(orc):
    rng = np.random.default_rng(4)
    D, bs, Hq, Hkv = 32, 16, 8, 2
    lens = [1, 30, 100]
    bt, nb = _layout(rng, lens, bs)
    kc = rng.standard_normal((nb, bs, Hkv, D))
    vc = rng.standard_normal((nb, bs, Hkv, D))
    q = rng.standard_normal((3, Hq, D))
    out = run_prefill(orc, q, kc, vc, bt, lens, [0, 1, 2, 3], Hq, Hkv, D, bs, 0.1)
    dec = oracle_f32(orc, q, kc, vc, bt, lens, Hq, Hkv, D, bs, 0.1)
    assert np.array_equal(out, dec)


def test_prefill_over_e4m3_codes_matches_brute_force_with_scales(orc):
    # E4M3 pool: K[t] = code value * k_scale, V[t] = code value * v_scale. The
    # brute force decodes the codes with torch's float8_e4m3fn (not the oracle's
    # decoder) and takes the bf16 query values from torch as well.
    import torch
    rng = np.random.default_rng(11)
    D, bs, Hq, Hkv = 32, 8, 4, 2
    lens, qlens = [23, 40], [23, 6]
    qs = np.concatenate([[0], np.cumsum(qlens)])
    bt, nb = _layout(rng, lens, bs)
    codes_k = rng.integers(0, 256, size=(nb, bs, Hkv, D), dtype=np.uint8)
    codes_v = rng.integers(0, 256, size=(nb, bs, Hkv, D), dtype=np.uint8)
    for c in (codes_k, codes_v):      # no NaN codes (S.1111.111)
        c[(c & 0x7F) == 0x7F] = 0x3A
    qb = torch.randn((int(qs[-1]), Hq, D), generator=torch.Generator().manual_seed(3)).to(
        torch.bfloat16)
    ks, vs = 0.0625, 0.375             # exact in binary32
    out, _ = orc.prefill(qb.view(torch.int16).numpy().view(np.uint16), codes_k, codes_v, bt,
                         np.asarray(lens, np.int32), qs.astype(np.int32), num_heads=Hq,
                         num_kv_heads=Hkv, head_dim=D, block_size=bs, scale=0.25,
                         q_dtype="bf16", cache_dtype="e4m3", k_scale=ks, v_scale=vs)
    dec = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    kv, vv = dec(codes_k) * ks, dec(codes_v) * vs
    qv = qb.to(torch.float64).numpy()
    g = Hq // Hkv
    for i, (L, n) in enumerate(zip(lens, qlens)):
        rows_k = np.stack([kv[bt[i, t // bs], t % bs] for t in range(L)])
        rows_v = np.stack([vv[bt[i, t // bs], t % bs] for t in range(L)])
        pos = np.arange(L - n, L)
        for j in range(Hq):
            want = brute_causal(qv[qs[i]:qs[i + 1], j], rows_k[:, j // g], rows_v[:, j // g],
                                pos, 0.25)
            assert np.max(np.abs(out[qs[i]:qs[i + 1], j] - want)) <= 1e-12
