"""Random operation traces for the block manager, checked against the plain
logical model in oracle/block_model.py.

A trace admits prompts (drawn from a few shared system prompts plus random
suffixes, so prefix-cache hits happen), appends tokens, forks, frees, and swaps
groups of sequences out and back in. The K/V row of a token is a pure function
of the sequence's token ids up to and including it (as a model's K/V would be),
so two sequences may share a block exactly when their tokens agree up to the
end of it. The pool operations are pluggable: `NumpyPools` applies writes and
copies on the CPU with the oracle's plain copy; the GPU tests plug in the
library's kernels.
"""
from __future__ import annotations

import zlib

import numpy as np

from oracle import block_model as M
from paged_kv_cache_367_b200.blocks import BlockManager


def token_row(prefix_tokens, shape, seed) -> tuple[np.ndarray, np.ndarray]:
    """K and V rows (float32, `shape`) determined by the token-id prefix."""
    key = zlib.crc32(np.asarray(prefix_tokens, dtype=np.int32).tobytes(), seed)
    r = np.random.default_rng(key)
    return (r.standard_normal(shape).astype(np.float32),
            r.standard_normal(shape).astype(np.float32))


class NumpyPools:
    """Device and host pools as numpy arrays (float32 rows)."""

    def __init__(self, num_blocks, num_host_blocks, bs, row_shape):
        self.k = np.full((num_blocks, bs) + row_shape, np.nan, np.float32)
        self.v = np.full_like(self.k, np.nan)
        self.hk = np.full((max(num_host_blocks, 1), bs) + row_shape, np.nan, np.float32)
        self.hv = np.full_like(self.hk, np.nan)

    def write(self, slots, k_rows, v_rows):
        bs = self.k.shape[1]
        for s, kr, vr in zip(slots, k_rows, v_rows):
            if s >= 0:
                self.k[s // bs, s % bs] = kr
                self.v[s // bs, s % bs] = vr

    def copy(self, pairs):
        M.copy_blocks(self.k, self.v, self.k, self.v, pairs)

    def swap_out(self, pairs):
        M.copy_blocks(self.k, self.v, self.hk, self.hv, pairs)

    def swap_in(self, pairs):
        M.copy_blocks(self.hk, self.hv, self.k, self.v, pairs)

    def device_pools(self):
        return self.k, self.v


class Trace:
    def __init__(self, pools, *, num_blocks, bs, num_host_blocks=0, prefix_caching=False,
                 row_shape=(1, 4), seed=0, vocab=6, quantize=None):
        self.bm = BlockManager(num_blocks, bs, num_host_blocks, prefix_caching)
        self.model = M.LogicalSequences()
        self.pools = pools
        self.bs, self.num_blocks, self.row_shape = bs, num_blocks, row_shape
        self.rng = np.random.default_rng(seed)
        self.seed, self.vocab = seed, vocab
        self.quantize = quantize or (lambda a: a)  # rows as the pool stores them
        self.next_id = 1
        self.swapped: set[int] = set()
        self.prompts = [list(self.rng.integers(0, vocab, size=n))
                        for n in (0, bs, 2 * bs + 3, 3 * bs)]
        self.stats = dict(cow=0, cached=0, swap_out=0, swap_in=0, no_blocks=0)

    def rows_for(self, tokens, start):
        ks, vs = zip(*[self.row(tokens[:t + 1]) for t in range(start, len(tokens))]) \
            if len(tokens) > start else ((), ())
        return list(ks), list(vs)

    def row(self, prefix_tokens):
        k, v = token_row(prefix_tokens, self.row_shape, self.seed)
        return self.quantize(k), self.quantize(v)

    def resident(self):
        return [s for s in self.model.tokens if s not in self.swapped]

    # -- operations ------------------------------------------------------------
    def admit(self):
        base = self.prompts[self.rng.integers(len(self.prompts))]
        toks = base + list(self.rng.integers(0, self.vocab, size=self.rng.integers(0, 2 * self.bs)))
        if not self.bm.can_allocate(len(toks)):
            self.stats["no_blocks"] += 1
            return
        sid = self.next_id
        self.next_id += 1
        slots, cached = self.bm.allocate(sid, toks)
        assert cached % self.bs == 0 and cached <= len(toks)
        assert np.all(slots[:cached] == -1)
        self.stats["cached"] += cached
        k, v = self.rows_for(toks, 0)
        self.pools.write(slots, k, v)
        self.model.add(sid, toks, k, v)

    def append(self):
        res = self.resident()
        if not res:
            return
        sid = res[self.rng.integers(len(res))]
        if not self.bm.can_append(sid):
            self.stats["no_blocks"] += 1
            return
        tok = int(self.rng.integers(0, self.vocab))
        slot, src, dst = self.bm.append_slot(sid, tok)
        if src >= 0:
            self.stats["cow"] += 1
            self.pools.copy(np.array([[src, dst]], dtype=np.int64))
        toks = self.model.tokens[sid] + [tok]
        k, v = self.row(toks)
        self.pools.write([slot], [k], [v])
        self.model.append(sid, tok, k, v)

    def decode_step(self):
        """One batched decode step: every resident sequence gets a token."""
        res = self.resident()
        if not res:
            return
        toks = [int(t) for t in self.rng.integers(0, self.vocab, size=len(res))]
        try:
            slots, cow = self.bm.append_slots(res, toks)
        except Exception:
            self.stats["no_blocks"] += 1
            return
        if len(cow):
            self.stats["cow"] += len(cow)
            self.pools.copy(cow)
        ks, vs = [], []
        for sid, tok in zip(res, toks):
            k, v = self.row(self.model.tokens[sid] + [tok])
            self.model.append(sid, tok, k, v)
            ks.append(k)
            vs.append(v)
        self.pools.write(slots, ks, vs)

    def fork(self):
        res = self.resident()
        if not res:
            return
        parent = res[self.rng.integers(len(res))]
        child = self.next_id
        self.next_id += 1
        self.bm.fork(parent, child)
        self.model.fork(parent, child)

    def free(self):
        ids = list(self.model.tokens)
        if not ids:
            return
        sid = ids[self.rng.integers(len(ids))]
        self.bm.free(sid)
        self.model.remove(sid)
        self.swapped.discard(sid)

    def swap_out(self):
        res = self.resident()
        if not res:
            return
        group = list(self.rng.choice(res, size=min(len(res), 1 + self.rng.integers(3)),
                                     replace=False))
        try:
            pairs = self.bm.swap_out(group)
        except Exception:
            self.stats["no_blocks"] += 1
            return
        self.stats["swap_out"] += 1
        self.pools.swap_out(pairs)
        self.swapped |= set(int(g) for g in group)

    def swap_in(self):
        if not self.swapped:
            return
        sw = sorted(self.swapped)
        group = list(self.rng.choice(sw, size=min(len(sw), 1 + self.rng.integers(2)),
                                     replace=False))
        try:
            pairs = self.bm.swap_in(group)
        except Exception:
            self.stats["no_blocks"] += 1
            return
        self.stats["swap_in"] += 1
        self.pools.swap_in(pairs)
        self.swapped -= set(int(g) for g in group)

    def step(self, swaps=True):
        ops = [self.admit, self.append, self.append, self.decode_step, self.fork, self.free]
        if swaps:
            ops += [self.swap_out, self.swap_in]
        ops[self.rng.integers(len(ops))]()

    # -- checks ------------------------------------------------------------------
    def tables(self, ids=None):
        ids = self.resident() if ids is None else ids
        mb = max([M.blocks_needed(self.model.length(s), self.bs) for s in ids] + [1])
        return ids, *self.bm.block_tables(ids, mb)

    def check_ledger(self):
        """Ledger invariants against the plain model (no pool contents)."""
        self.bm.check()
        ids, table, lens = self.tables()
        held = set()
        for i, s in enumerate(ids):
            L = self.model.length(s)
            assert lens[i] == L
            nb = M.blocks_needed(L, self.bs)
            assert np.all(table[i, :nb] >= 0) and np.all(table[i, nb:] == -1)
            held |= set(table[i, :nb].tolist())
        assert self.bm.num_free == self.num_blocks - len(held)
        # A block is shared only by sequences whose tokens agree up to its end.
        owner = {}
        for i, s in enumerate(ids):
            for j in range(M.blocks_needed(self.model.length(s), self.bs)):
                owner.setdefault(int(table[i, j]), []).append((s, j))
        for b, users in owner.items():
            assert self.bm.refcount(b) >= len(users)
            (s0, j0) = users[0]
            for s, j in users[1:]:
                assert j == j0
                end = min((j + 1) * self.bs, self.model.length(s), self.model.length(s0))
                assert self.model.tokens[s][:end] == self.model.tokens[s0][:end]

    def check_contents(self, pool_k, pool_v):
        """Every resident sequence's rows, gathered through its block table,
        equal the model's rows exactly."""
        ids, table, lens = self.tables()
        for i, s in enumerate(ids):
            L = int(lens[i])
            if L == 0:
                continue
            k, v = self.model.rows(s)
            assert np.array_equal(M.gather(pool_k, table[i], L, self.bs), k), s
            assert np.array_equal(M.gather(pool_v, table[i], L, self.bs), v), s
