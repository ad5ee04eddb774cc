"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU involved).

Each pin takes `mutant`: None checks the real oracle; a macro name checks a build with one planted
mistake (tests/test_oracle_mutants.py asserts that every planted mistake fails at least one pin).
Scenarios are built here, on the test side, by placing contiguous per-request K/V into a pool with
NumPy block reshapes; the oracle must read them back through the tables.
"""
import json
import math
import os

import numpy as np
import torch

import oracle
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
BS = 16


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def draw(dtype, shape, rng):
    """(storage array handed to the oracle, exact float64 values of those stored elements)."""
    x = rng.standard_normal(shape).astype(np.float32)
    if dtype == "f32":
        return x, x.astype(np.float64)
    if dtype == "f16":
        h = x.astype(np.float16)
        return h.view(np.uint16), h.astype(np.float64)
    t = torch.from_numpy(x).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy(), t.to(torch.float64).numpy()


class Scenario:
    """Requests given as (prior, n) pairs over a shuffled pool, with their contiguous K/V kept aside."""

    def __init__(self, rng, dtype, Hq, Hkv, D, specs, extra_blocks=3, scale=None):
        self.dtype, self.Hq, self.Hkv, self.D = dtype, Hq, Hkv, D
        self.specs = specs
        self.ctx = np.asarray([p + n for p, n in specs], dtype=np.int32)
        self.qsl = np.concatenate([[0], np.cumsum([n for _, n in specs])]).astype(np.int32)
        need = [math.ceil(c / BS) for c in self.ctx]
        self.NB = sum(need) + extra_blocks
        perm = rng.permutation(self.NB).astype(np.int32)
        self.bt = np.full((len(specs), max(need)), -1, dtype=np.int32)
        pos = 0
        for r, k in enumerate(need):
            self.bt[r, :k] = perm[pos:pos + k]
            pos += k
        self.k_pool, _ = draw(dtype, (self.NB, Hkv, BS, D), rng)       # stale filler everywhere
        self.v_pool, _ = draw(dtype, (self.NB, Hkv, BS, D), rng)
        self.K, self.V = [], []
        for r, c in enumerate(self.ctx):
            Ks, K64 = draw(dtype, (int(c), Hkv, D), rng)
            Vs, V64 = draw(dtype, (int(c), Hkv, D), rng)
            self.place(self.k_pool, self.bt[r], Ks)
            self.place(self.v_pool, self.bt[r], Vs)
            self.K.append(K64)
            self.V.append(V64)
        self.q, self.q64 = draw(dtype, (int(self.qsl[-1]), Hq, D), rng)
        self.scale = float(np.float32(1.0 / math.sqrt(D))) if scale is None else scale

    @staticmethod
    def place(pool, table_row, X):
        """Write contiguous rows X [ctx, Hkv, D] into the pool blocks listed by table_row."""
        c, Hkv, D = X.shape
        nb = math.ceil(c / BS)
        blocks = pool[table_row[:nb]].transpose(0, 2, 1, 3).reshape(nb * BS, Hkv, D).copy()
        blocks[:c] = X
        pool[table_row[:nb]] = blocks.reshape(nb, BS, Hkv, D).transpose(0, 2, 1, 3)

    def run(self, mutant=None, **kw):
        args = dict(q=self.q, k_pool=self.k_pool, v_pool=self.v_pool, block_tables=self.bt,
                    context_lens=self.ctx, query_start_loc=self.qsl, scale=self.scale, dtype=self.dtype)
        args.update(kw)
        return oracle.paged_attention(mutant=mutant, **args)

    def brute(self, r):
        prior, n = self.specs[r]
        rows = slice(self.qsl[r], self.qsl[r + 1])
        return brute.contiguous_attention(self.q64[rows], self.K[r], self.V[r], prior, self.scale)


CASES = [
    # dtype, Hq, Hkv, D, [(prior, n)]
    ("f32", 4, 4, 16, [(0, 1), (16, 1), (40, 1), (99, 1)]),
    ("f16", 8, 2, 16, [(0, 5), (33, 1), (20, 19)]),
    ("bf16", 6, 3, 8, [(47, 3), (0, 1), (15, 2), (64, 1)]),
    ("f32", 8, 1, 64, [(5, 12), (0, 33)]),
    ("bf16", 4, 4, 64, [(0, 1), (31, 1), (16, 17)]),
]


def pin_brute_force(mutant=None):
    """Paged result == contiguous attention (blog.mckayzhao.com/?p=56, PagedAttention section)."""
    for i, (dt, Hq, Hkv, D, specs) in enumerate(CASES):
        sc = Scenario(np.random.default_rng(100 + i), dt, Hq, Hkv, D, specs)
        out = sc.run(mutant)
        for r in range(len(specs)):
            ref = sc.brute(r)
            got = out[sc.qsl[r]:sc.qsl[r + 1]]
            err = np.max(np.abs(got - ref)) if ref.size else 0.0
            assert np.all(np.isfinite(got)) and err <= 1e-10, f"case {i} req {r}: max err {err}"


def pin_permutation(mutant=None):
    """Relabelling physical blocks (permuting the pool and the tables together) changes nothing, bit for bit."""
    rng = np.random.default_rng(7)
    sc = Scenario(rng, "f16", 8, 4, 16, [(30, 1), (7, 9), (50, 1)], extra_blocks=5)
    base = sc.run(mutant)
    pi = rng.permutation(sc.NB).astype(np.int32)
    kp = np.empty_like(sc.k_pool)
    vp = np.empty_like(sc.v_pool)
    kp[pi] = sc.k_pool
    vp[pi] = sc.v_pool
    bt = np.where(sc.bt >= 0, pi[np.maximum(sc.bt, 0)], -1).astype(np.int32)
    out = sc.run(mutant, k_pool=kp, v_pool=vp, block_tables=bt)
    assert np.array_equal(out, base)


def pin_closed_forms(mutant=None):
    """ctx = 1 gives v0 exactly; equal keys or scale 0 give the mean of V."""
    rng = np.random.default_rng(11)
    sc = Scenario(rng, "f32", 4, 2, 16, [(0, 1)])
    out = sc.run(mutant)
    assert np.array_equal(out[0], np.repeat(sc.V[0][0], 2, axis=0)), "ctx=1 must return v0"
    sc = Scenario(rng, "f32", 4, 2, 16, [(36, 1)], scale=0.0)
    out = sc.run(mutant)
    ref = np.repeat(sc.V[0].mean(axis=0), 2, axis=0)
    assert np.max(np.abs(out[0] - ref)) < 1e-12, "scale=0 must average V"
    sc = Scenario(rng, "f32", 4, 2, 16, [(36, 1)])
    same = np.broadcast_to(sc.K[0][:1], sc.K[0].shape).astype(np.float32)
    Scenario.place(sc.k_pool, sc.bt[0], same)
    out = sc.run(mutant)
    ref = np.repeat(sc.V[0].mean(axis=0), 2, axis=0)
    assert np.max(np.abs(out[0] - ref)) < 1e-12, "identical keys must average V"


def pin_chunked_equals_incremental(mutant=None):
    """Chunked-prefill row j at prior P == a decode row with context P+j+1 over the same blocks."""
    rng = np.random.default_rng(13)
    sc = Scenario(rng, "bf16", 4, 2, 16, [(21, 11)])
    chunk = sc.run(mutant)
    for j in range(11):
        dec = sc.run(mutant, q=sc.q[j:j + 1], context_lens=np.asarray([21 + j + 1], np.int32),
                     query_start_loc=np.asarray([0, 1], np.int32))
        assert np.array_equal(dec[0], chunk[j]), f"row {j}"


def pin_batch_independence(mutant=None):
    """A request's output does not depend on which other requests share the batch."""
    rng = np.random.default_rng(17)
    sc = Scenario(rng, "f16", 4, 4, 16, [(10, 1), (3, 6), (40, 1)])
    full = sc.run(mutant)
    r = 1
    alone = sc.run(mutant, q=sc.q[sc.qsl[r]:sc.qsl[r + 1]], block_tables=sc.bt[r:r + 1],
                   context_lens=sc.ctx[r:r + 1], query_start_loc=np.asarray([0, 6], np.int32))
    assert np.array_equal(alone, full[sc.qsl[r]:sc.qsl[r + 1]])


def pin_sharing(mutant=None):
    """Tables pointing at one shared copy of a prefix give the same output as private copies.

    Layout from 一文搞懂vLLM, "PagedAttention 是怎么共享内存的" figure: shared B1, B2 plus one own block each.
    """
    g = golden("sharing_figure.json")
    rng = np.random.default_rng(19)
    Hkv, D = 2, 16
    seqs = list(g["own"].keys())
    shared_ids = [int(b[1:]) - 1 for b in g["shared"]]
    own_ids = [int(g["own"][s][1:]) - 1 for s in seqs]
    NB = 12
    kp, _ = draw("f16", (NB, Hkv, BS, D), rng)
    vp, _ = draw("f16", (NB, Hkv, BS, D), rng)
    tails = [5, 16, 1]
    ctx = np.asarray([2 * BS + t for t in tails], np.int32)
    bt_shared = np.asarray([shared_ids + [o] for o in own_ids], np.int32)
    q, _ = draw("f16", (len(seqs), 4, D), rng)
    qsl = np.arange(len(seqs) + 1, dtype=np.int32)
    shared_out = oracle.paged_attention(q, kp, vp, bt_shared, ctx, qsl, 0.25, "f16", mutant=mutant)
    # Private copies of the shared blocks for every sequence (free ids 7..11 and beyond).
    kp2, vp2 = kp.copy(), vp.copy()
    kp2 = np.concatenate([kp2, np.zeros((2 * len(seqs), Hkv, BS, D), kp.dtype)])
    vp2 = np.concatenate([vp2, np.zeros((2 * len(seqs), Hkv, BS, D), vp.dtype)])
    bt_priv = bt_shared.copy()
    for s in range(len(seqs)):
        for i, b in enumerate(shared_ids):
            nid = NB + 2 * s + i
            kp2[nid] = kp[b]
            vp2[nid] = vp[b]
            bt_priv[s, i] = nid
    priv_out = oracle.paged_attention(q, kp2, vp2, bt_priv, ctx, qsl, 0.25, "f16", mutant=mutant)
    assert np.array_equal(shared_out, priv_out)
    assert not np.array_equal(shared_out[0], shared_out[1])


def pin_slot_mapping_figure(mutant=None):
    """Slots of request A of the block-pool figure (table B1, B4, B7) fill B1, then B4, then B7."""
    g = golden("block_pool_figure.json")
    ids = [int(b[1:]) - 1 for b in g["tables"]["A"]]
    bs = g["block_size"]
    n = 2 * bs + 5                                   # three blocks: the last one partly filled
    expect = []
    for b in ids:                                    # enumerate each block's slots in order
        expect.extend(range(b * bs, b * bs + bs))
    expect = np.asarray(expect[:n], dtype=np.int64)
    bt = np.asarray([ids], np.int32)
    got = oracle.slot_mapping(bt, np.asarray([0, n], np.int32), np.asarray([n], np.int32), bs, mutant=mutant)
    assert np.array_equal(got, expect)
    # Decode step: the (n+1)-th token of A goes to the slot right after the last one.
    got1 = oracle.slot_mapping(bt, np.asarray([0, 1], np.int32), np.asarray([n + 1], np.int32), bs, mutant=mutant)
    assert got1[0] == ids[2] * bs + 5


def pin_append_then_attend(mutant=None):
    """Appending a token's K/V through its slot, then attending, equals contiguous attention over the
    grown sequence (一文搞懂vLLM, "快速回顾 prefill、decode 和 KV cache": each token adds one entry)."""
    rng = np.random.default_rng(23)
    sc = Scenario(rng, "f16", 4, 2, 16, [(18, 1), (31, 1), (0, 1)])
    kn, kn64 = draw("f16", (3, 2, 16), rng)
    vn, vn64 = draw("f16", (3, 2, 16), rng)
    slots = oracle.slot_mapping(sc.bt, sc.qsl, sc.ctx, mutant=mutant)
    oracle.kv_cache_write(kn, vn, sc.k_pool, sc.v_pool, slots, mutant=mutant)
    out = sc.run(mutant)
    for r in range(3):
        K = sc.K[r].copy()
        V = sc.V[r].copy()
        K[-1] = kn64[r]
        V[-1] = vn64[r]
        ref = brute.contiguous_attention(sc.q64[r:r + 1], K, V, sc.specs[r][0], sc.scale)
        assert np.max(np.abs(out[r:r + 1] - ref)) <= 1e-10, f"request {r}"


def pin_copy_on_write(mutant=None):
    """Copy the shared block, modify only the copy; the original stays bit-identical
    (blog.mckayzhao.com/?p=56, "还不止是分页：Copy-on-Write 和内存共享")."""
    rng = np.random.default_rng(29)
    NB, Hkv, D = 6, 2, 16
    kp, _ = draw("f16", (NB, Hkv, BS, D), rng)
    vp, _ = draw("f16", (NB, Hkv, BS, D), rng)
    src, dst = 1, 4
    k_src, v_src = kp[src].copy(), vp[src].copy()
    others = [b for b in range(NB) if b != dst]
    k_others, v_others = kp[others].copy(), vp[others].copy()
    oracle.copy_blocks([kp], [vp], np.asarray([[src, dst]], np.int32), mutant=mutant)
    assert np.array_equal(kp[dst], k_src) and np.array_equal(vp[dst], v_src), "copy must equal source"
    # The sequence that owns the copy appends a token at offset 9 of its (formerly shared) block.
    kn, _ = draw("f16", (1, Hkv, D), rng)
    vn, _ = draw("f16", (1, Hkv, D), rng)
    oracle.kv_cache_write(kn, vn, kp, vp, np.asarray([dst * BS + 9], np.int64), mutant=mutant)
    assert np.array_equal(kp[others], k_others) and np.array_equal(vp[others], v_others), "source changed"
    assert np.array_equal(kp[dst][:, 9], kn[0]) and np.array_equal(vp[dst][:, 9], vn[0])
    keep = [i for i in range(BS) if i != 9]
    assert np.array_equal(kp[dst][:, keep], k_src[:, keep]) and np.array_equal(vp[dst][:, keep], v_src[:, keep])


def pin_block_accounting(mutant=None):
    """ceil(N/16) blocks and at most 15 wasted slots; the naive-reservation worked example."""
    acc = golden("block_accounting.json")
    bs = acc["block_size"]
    for n in list(range(0, 70)) + [1000, 1024, 1025, 2047, 2048, 33280]:
        nb = oracle.blocks_for_tokens(n, bs, mutant=mutant)
        assert nb == math.ceil(n / bs)
        assert 0 <= oracle.wasted_slots(n, bs, mutant=mutant) <= acc["max_wasted_slots"]
    nv = golden("naive_reservation.json")
    for name, used in nv["used"].items():
        assert brute.naive_reserved_waste(used, nv["reserved_tokens"]) == nv["naive_wasted"][name]
        paged = oracle.wasted_slots(used, bs, mutant=mutant)
        assert paged == {"A": 14, "B": 8, "C": 12}[name]
        assert paged < nv["naive_wasted"][name]
    fig = golden("block_pool_figure.json")
    for name, blocks in fig["tables"].items():
        k = len(blocks)
        assert oracle.blocks_for_tokens(bs * (k - 1) + 1, bs, mutant=mutant) == k
        assert oracle.blocks_for_tokens(bs * k, bs, mutant=mutant) == k
    used = {b for t in fig["tables"].values() for b in t}
    assert sorted(set(fig["pool_blocks"]) - used) == fig["free"]


def pin_storage_decoders(mutant=None):
    """The oracle's binary16 / bfloat16 decoders agree with NumPy's and torch's conversions on every
    finite bit pattern."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    h = bits.view(np.float16).astype(np.float64)
    b = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    lib = oracle.load(mutant)
    for i in range(0, 1 << 16, 7):
        if np.isfinite(h[i]):
            assert lib.oracle_half_to_double(int(bits[i])) == h[i], f"half {i:#06x}"
        if np.isfinite(b[i]):
            assert lib.oracle_bf16_to_double(int(bits[i])) == b[i], f"bf16 {i:#06x}"


def pin_flatten_batch(mutant=None):
    """blog.mckayzhao.com/?p=56, "V1 架构：推倒重来的勇气": a step is {request_id: num_tokens}. Hand-derived
    flattenings (tests/golden/flatten_batch.json) -- mixed prefill/decode rows, requests with 0 tokens,
    ids out of order, an empty step -- and, on seeded random dicts, the defining properties: request
    r's rows are the range [query_start_loc[r], query_start_loc[r+1]) of length num_tokens, laid out
    in the dict's order, and context_lens[r] = prior + num_tokens."""
    for case in golden("flatten_batch.json")["cases"]:
        batch = {int(r): int(n) for r, n in case["batch"]}
        qsl, ctx = oracle.flatten_batch(batch, case["prior_lens"], mutant=mutant)
        assert qsl.dtype == np.int32 and ctx.dtype == np.int32
        assert qsl.tolist() == case["query_start_loc"], (case["name"], qsl.tolist())
        assert ctx.tolist() == case["context_lens"], (case["name"], ctx.tolist())
    rng = np.random.default_rng(7)
    for _ in range(50):
        R = int(rng.integers(0, 40))
        ids = rng.permutation(1000)[:R]
        counts = rng.integers(0, 600, R) * (rng.random(R) < 0.8)
        prior = rng.integers(0, 40000, R)
        batch = {int(i): int(c) for i, c in zip(ids, counts)}
        qsl, ctx = oracle.flatten_batch(batch, prior, mutant=mutant)
        assert qsl.shape == (R + 1,) and ctx.shape == (R,) and qsl[0] == 0
        for r, (rid, n) in enumerate(batch.items()):
            assert qsl[r + 1] - qsl[r] == n, (rid, n)
            assert ctx[r] == prior[r] + n


ALL_PINS = [pin_brute_force, pin_permutation, pin_closed_forms, pin_chunked_equals_incremental,
            pin_batch_independence, pin_sharing, pin_slot_mapping_figure, pin_append_then_attend,
            pin_copy_on_write, pin_block_accounting, pin_storage_decoders, pin_flatten_batch]
