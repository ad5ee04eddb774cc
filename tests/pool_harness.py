"""Test-side helpers for block-pool bookkeeping: a content simulator and random operation scripts.

ContentCheck stores a distinct token value in every slot a sequence writes, following that
sequence's block list, performs the copy-on-write copies an append reports, and checks that every
live sequence reads back exactly its own tokens in order -- what contiguous per-sequence storage
would return (blog.mckayzhao.com/?p=56, "PagedAttention：操作系统课本里翻出来的灵感" and
"还不止是分页：Copy-on-Write 和内存共享"). It works on any manager exposed through the small adapter
interface below (the oracle model or the product's host block manager).
"""
import numpy as np

from oracle.block_pool import BlockPool, OutOfBlocks


class OracleAdapter:
    def __init__(self, num_blocks, block_size=16, mutant=None, prefix_cache=False):
        self.m = BlockPool(num_blocks, block_size, mutant, prefix_cache)
        self.block_size = block_size

    def add(self, s, n):
        self.m.add(s, n)

    def prompt(self, s, tokens):
        """Starts s from its cached prefix and appends the rest of the prompt; returns
        (cached tokens, copy pairs)."""
        cached = self.m.add_cached_prefix(s, list(tokens))
        try:
            return cached, self.m.append(s, len(tokens) - cached, list(tokens[cached:]))
        except OutOfBlocks:
            self.m.free(s)                   # no room for the rest: give the prompt up entirely
            raise

    def fork(self, p, c):
        self.m.fork(p, c)

    def append(self, s, n, tokens=None):
        return self.m.append(s, n, None if tokens is None else list(tokens))

    def free(self, s):
        self.m.free(s)

    def table(self, s):
        return list(self.m.tables[s])

    def length(self, s):
        return self.m.lengths[s]

    def holders(self, b):
        return self.m.holders[b]

    def stats(self):
        return self.m.stats()

    def step(self, batch, tokens=None):
        return self.m.step(batch, tokens)


class ProductAdapter:
    def __init__(self, num_blocks, block_size=16, prefix_cache=False):
        from paged_kv_cache_446_b200 import pkv
        self.pkv = pkv
        self.m = pkv.BlockManager(num_blocks, block_size, prefix_cache=prefix_cache)
        self.block_size = block_size

    def _guard(self, fn, *a):
        try:
            return fn(*a)
        except self.pkv.PkvError as e:
            if e.status == self.pkv.PKV_ERR_OUT_OF_BLOCKS:
                raise OutOfBlocks() from e
            raise

    def add(self, s, n):
        self._guard(self.m.add, s, n)

    def prompt(self, s, tokens):
        cached = self.m.add_cached_prefix(s, tokens)
        try:
            pair = self._guard(self.m.append, s, len(tokens) - cached, tokens[cached:])
        except OutOfBlocks:
            self.m.free(s)                   # no room for the rest: give the prompt up entirely
            raise
        return cached, [] if pair is None else [pair]

    def fork(self, p, c):
        self.m.fork(p, c)

    def append(self, s, n, tokens=None):
        pair = self._guard(self.m.append, s, n, tokens)
        return [] if pair is None else [pair]

    def free(self, s):
        self.m.free(s)

    def table(self, s):
        return self.m.sequence(s)[1]

    def length(self, s):
        return self.m.sequence(s)[0]

    def holders(self, b):
        return self.m.refcount(b)

    def stats(self):
        return self.m.stats()

    def step(self, batch, tokens=None):
        max_blocks = max([-(-(self.length(s) + n) // self.block_size) for s, n in batch.items()] + [1])
        tables, ctx, qsl, pairs = self._guard(self.m.step, batch, max_blocks, tokens)
        return ([[int(b) for b in row if b >= 0] for row in tables], ctx.tolist(), qsl.tolist(),
                [tuple(int(x) for x in p) for p in pairs])


class ContentCheck:
    """Drives a manager and mirrors slot contents; check() verifies what every sequence reads."""

    def __init__(self, mgr, num_blocks):
        self.mgr = mgr
        self.bs = mgr.block_size
        self.slots = np.full((num_blocks, self.bs), -1, np.int64)
        self.logical = {}
        self.next_value = 0

    def _write(self, s, first, n):
        table = self.mgr.table(s)
        for p in range(first, first + n):
            b = table[p // self.bs]
            self.slots[b, p % self.bs] = self.next_value
            self.logical[s].append(self.next_value)
            self.next_value += 1

    def _copy(self, pairs):
        for src, dst in pairs:
            self.slots[dst] = self.slots[src]

    def add(self, s, n):
        self.mgr.add(s, n)
        self.logical[s] = []
        self._write(s, 0, n)

    def fork(self, p, c):
        self.mgr.fork(p, c)
        self.logical[c] = list(self.logical[p])

    def append(self, s, n):
        first = len(self.logical[s])
        pairs = self.mgr.append(s, n)
        self._copy(pairs)
        self._write(s, first, n)
        return pairs

    def step(self, batch):
        firsts = {s: len(self.logical[s]) for s in batch}
        out = self.mgr.step(batch)
        self._copy(out[3])
        for s, n in batch.items():
            self._write(s, firsts[s], n)
        return out

    def free(self, s):
        self.mgr.free(s)
        del self.logical[s]

    def check(self):
        for s, vals in self.logical.items():
            table = self.mgr.table(s)
            assert self.mgr.length(s) == len(vals)
            got = [self.slots[table[p // self.bs], p % self.bs] for p in range(len(vals))]
            assert got == vals, f"sequence {s} reads {got[:8]}... expected {vals[:8]}..."


def random_script(seed, num_ops=300, max_len=70):
    """A seeded list of operations: ('add', s, n), ('fork', p, c), ('append', s, n), ('free', s),
    ('step', {s: n}). Ids refer to sequences live at that point of the script."""
    rng = np.random.default_rng(seed)
    live, ops, next_id = [], [], 0
    for _ in range(num_ops):
        r = rng.random()
        if not live or r < 0.15:
            n = int(rng.integers(0, max_len))
            ops.append(("add", next_id, n))
            live.append(next_id)
            next_id += 1
        elif r < 0.35:
            p = live[int(rng.integers(len(live)))]
            ops.append(("fork", p, next_id))
            live.append(next_id)
            next_id += 1
        elif r < 0.7:
            s = live[int(rng.integers(len(live)))]
            ops.append(("append", s, int(rng.choice([0, 1, 1, 1, 3, 15, 16, 17, 40]))))
        elif r < 0.85:
            k = int(rng.integers(1, len(live) + 1))
            chosen = rng.choice(len(live), size=k, replace=False)
            ops.append(("step", {live[i]: int(rng.choice([0, 1, 1, 2, 9, 16])) for i in chosen}))
        else:
            s = live.pop(int(rng.integers(len(live))))
            ops.append(("free", s))
    return ops


def run_script(target, ops, after_each=None):
    """Applies scripted ops in order, skipping any that name a sequence not live (an add that ran
    out of blocks leaves its id unused). Returns one outcome per op: ('ok', result),
    ('out_of_blocks', None) or ('skipped', None). after_each(i, op, outcome) runs after every op."""
    live, out = set(), []
    for i, op in enumerate(ops):
        kind = op[0]
        if kind == "step":
            batch = {s: n for s, n in op[1].items() if s in live}
            op = ("step", batch)
            skip = not batch
        elif kind == "add":
            skip = False
        else:
            skip = op[1] not in live
        if skip:
            res = ("skipped", None)
        else:
            try:
                if kind == "add":
                    res = ("ok", target.add(op[1], op[2]))
                    live.add(op[1])
                elif kind == "fork":
                    res = ("ok", target.fork(op[1], op[2]))
                    live.add(op[2])
                elif kind == "append":
                    res = ("ok", target.append(op[1], op[2]))
                elif kind == "step":
                    res = ("ok", target.step(op[1]))
                else:
                    res = ("ok", target.free(op[1]))
                    live.discard(op[1])
            except OutOfBlocks:
                res = ("out_of_blocks", None)
        out.append(res)
        if after_each:
            after_each(i, op, res)
    return out


def prefix_value(ids):
    """What a token's K/V would be: a function of every token id up to and including it."""
    return hash(tuple(ids))


class PrefixContentCheck:
    """Like ContentCheck, for token-tracked sequences: a stored slot holds prefix_value of the
    sequence's ids up to that position, so a block reused from the prefix cache reads back right
    only if it holds exactly the prefix the new sequence starts with. Cached prompt tokens are not
    written (their K/V are reused, not computed again)."""

    def __init__(self, mgr, num_blocks):
        self.mgr = mgr
        self.bs = mgr.block_size
        self.slots = np.full((num_blocks, self.bs), -1, dtype=object)
        self.ids = {}
        self.cached_tokens = 0
        self.prompt_tokens = 0

    def _write(self, s, first):
        table = self.mgr.table(s)
        ids = self.ids[s]
        for p in range(first, len(ids)):
            self.slots[table[p // self.bs], p % self.bs] = prefix_value(ids[:p + 1])

    def _copy(self, pairs):
        for src, dst in pairs:
            self.slots[dst] = self.slots[src]

    def prompt(self, s, tokens):
        cached, pairs = self.mgr.prompt(s, tokens)
        assert 0 <= cached < max(len(tokens), 1) and cached % self.bs == 0
        self.ids[s] = list(tokens)
        self._copy(pairs)
        self._write(s, cached)
        self.cached_tokens += cached
        self.prompt_tokens += len(tokens)
        return cached

    def fork(self, p, c):
        self.mgr.fork(p, c)
        self.ids[c] = list(self.ids[p])

    def append(self, s, n, tokens):
        first = len(self.ids[s])
        pairs = self.mgr.append(s, n, tokens)
        self.ids[s] += list(tokens)
        self._copy(pairs)
        self._write(s, first)
        return pairs

    def step(self, batch, tokens):
        firsts = {s: len(self.ids[s]) for s in batch}
        out = self.mgr.step(batch, tokens)
        at = 0
        for s, n in batch.items():
            self.ids[s] += list(tokens[at:at + n])
            at += n
        self._copy(out[3])
        for s in batch:
            self._write(s, firsts[s])
        return out

    def free(self, s):
        self.mgr.free(s)
        del self.ids[s]

    def check(self):
        for s, ids in self.ids.items():
            table = self.mgr.table(s)
            assert self.mgr.length(s) == len(ids)
            for p in range(len(ids)):
                assert self.slots[table[p // self.bs], p % self.bs] == prefix_value(ids[:p + 1]), \
                    f"sequence {s} position {p} reads another prefix's K/V"


def random_cache_script(seed, num_ops=200, vocab=50):
    """Seeded ops for prefix-caching managers: ('prompt', s, ids) starts a request whose prompt is
    a shared system prompt plus a suffix, or a finished conversation continued (history + a new
    message); ('append', s, n, ids); ('step', {s: n}, ids); ('fork', p, c); ('free', s)."""
    rng = np.random.default_rng(seed)
    systems = [list(rng.integers(0, vocab, size=n)) for n in (16, 20, 37, 64)]
    history, live, ops, next_id = [], [], [], 0
    full = {}

    def toks(n):
        return [int(x) for x in rng.integers(0, vocab, size=n)]

    for _ in range(num_ops):
        r = rng.random()
        if not live or r < 0.25:
            if history and rng.random() < 0.4:
                base = history[int(rng.integers(len(history)))]
            else:
                base = systems[int(rng.integers(len(systems)))]
            ids = [int(x) for x in base] + toks(int(rng.choice([0, 1, 5, 16, 30])))
            if not ids:
                ids = toks(1)
            ops.append(("prompt", next_id, ids))
            full[next_id] = list(ids)
            live.append(next_id)
            next_id += 1
        elif r < 0.35:
            p = live[int(rng.integers(len(live)))]
            ops.append(("fork", p, next_id))
            full[next_id] = list(full[p])
            live.append(next_id)
            next_id += 1
        elif r < 0.6:
            s = live[int(rng.integers(len(live)))]
            n = int(rng.choice([1, 1, 3, 16, 20]))
            t = toks(n)
            ops.append(("append", s, n, t))
            full[s] += t
        elif r < 0.75:
            k = int(rng.integers(1, len(live) + 1))
            chosen = [live[i] for i in rng.choice(len(live), size=k, replace=False)]
            batch = {s: int(rng.choice([0, 1, 1, 4])) for s in chosen}
            t = toks(sum(batch.values()))
            at = 0
            for s2, n2 in batch.items():
                full[s2] += t[at:at + n2]
                at += n2
            ops.append(("step", batch, t))
        else:
            s = live.pop(int(rng.integers(len(live))))
            history.append(full[s])
            ops.append(("free", s))
    return ops


def run_cache_script(target, ops, after_each=None):
    """Like run_script, for random_cache_script ops. A prompt that runs out of blocks leaves its id
    unused; later ops naming a sequence not live are skipped (a step keeps its live members and
    their token ids)."""
    live, out = set(), []
    for i, op in enumerate(ops):
        kind = op[0]
        res = ("skipped", None)
        try:
            if kind == "prompt":
                res = ("ok", target.prompt(op[1], op[2]))
                live.add(op[1])
            elif kind == "fork" and op[1] in live:
                res = ("ok", target.fork(op[1], op[2]))
                live.add(op[2])
            elif kind == "append" and op[1] in live:
                res = ("ok", target.append(op[1], op[2], op[3]))
            elif kind == "step":
                at, batch, t = 0, {}, []
                for s, n in op[1].items():
                    if s in live:
                        batch[s] = n
                        t += op[2][at:at + n]
                    at += n
                if batch:
                    op = ("step", batch, t)
                    res = ("ok", target.step(batch, t))
            elif kind == "free" and op[1] in live:
                res = ("ok", target.free(op[1]))
                live.discard(op[1])
        except OutOfBlocks:
            res = ("out_of_blocks", None)
        out.append(res)
        if after_each:
            after_each(i, op, res)
    return out
