"""Block-pool bookkeeping of the paged KV cache, restated plainly -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference arm may import this
module. It shares no code with the product's host block manager and does not import it.

What it follows:
  * 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？, "PagedAttention：核心思路": a sequence takes a
    block when it starts and another one each time its last block is full; any free block will do;
    a finished sequence returns all its blocks.
  * blog.mckayzhao.com/?p=56, "PagedAttention：操作系统课本里翻出来的灵感": N tokens hold
    ceil(N / block_size) blocks.
  * same page, "还不止是分页：Copy-on-Write 和内存共享": sequences forked from one another share
    blocks under a count of holders; one about to write into a shared block copies it first and
    writes the copy, the original staying as it was.
  * 一文搞懂vLLM, "PagedAttention 是怎么共享内存的"; blog.mckayzhao.com/?p=56, "进阶特性：让推理再快一点"
    (Prefix Caching); vLLM 简介, "自动前缀缓存": when the beginning of a new request matches blocks
    computed before, those blocks are reused instead of being computed again.

Steps are taken one token at a time, exactly as described: before token p is stored, a sequence
whose last block is full (p a multiple of the block size) takes a new block; otherwise, if its
last block has more than one holder, it takes a new block, records (old, new) as a copy to make
and drops its hold on the old one. Which free block is taken is not fixed by the pages; this model
takes the lowest free id (the product uses another order, so comparisons map ids one to one).
An operation that runs out of blocks raises OutOfBlocks and changes nothing.

Prefix caching (prefix_cache=True), in its plainest form: a full block of a sequence whose token
ids are known is remembered under the tuple of ALL token ids from the start of the sequence to the
block's end. A new prompt reuses, block by block from its start, the remembered blocks of its own
leading tuples, stopping at the first miss and leaving at least its last token to compute. A
released block stays remembered until it is taken for new data. In this mode blocks are taken in
the order they became free (least recently released first; a new pool in id order, a finishing
sequence releasing its blocks last to first), the eviction order the product documents, since
which blocks survive decides which prompts hit.

`mutant` plants one named mistake (for the pin tests only): "no_cow" writes shared blocks in place,
"early_block" takes a new block one token early, "fork_no_ref" forks without counting the new
holder, "free_shared" frees blocks on release even when other holders remain; for the prefix cache,
"cache_block_only" remembers a block under its own 16 ids instead of the whole prefix,
"keep_on_evict" keeps remembering a block after it is taken for new data, "no_token_cap" lets a
whole prompt hit, "hit_no_hold" reuses a cached block without counting the new holder.
"""
import copy

MUTANTS = ("no_cow", "early_block", "fork_no_ref", "free_shared")
CACHE_MUTANTS = ("cache_block_only", "keep_on_evict", "no_token_cap", "hit_no_hold")


class OutOfBlocks(Exception):
    pass


class BlockPool:
    def __init__(self, num_blocks, block_size=16, mutant=None, prefix_cache=False):
        assert mutant is None or mutant in MUTANTS + CACHE_MUTANTS
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.mutant = mutant
        self.holders = [0] * num_blocks   # how many sequences hold each block
        self.tables = {}                  # sequence id -> list of block ids, in token order
        self.lengths = {}                 # sequence id -> tokens stored
        self.copies = 0
        self.prefix_cache = prefix_cache
        self.free_order = list(range(num_blocks))  # prefix-cache mode: least recently released first
        self.remembered = {}              # tuple of token ids from the start -> block holding its end
        self.token_ids = {}               # sequence id -> its token ids, when known
        self.queries = 0
        self.hits = 0

    # ---- one step at a time ---------------------------------------------------------------
    def _take_free_block(self):
        if self.prefix_cache:
            if not self.free_order:
                raise OutOfBlocks()
            b = self.free_order.pop(0)
            if self.mutant != "keep_on_evict":
                for prefix in [p for p, blk in self.remembered.items() if blk == b]:
                    del self.remembered[prefix]      # its old contents are about to be overwritten
            self.holders[b] = 1
            return b
        for b in range(self.num_blocks):
            if self.holders[b] == 0:
                self.holders[b] = 1
                return b
        raise OutOfBlocks()

    def _release(self, b):
        if self.mutant == "free_shared":
            self.holders[b] = 0
        else:
            self.holders[b] -= 1
        if self.prefix_cache and self.holders[b] == 0:
            self.free_order.append(b)

    def _store_one_token(self, seq, token_id=None):
        """Makes room for the next token of `seq`; returns (old, new) if a copy was needed."""
        table = self.tables[seq]
        p = self.lengths[seq]
        boundary = (p + 1) % self.block_size == 0 if self.mutant == "early_block" else p % self.block_size == 0
        pair = None
        if boundary or not table:
            table.append(self._take_free_block())
        elif self.holders[table[-1]] > 1 and self.mutant != "no_cow":
            old = table[-1]
            new = self._take_free_block()
            self._release(old)
            table[-1] = new
            pair = (old, new)
            self.copies += 1
        self.lengths[seq] = p + 1
        if seq in self.token_ids:
            if token_id is None:
                del self.token_ids[seq]              # ids unknown from here on
            else:
                ids = self.token_ids[seq]
                ids.append(token_id)
                if len(ids) % self.block_size == 0:  # the last block just became full
                    prefix = tuple(ids[-self.block_size:]) if self.mutant == "cache_block_only" else tuple(ids)
                    if prefix not in self.remembered:
                        self.remembered[prefix] = table[-1]
        return pair

    def _atomic(self, fn):
        fields = ("holders", "tables", "lengths", "copies", "free_order", "remembered", "token_ids")
        saved = copy.deepcopy([getattr(self, f) for f in fields])
        try:
            return fn()
        except OutOfBlocks:
            for f, v in zip(fields, saved):
                setattr(self, f, v)
            raise

    # ---- operations -------------------------------------------------------------------------
    def add(self, seq, num_tokens):
        assert seq not in self.tables

        def run():
            self.tables[seq] = []
            self.lengths[seq] = 0
            for _ in range(num_tokens):
                self._store_one_token(seq)

        self._atomic(run)

    def add_cached_prefix(self, seq, tokens):
        """Starts `seq` from the remembered blocks of its prompt's leading tuples; returns how many
        tokens they hold (the caller appends the rest with their ids)."""
        assert seq not in self.tables
        bs = self.block_size
        self.tables[seq] = []
        self.lengths[seq] = 0
        if not self.prefix_cache:
            return 0
        self.token_ids[seq] = []
        limit = len(tokens) // bs if self.mutant == "no_token_cap" else ((len(tokens) - 1) // bs if tokens else 0)
        for i in range(limit):
            self.queries += 1
            prefix = tuple(tokens[bs * i:bs * (i + 1)]) if self.mutant == "cache_block_only" else tuple(tokens[:bs * (i + 1)])
            if prefix not in self.remembered:
                break
            b = self.remembered[prefix]
            if self.mutant != "hit_no_hold":
                if self.holders[b] == 0:
                    self.free_order.remove(b)
                self.holders[b] += 1
            self.tables[seq].append(b)
            self.hits += 1
        self.lengths[seq] = bs * len(self.tables[seq])
        self.token_ids[seq] = list(tokens[:self.lengths[seq]])
        return self.lengths[seq]

    def fork(self, parent, child):
        assert parent in self.tables and child not in self.tables
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        if parent in self.token_ids:
            self.token_ids[child] = list(self.token_ids[parent])
        if self.mutant != "fork_no_ref":
            for b in self.tables[child]:
                self.holders[b] += 1

    def append(self, seq, num_tokens, tokens=None):
        """Returns the list of (old, new) copies the append needs (at most one). `tokens`: the new
        tokens' ids, when known."""
        def run():
            pairs = []
            for t in range(num_tokens):
                pair = self._store_one_token(seq, None if tokens is None else tokens[t])
                if pair:
                    pairs.append(pair)
            return pairs

        return self._atomic(run)

    def free(self, seq):
        for b in reversed(self.tables.pop(seq)):     # last block first
            self._release(b)
        del self.lengths[seq]
        self.token_ids.pop(seq, None)

    def step(self, batch, new_tokens=None):
        """batch: {sequence id: new tokens}, in order; new_tokens: their ids concatenated in batch
        order, or None. Returns (tables, context_lens, query_start_loc, copies) for the batch, each
        table a list of block ids."""
        def run():
            pairs = []
            at = 0
            for seq, n in batch.items():
                pairs += self.append(seq, n, None if new_tokens is None else list(new_tokens[at:at + n]))
                at += n
            return pairs

        pairs = self._atomic(run)
        seqs = list(batch)
        qsl = [0]
        for seq in seqs:
            qsl.append(qsl[-1] + batch[seq])
        return [list(self.tables[s]) for s in seqs], [self.lengths[s] for s in seqs], qsl, pairs

    # ---- accounting ---------------------------------------------------------------------------
    def stats(self):
        bs = self.block_size
        used = [b for b in range(self.num_blocks) if self.holders[b] > 0]
        filled = {}
        for seq, table in self.tables.items():
            for i, b in enumerate(table):
                filled[b] = max(filled.get(b, 0), min(bs, self.lengths[seq] - i * bs))
        stored = sum(filled.values())
        return {
            "num_blocks": self.num_blocks,
            "free_blocks": self.num_blocks - len(used),
            "used_blocks": len(used),
            "shared_blocks": sum(1 for b in used if self.holders[b] > 1),
            "num_sequences": len(self.tables),
            "logical_tokens": sum(self.lengths.values()),
            "stored_tokens": stored,
            "wasted_slots": len(used) * bs - stored,
            "cow_copies": self.copies,
            "cached_blocks": len(self.remembered),
            "cache_queries": self.queries,
            "cache_hits": self.hits,
        }
