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

Steps are taken one token at a time, exactly as described: before token p is stored, a sequence
whose last block is full (p a multiple of the block size) takes a new block; otherwise, if its
last block has more than one holder, it takes a new block, records (old, new) as a copy to make
and drops its hold on the old one. Which free block is taken is not fixed by the pages; this model
takes the lowest free id (the product uses another order, so comparisons map ids one to one).
An operation that runs out of blocks raises OutOfBlocks and changes nothing.

`mutant` plants one named mistake (for the pin tests only): "no_cow" writes shared blocks in place,
"early_block" takes a new block one token early, "fork_no_ref" forks without counting the new
holder, "free_shared" frees blocks on release even when other holders remain.
"""
import copy

MUTANTS = ("no_cow", "early_block", "fork_no_ref", "free_shared")


class OutOfBlocks(Exception):
    pass


class BlockPool:
    def __init__(self, num_blocks, block_size=16, mutant=None):
        assert mutant is None or mutant in MUTANTS
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.mutant = mutant
        self.holders = [0] * num_blocks   # how many sequences hold each block
        self.tables = {}                  # sequence id -> list of block ids, in token order
        self.lengths = {}                 # sequence id -> tokens stored
        self.copies = 0

    # ---- one step at a time ---------------------------------------------------------------
    def _take_free_block(self):
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

    def _store_one_token(self, seq):
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
        return pair

    def _atomic(self, fn):
        saved = copy.deepcopy((self.holders, self.tables, self.lengths, self.copies))
        try:
            return fn()
        except OutOfBlocks:
            self.holders, self.tables, self.lengths, self.copies = saved
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

    def fork(self, parent, child):
        assert parent in self.tables and child not in self.tables
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        if self.mutant != "fork_no_ref":
            for b in self.tables[child]:
                self.holders[b] += 1

    def append(self, seq, num_tokens):
        """Returns the list of (old, new) copies the append needs (at most one)."""
        def run():
            pairs = []
            for _ in range(num_tokens):
                pair = self._store_one_token(seq)
                if pair:
                    pairs.append(pair)
            return pairs

        return self._atomic(run)

    def free(self, seq):
        for b in self.tables.pop(seq):
            self._release(b)
        del self.lengths[seq]

    def step(self, batch):
        """batch: {sequence id: new tokens}, in order. Returns (tables, context_lens,
        query_start_loc, copies) for the batch, each table a list of block ids."""
        def run():
            pairs = []
            for seq, n in batch.items():
                pairs += self.append(seq, n)
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
        }
