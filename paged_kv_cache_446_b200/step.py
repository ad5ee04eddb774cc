"""One attention-layer step of a paged KV cache, as a serving engine runs it on the GPU.

Order (blog.mckayzhao.com/?p=56: "还不止是分页：Copy-on-Write 和内存共享" then "V1 架构：推倒重来的勇气";
一文搞懂vLLM, "快速回顾 prefill、decode 和 KV cache"):
  1. copy_blocks   -- copy-on-write copies of shared blocks that this step writes into;
  2. slot_mapping  -- the physical slot of every token the step appends;
  3. kv_cache_write -- append the step's new K/V rows into those slots;
  4. paged_attention -- every query row of the mixed {request_id: num_tokens} batch attends its
     request's cache through the block table (decode rows and chunked-prefill rows together).
All four run in libpkv.so on one stream; this class only keeps the device-side batch description.
"""
from __future__ import annotations

import numpy as np
import torch

from . import pkv


class PagedAttentionStep:
    def __init__(self, batch: dict, prior_lens, block_tables: np.ndarray, num_blocks: int, num_q_heads: int,
                 num_kv_heads: int, head_dim: int, dtype: torch.dtype, device, write_batch: dict | None = None,
                 copy_pairs: np.ndarray | None = None, stream=None, **plan_opts):
        self.device = torch.device(device)
        self.num_blocks = int(num_blocks)
        self.dtype = dtype
        self.block_tables = torch.from_numpy(np.ascontiguousarray(block_tables, dtype=np.int32)).to(self.device)
        # The host tables let the planner read blocks shared by several requests once.
        if plan_opts.pop("share_prefixes", True):
            plan_opts.setdefault("shared_tables", np.ascontiguousarray(block_tables, dtype=np.int32))
        self.plan = pkv.AttentionPlan(batch, prior_lens, num_q_heads, num_kv_heads, head_dim, dtype, self.device,
                                      stream=stream, **plan_opts)
        # The write batch shares the requests and their context after the step; its rows are the
        # last write_batch[r] positions of each context.
        counts = np.asarray(list(batch.values()), dtype=np.int64)
        ctx_after = np.asarray(prior_lens, dtype=np.int64) + counts
        self.num_write = 0
        if write_batch:
            wcounts = np.asarray([write_batch.get(r, 0) for r in batch.keys()], dtype=np.int64)
            wqsl, wctx = pkv.flatten_batch(dict(zip(batch.keys(), wcounts)), ctx_after - wcounts)
            self.write_qsl = torch.from_numpy(wqsl).to(self.device)
            self.write_ctx = torch.from_numpy(wctx).to(self.device)
            self.num_write = int(wqsl[-1])
            self.slots = torch.empty(self.num_write, dtype=torch.int64, device=self.device)
        self.pairs = None
        if copy_pairs is not None and len(copy_pairs):
            self.pairs = torch.from_numpy(np.ascontiguousarray(copy_pairs, dtype=np.int32).reshape(-1, 2)).to(self.device)

    def run(self, q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor, scale: float,
            k_new: torch.Tensor | None = None, v_new: torch.Tensor | None = None,
            out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        if self.pairs is not None:
            pkv.copy_blocks([k_pool], [v_pool], self.pairs, stream=stream)
        if self.num_write:
            pkv.slot_mapping(self.block_tables, self.write_qsl, self.write_ctx, self.num_blocks, self.num_write,
                             out=self.slots, stream=stream)
            pkv.kv_cache_write(k_new, v_new, k_pool, v_pool, self.slots, stream=stream)
        return pkv.paged_attention(self.plan, q, k_pool, v_pool, self.block_tables, scale, out=out, stream=stream)

    @property
    def kernels_per_run(self) -> int:
        p = self.plan.plan
        n = int(p.num_tiles > 0) + int(p.num_items > 0) + int(p.num_merge_rows > 0)
        if self.pairs is not None:
            n += 1
        if self.num_write:
            n += 2
        return n
