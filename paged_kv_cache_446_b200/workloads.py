"""Seeded synthetic workloads for the measured configurations.

This module only draws inputs: request lengths, block-table contents (physical block ids taken from
a seeded permutation of the pool), copy-on-write pairs and the random q/k/v values. It performs none
of the attention, slot or block arithmetic that the library and the oracle compute; both consume
exactly what is generated here. Lengths and tables come from numpy.random.default_rng(seed); tensor
contents come from a torch.Generator seeded with the same seed on the device the tensors live on
(so full-size pools can be drawn directly in HBM).

Configurations (the pages' workloads are described only in prose; the shapes follow the model
families the pages mention -- LLaMA-13B in blog.mckayzhao.com/?p=56 "故事要从 KV Cache 说起"):
  c1  tiny fp32: 4 decode rows, context {1,17,33,100}, 8/8 heads, head_dim 64, 64-block pool
  c2  LLaMA-13B-shaped fp16 decode: 64 rows, 40/40 heads, context U[128,2048], pool 1.2x need,
      one new token per row appended before attention
  c3  LLaMA-3-8B-shaped bf16 GQA decode: 256 rows, 32/8 heads, context lognormal(median 1000,
      sigma 1.0) clipped to [16,8192], one new token appended per row
  c4  parallel sampling fp16: 16 prompts x 8 samples, prompt 1024+U[1,15] tokens whose 64 full
      blocks are shared by the 8 samples; the partial 65th block is copied once per sample
      (copy-on-write), then each sample appends a tail of U[0,512] tokens and decodes one row
  c5  70B-shaped bf16 mixed batch: 4 chunked-prefill requests of 512 rows at prior context
      {0,4096,16384,32768} followed by 128 decode rows with context U[256,16384]; every scheduled
      token is appended before attention
  c6  speculative verify, LLaMA-13B-shaped fp16: 32 requests each submitting k = 4 draft tokens plus
      one as k+1 = 5 query rows ({request_id: 5}, 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？,
      "V1 架构：推倒重来的勇气"), prior context U[512,4096]; the 5 new K/V rows are appended first

`small=True` keeps each configuration's dtype, heads, head_dim and row mix but shrinks the number of
requests and the lengths so the CPU oracle checks every output in seconds.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK_SIZE = 16
TORCH_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
CONFIGS = ("c1", "c2", "c3", "c4", "c5", "c6")


@dataclass
class Workload:
    name: str
    dtype: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    scale: float
    # The step's batch, {request_id: num_tokens} in insertion order, and each request's context
    # before this step's tokens.
    batch: dict
    prior_lens: np.ndarray             # int32 [R]
    block_tables: np.ndarray           # int32 [R, max_blocks], -1 padded
    num_blocks: int
    # Tokens appended through kv_cache_write this step, as their own {request_id: num_tokens}
    # batch over the same requests (empty when the pool is pre-filled for the whole context).
    write_batch: dict
    copy_pairs: np.ndarray             # int32 [P, 2] (src, dst); may be empty
    q: torch.Tensor = None             # [T, Hq, D]
    k_pool: torch.Tensor = None        # [NB, Hkv, 16, D]
    v_pool: torch.Tensor = None
    k_new: torch.Tensor = None         # [T_write, Hkv, D]
    v_new: torch.Tensor = None
    seed: int = 0
    notes: dict = field(default_factory=dict)

    @property
    def num_reqs(self) -> int:
        return len(self.batch)

    @property
    def num_q_tokens(self) -> int:
        return int(sum(self.batch.values()))

    @property
    def num_write_tokens(self) -> int:
        return int(sum(self.write_batch.values()))

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


def _nblocks(n: np.ndarray | int):
    # Table width needed to hold n tokens (sizing of the generated tables only).
    return -(-np.asarray(n) // BLOCK_SIZE)


def _fill_normal(shape, dtype: str, gen: torch.Generator, device) -> torch.Tensor:
    """N(0,1) values drawn in float32 and rounded to `dtype`, generated in slabs to bound memory."""
    out = torch.empty(shape, dtype=TORCH_DTYPES[dtype], device=device)
    flat = out.view(-1)
    step = 1 << 26
    for s in range(0, flat.numel(), step):
        e = min(flat.numel(), s + step)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32).to(out.dtype)
    return out


def _tables_from_permutation(rng, lens_blocks: list[int], num_blocks: int) -> np.ndarray:
    perm = rng.permutation(num_blocks).astype(np.int32)
    width = max(1, max(lens_blocks) if lens_blocks else 1)
    bt = np.full((len(lens_blocks), width), -1, dtype=np.int32)
    pos = 0
    for r, nb in enumerate(lens_blocks):
        bt[r, :nb] = perm[pos:pos + nb]
        pos += nb
    return bt


def make(config: str, device: str | torch.device = "cpu", small: bool = False, seed: int | None = None,
         with_tensors: bool = True, part: str = "all", max_requests: int = 0) -> Workload:
    """Build configuration `config` ("c1".."c6"); seed defaults to 1000 + the configuration number.

    part="prefill" / "decode" keeps only the requests with more than one / exactly one row this
    step (their tables are relabelled onto a pool sized 1.2x their blocks, keeping the seeded
    placement order), so each half of a mixed batch can be timed on its own. max_requests > 0 then
    keeps only the first that many requests (a smaller case of the same structure, for profiling).
    """
    if config not in CONFIGS:
        raise ValueError(f"unknown configuration {config!r}")
    seed = 1000 + int(config[1]) if seed is None else int(seed)
    rng = np.random.default_rng(seed)
    builder = {"c1": _c1, "c2": _c2, "c3": _c3, "c4": _c4, "c5": _c5, "c6": _c6}[config]
    wl = builder(rng, small)
    wl.seed = seed
    if part != "all" or max_requests > 0:
        _keep_part(wl, part, max_requests)
    if with_tensors:
        _draw_tensors(wl, device)
    return wl


def _keep_part(wl: Workload, part: str, max_requests: int = 0) -> None:
    if part not in ("all", "prefill", "decode"):
        raise ValueError(f"unknown part {part!r}")
    if len(wl.copy_pairs):
        raise ValueError("parts are defined for workloads without copy-on-write pairs")
    keys = list(wl.batch.keys())
    keep = [i for i, r in enumerate(keys) if part == "all" or (wl.batch[r] > 1) == (part == "prefill")]
    if max_requests > 0:
        keep = keep[:max_requests]
    if not keep:
        raise ValueError(f"{wl.name} has no {part} rows")
    bt = wl.block_tables[keep]
    used = np.unique(bt[bt >= 0])
    order = np.argsort(np.argsort(used))            # rank of each used id: keeps the placement order
    remap = np.full(wl.num_blocks, -1, dtype=np.int64)
    remap[used] = order
    nb = int(math.ceil(1.2 * len(used)))
    wl.block_tables = np.where(bt >= 0, remap[np.maximum(bt, 0)], -1).astype(np.int32)
    wl.num_blocks = max(nb, 1)
    wl.prior_lens = np.asarray(wl.prior_lens)[keep].astype(np.int32)
    wl.batch = {keys[i]: wl.batch[keys[i]] for i in keep}
    wl.write_batch = {r: n for r, n in wl.write_batch.items() if r in wl.batch}
    wl.name = wl.name + ("" if part == "all" else f"-{part}") + (f"-first{max_requests}" if max_requests > 0 else "")


def _draw_tensors(wl: Workload, device) -> None:
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed)
    Hq, Hkv, D = wl.num_q_heads, wl.num_kv_heads, wl.head_dim
    pool_shape = (wl.num_blocks, Hkv, BLOCK_SIZE, D)
    wl.k_pool = _fill_normal(pool_shape, wl.dtype, gen, device)
    wl.v_pool = _fill_normal(pool_shape, wl.dtype, gen, device)
    wl.q = _fill_normal((wl.num_q_tokens, Hq, D), wl.dtype, gen, device)
    wl.k_new = _fill_normal((wl.num_write_tokens, Hkv, D), wl.dtype, gen, device)
    wl.v_new = _fill_normal((wl.num_write_tokens, Hkv, D), wl.dtype, gen, device)


def _decode_only(name, dtype, Hq, Hkv, D, ctx, rng, pool_factor=1.2, fixed_pool=None, write=True) -> Workload:
    ctx = np.asarray(ctx, dtype=np.int64)
    need = [int(x) for x in _nblocks(ctx)]
    num_blocks = fixed_pool if fixed_pool is not None else int(math.ceil(pool_factor * sum(need)))
    bt = _tables_from_permutation(rng, need, num_blocks)
    R = len(ctx)
    batch = {r: 1 for r in range(R)}
    return Workload(name=name, dtype=dtype, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                    scale=float(np.float32(1.0 / math.sqrt(D))), batch=batch,
                    prior_lens=(ctx - 1).astype(np.int32), block_tables=bt, num_blocks=num_blocks,
                    write_batch=dict(batch) if write else {}, copy_pairs=np.zeros((0, 2), np.int32))


def _c1(rng, small):
    # Tiny fp32 reference: fixed lengths, 64-block pool, tables a seeded permutation; pre-filled pool.
    return _decode_only("c1", "f32", 8, 8, 64, [1, 17, 33, 100], rng, fixed_pool=64, write=False)


def _c2(rng, small):
    R, lo, hi = (8, 17, 700) if small else (64, 128, 2048)
    ctx = rng.integers(lo, hi + 1, size=R)
    return _decode_only("c2" + ("-small" if small else ""), "f16", 40, 40, 128, ctx, rng)


def _c3(rng, small):
    R, cap = (24, 900) if small else (256, 8192)
    sigma = 1.0
    ctx = np.clip(np.rint(rng.lognormal(mean=math.log(1000.0), sigma=sigma, size=R)), 16, cap).astype(np.int64)
    wl = _decode_only("c3" + ("-small" if small else ""), "bf16", 32, 8, 128, ctx, rng)
    wl.notes["lognormal_sigma"] = sigma
    return wl


def _c4(rng, small):
    prompts, samples, tail_hi, base = (3, 4, 60, 64) if small else (16, 8, 512, 1024)
    Hq, Hkv, D = 32, 8, 128
    prompt_len = base + rng.integers(1, 16, size=prompts)          # never a whole number of blocks
    tails = rng.integers(0, tail_hi + 1, size=(prompts, samples))
    full = base // BLOCK_SIZE                                        # shared full prompt blocks
    # Blocks each sample needs beyond the shared ones: its copy of the partial block plus the
    # blocks its tail spills into.
    ctx = (prompt_len[:, None] + tails).astype(np.int64)
    extra = _nblocks(ctx) - full                                    # >= 1 (the copied block)
    need = prompts * (full + 1) + int(extra.sum())
    num_blocks = int(math.ceil(1.2 * need))
    perm = rng.permutation(num_blocks).astype(np.int32)
    pos = 0

    def take(k):
        nonlocal pos
        ids = perm[pos:pos + k]
        pos += k
        return ids

    width = int(_nblocks(ctx).max())
    bt = np.full((prompts * samples, width), -1, dtype=np.int32)
    pairs = []
    for p in range(prompts):
        shared = take(full)
        partial = take(1)[0]
        for s in range(samples):
            r = p * samples + s
            own = take(int(extra[p, s]))                            # own[0] receives the copy
            bt[r, :full] = shared
            bt[r, full:full + len(own)] = own
            pairs.append((int(partial), int(own[0])))
    R = prompts * samples
    batch = {r: 1 for r in range(R)}
    flat_tails = tails.reshape(-1)
    # Attention: one decode row per sample at the end of its context; the tail tokens are appended
    # first by their own write batch (a sample with an empty tail appends nothing).
    ctx_flat = ctx.reshape(-1)
    wl = Workload(name="c4" + ("-small" if small else ""), dtype="f16", num_q_heads=Hq, num_kv_heads=Hkv,
                  head_dim=D, scale=float(np.float32(1.0 / math.sqrt(D))), batch=batch,
                  prior_lens=(ctx_flat - 1).astype(np.int32), block_tables=bt, num_blocks=num_blocks,
                  write_batch={r: int(flat_tails[r]) for r in range(R)},
                  copy_pairs=np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    wl.notes.update(prompt_len=prompt_len.tolist(), shared_blocks_per_prompt=full, samples=samples)
    return wl


def _c5(rng, small):
    Hq, Hkv, D = 64, 8, 128
    if small:
        priors, chunk, n_dec, lo, hi = [0, 300], 80, 6, 20, 700
    else:
        priors, chunk, n_dec, lo, hi = [0, 4096, 16384, 32768], 512, 128, 256, 16384
    dec_ctx = rng.integers(lo, hi + 1, size=n_dec).astype(np.int64)
    pre_ctx = np.asarray(priors, dtype=np.int64) + chunk
    ctx = np.concatenate([pre_ctx, dec_ctx])
    need = [int(x) for x in _nblocks(ctx)]
    num_blocks = int(math.ceil(1.2 * sum(need)))
    bt = _tables_from_permutation(rng, need, num_blocks)
    R = len(ctx)
    batch = {r: (chunk if r < len(priors) else 1) for r in range(R)}
    n = np.asarray([batch[r] for r in range(R)], dtype=np.int64)
    wl = Workload(name="c5" + ("-small" if small else ""), dtype="bf16", num_q_heads=Hq, num_kv_heads=Hkv,
                  head_dim=D, scale=float(np.float32(1.0 / math.sqrt(D))), batch=batch,
                  prior_lens=(ctx - n).astype(np.int32), block_tables=bt, num_blocks=num_blocks,
                  write_batch=dict(batch), copy_pairs=np.zeros((0, 2), np.int32))
    wl.notes.update(prefill_priors=priors, chunk=chunk)
    return wl


def _c6(rng, small):
    R, lo, hi, rows = (6, 17, 300, 5) if small else (32, 512, 4096, 5)
    prior = rng.integers(lo, hi + 1, size=R).astype(np.int64)
    ctx = prior + rows
    need = [int(x) for x in _nblocks(ctx)]
    num_blocks = int(math.ceil(1.2 * sum(need)))
    bt = _tables_from_permutation(rng, need, num_blocks)
    batch = {r: rows for r in range(R)}
    wl = Workload(name="c6" + ("-small" if small else ""), dtype="f16", num_q_heads=40, num_kv_heads=40,
                  head_dim=128, scale=float(np.float32(1.0 / math.sqrt(128))), batch=batch,
                  prior_lens=prior.astype(np.int32), block_tables=bt, num_blocks=num_blocks,
                  write_batch=dict(batch), copy_pairs=np.zeros((0, 2), np.int32))
    wl.notes.update(draft_tokens=rows - 1)
    return wl
