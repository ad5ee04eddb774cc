"""Steps driven by the library's host block manager, on the GPU, against the oracle.

A small serving run: prompts are prefilled, forked into samples (parallel sampling / beam
candidates), decoded with one- and multi-token rows, some finish and free their blocks, new
requests reuse them. For every step the manager's pkv_bm_step returns the tables, lengths, batch
offsets and copy-on-write pairs; the GPU runs copy_blocks -> slot_mapping -> kv_cache_write ->
paged_attention on them, the oracle runs its own copy, slot mapping, append and attention on host
copies of the same pools. Outputs must agree within the dtype's tolerance and the pools bit for bit
(blog.mckayzhao.com/?p=56, "还不止是分页：Copy-on-Write 和内存共享"; 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？,
"PagedAttention：核心思路").
"""
import math
from types import SimpleNamespace

import numpy as np
import pytest
import torch

from gpu_harness import TOL, max_err, oracle_step, storage

pytestmark = pytest.mark.gpu


def _rand(shape, dtype, gen):
    return torch.randn(shape, generator=gen, dtype=torch.float32).to(dtype)


def _schedule(rng):
    """(operation, argument) list of a seeded serving run over prompts 0..3."""
    prompts = {p: int(rng.integers(17, 140)) for p in range(4)}
    prompts[3] = 64                                      # a prompt that fills its blocks exactly
    ops = [("add", {p: 0 for p in prompts}), ("step", dict(prompts))]
    samples = {}
    child = 100
    for p in prompts:
        for _ in range(3):
            ops.append(("fork", (p, child)))
            samples[child] = p
            child += 1
    live = list(prompts) + list(samples)
    ops.append(("step", {s: 1 for s in live}))                            # copy-on-write round
    ops.append(("step", {s: int(rng.choice([1, 1, 3, 8])) for s in live}))  # multi-token rows
    gone = [live[i] for i in rng.choice(len(live), size=6, replace=False)]
    ops.append(("free", gone))
    live = [s for s in live if s not in gone]
    ops.append(("add", {200: 0, 201: 0}))
    ops.append(("step", {**{s: 1 for s in live}, 200: 90, 201: 33}))      # mixed: prefill + decode
    live += [200, 201]
    ops.append(("fork", (200, 202)))
    live.append(202)
    for _ in range(3):
        ops.append(("step", {s: int(rng.choice([0, 1, 1, 2])) for s in live}))
    return ops


@pytest.mark.parametrize("dtype_name,Hq,Hkv", [("f16", 32, 8), ("bf16", 64, 8), ("f32", 8, 8)])
def test_manager_driven_serving_run(dtype_name, Hq, Hkv):
    from paged_kv_cache_446_b200 import pkv
    from paged_kv_cache_446_b200 import workloads as W
    from paged_kv_cache_446_b200.step import PagedAttentionStep

    dev = torch.device("cuda:0")
    dtype = W.TORCH_DTYPES[dtype_name]
    D, NB, width = 128, 160, 24
    scale = float(np.float32(1.0 / math.sqrt(D)))
    gen = torch.Generator().manual_seed(5)
    rng = np.random.default_rng(5)
    mgr = pkv.BlockManager(NB)
    k_pool = _rand((NB, Hkv, 16, D), dtype, gen).to(dev)
    v_pool = _rand((NB, Hkv, 16, D), dtype, gen).to(dev)
    h = {"k_pool": storage(k_pool), "v_pool": storage(v_pool)}
    steps = copies = 0
    for kind, arg in _schedule(rng):
        if kind == "add":
            for s, n in arg.items():
                mgr.add(s, n)
            continue
        if kind == "fork":
            mgr.fork(*arg)
            continue
        if kind == "free":
            for s in arg:
                mgr.free(s)
            continue
        batch = arg
        tables, ctx, qsl, pairs = mgr.step(batch, width)
        counts = np.asarray(list(batch.values()), np.int64)
        prior = (ctx - counts).astype(np.int32)
        T = int(qsl[-1])
        q = _rand((T, Hq, D), dtype, gen)
        k_new = _rand((T, Hkv, D), dtype, gen)
        v_new = _rand((T, Hkv, D), dtype, gen)
        # The oracle's run, on host copies taken before the GPU touches anything of this step.
        wl = SimpleNamespace(copy_pairs=pairs, write_batch=dict(batch), batch=batch, prior_lens=prior,
                             block_tables=tables, scale=scale, dtype=dtype_name)
        h.update(q=storage(q), k_new=storage(k_new), v_new=storage(v_new))
        ref = oracle_step(wl, h)
        step = PagedAttentionStep(batch, prior, tables, NB, Hq, Hkv, D, dtype, dev, write_batch=dict(batch),
                                  copy_pairs=pairs)
        out = step.run(q.to(dev), k_pool, v_pool, scale, k_new.to(dev), v_new.to(dev))
        torch.cuda.synchronize()
        assert pkv.device_error() == (0, -1)
        err = max_err(out, ref)
        assert err <= TOL[dtype_name], f"step {steps}: max |err| {err}"
        assert np.array_equal(storage(k_pool), h["k_pool"]) and np.array_equal(storage(v_pool), h["v_pool"])
        steps += 1
        copies += len(pairs)
    st = mgr.stats()
    assert steps == 7 and copies >= 9 and st["cow_copies"] == copies
    assert st["wasted_slots"] < 16 * st["used_blocks"]


@pytest.mark.parametrize("dtype_name,Hq,Hkv", [("f16", 32, 8), ("bf16", 64, 8)])
def test_prefix_cached_serving_run(dtype_name, Hq, Hkv):
    """Requests that share system prompts, with a prefix-caching manager: a new request computes
    only the prompt tokens past its cached blocks (its rows attend the cached blocks written by
    earlier requests), next to decode rows of running requests; finished conversations come back
    with a new message. Each step is compared with the oracle (outputs and whole pools)."""
    from paged_kv_cache_446_b200 import pkv
    from paged_kv_cache_446_b200 import workloads as W
    from paged_kv_cache_446_b200.step import PagedAttentionStep

    dev = torch.device("cuda:0")
    dtype = W.TORCH_DTYPES[dtype_name]
    D, NB, width = 128, 96, 24
    scale = float(np.float32(1.0 / math.sqrt(D)))
    gen = torch.Generator().manual_seed(9)
    rng = np.random.default_rng(9)
    mgr = pkv.BlockManager(NB, prefix_cache=True)
    k_pool = _rand((NB, Hkv, 16, D), dtype, gen).to(dev)
    v_pool = _rand((NB, Hkv, 16, D), dtype, gen).to(dev)
    h = {"k_pool": storage(k_pool), "v_pool": storage(v_pool)}
    systems = [list(range(1000, 1000 + 70)), list(range(2000, 2000 + 33))]
    ids, live, finished = {}, [], []
    cached_total = 0
    for step_no in range(8):
        batch, toks = {}, []
        for s in live:                                   # decode rows of running requests
            t = [int(rng.integers(0, 30000))]
            batch[s] = 1
            toks += t
            ids[s] += t
        for k in range(2):                               # two new requests per step
            s = 100 * step_no + k
            if finished and rng.random() < 0.5:
                prompt = finished.pop(0) + [int(x) for x in rng.integers(0, 30000, size=9)]
            else:
                prompt = systems[int(rng.integers(2))] + [int(x) for x in rng.integers(0, 30000, size=int(rng.integers(1, 20)))]
            cached = mgr.add_cached_prefix(s, prompt)
            cached_total += cached
            batch[s] = len(prompt) - cached
            toks += prompt[cached:]
            ids[s] = list(prompt)
            live.append(s)
        tables, ctx, qsl, pairs = mgr.step(batch, width, toks)
        counts = np.asarray(list(batch.values()), np.int64)
        prior = (ctx - counts).astype(np.int32)
        T = int(qsl[-1])
        q = _rand((T, Hq, D), dtype, gen)
        k_new = _rand((T, Hkv, D), dtype, gen)
        v_new = _rand((T, Hkv, D), dtype, gen)
        wl = SimpleNamespace(copy_pairs=pairs, write_batch=dict(batch), batch=batch, prior_lens=prior,
                             block_tables=tables, scale=scale, dtype=dtype_name)
        h.update(q=storage(q), k_new=storage(k_new), v_new=storage(v_new))
        ref = oracle_step(wl, h)
        step = PagedAttentionStep(batch, prior, tables, NB, Hq, Hkv, D, dtype, dev, write_batch=dict(batch),
                                  copy_pairs=pairs)
        out = step.run(q.to(dev), k_pool, v_pool, scale, k_new.to(dev), v_new.to(dev))
        torch.cuda.synchronize()
        assert pkv.device_error() == (0, -1)
        err = max_err(out, ref)
        assert err <= TOL[dtype_name], f"step {step_no}: max |err| {err}"
        assert np.array_equal(storage(k_pool), h["k_pool"]) and np.array_equal(storage(v_pool), h["v_pool"])
        while len(live) > 4:                             # the oldest requests finish
            s = live.pop(0)
            finished.append(ids.pop(s))
            mgr.free(s)
    assert cached_total > 0 and mgr.stats()["cache_hits"] > 0


@pytest.mark.parametrize("dtype_name,Hq,Hkv", [("f16", 32, 8), ("bf16", 16, 16)])
def test_beam_search_run(dtype_name, Hq, Hkv):
    """Beam search over a paged cache (blog.mckayzhao.com/?p=56, "还不止是分页：Copy-on-Write 和内存
    共享"): each step every beam forks candidates, the best (here: seeded random) keep going and the
    rest are freed, so beams share ever deeper trees of blocks; a candidate writing into a shared
    partial block gets a copy. Each step's decode rows and pools are compared with the oracle."""
    from paged_kv_cache_446_b200 import pkv
    from paged_kv_cache_446_b200 import workloads as W
    from paged_kv_cache_446_b200.step import PagedAttentionStep

    dev = torch.device("cuda:0")
    dtype = W.TORCH_DTYPES[dtype_name]
    D, NB, width, beams, fan = 128, 128, 16, 4, 3
    scale = float(np.float32(1.0 / math.sqrt(D)))
    gen = torch.Generator().manual_seed(13)
    rng = np.random.default_rng(13)
    mgr = pkv.BlockManager(NB)
    k_pool = _rand((NB, Hkv, 16, D), dtype, gen).to(dev)
    v_pool = _rand((NB, Hkv, 16, D), dtype, gen).to(dev)
    h = {"k_pool": storage(k_pool), "v_pool": storage(v_pool)}
    mgr.add(0, 0)
    live, next_id, copies = [0], 1, 0
    first = True
    for step_no in range(12):
        if first:
            batch = {0: 45}                      # the prompt
            first = False
        else:
            cands = []
            for b in live:                       # every beam proposes `fan` continuations
                for _ in range(fan):
                    mgr.fork(b, next_id)
                    cands.append(next_id)
                    next_id += 1
            for b in live:
                mgr.free(b)
            keep = sorted(rng.choice(len(cands), size=min(beams, len(cands)), replace=False).tolist())
            for i, c in enumerate(cands):
                if i not in keep:
                    mgr.free(c)
            live = [cands[i] for i in keep]
            batch = {b: 1 for b in live}
        tables, ctx, qsl, pairs = mgr.step(batch, width)
        counts = np.asarray(list(batch.values()), np.int64)
        prior = (ctx - counts).astype(np.int32)
        T = int(qsl[-1])
        q = _rand((T, Hq, D), dtype, gen)
        k_new = _rand((T, Hkv, D), dtype, gen)
        v_new = _rand((T, Hkv, D), dtype, gen)
        wl = SimpleNamespace(copy_pairs=pairs, write_batch=dict(batch), batch=batch, prior_lens=prior,
                             block_tables=tables, scale=scale, dtype=dtype_name)
        h.update(q=storage(q), k_new=storage(k_new), v_new=storage(v_new))
        ref = oracle_step(wl, h)
        step = PagedAttentionStep(batch, prior, tables, NB, Hq, Hkv, D, dtype, dev, write_batch=dict(batch),
                                  copy_pairs=pairs)
        out = step.run(q.to(dev), k_pool, v_pool, scale, k_new.to(dev), v_new.to(dev))
        torch.cuda.synchronize()
        assert pkv.device_error() == (0, -1)
        err = max_err(out, ref)
        assert err <= TOL[dtype_name], f"step {step_no}: max |err| {err}"
        assert np.array_equal(storage(k_pool), h["k_pool"]) and np.array_equal(storage(v_pool), h["v_pool"])
        copies += len(pairs)
    st = mgr.stats()
    assert copies > 0 and st["shared_blocks"] > 0 and st["num_sequences"] == beams
