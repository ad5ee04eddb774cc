"""Shared helpers for the GPU parity tests: run a workload step through the library and through
the oracle on the same seeded inputs. The oracle side never sees a value produced by the CUDA path:
its pools are host copies taken before the GPU step runs, and it applies its own copy-on-write,
slot mapping and KV append.
"""
import numpy as np
import torch

import oracle
from paged_kv_cache_446_b200 import workloads as W

# max |err| bounds: fp16 and bf16 outputs as stated for the method's workloads; fp32 output is
# bounded by fp32 accumulation over at most a few thousand terms of magnitude <= ~5 (1e-4).
TOL = {"f32": 1e-4, "f16": 2e-3, "bf16": 1.6e-2}


def storage(t: torch.Tensor) -> np.ndarray:
    """Host numpy view of a tensor's stored bits (uint16 for 16-bit types)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy().copy()
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def make_step(wl, device, **opts):
    from paged_kv_cache_446_b200.step import PagedAttentionStep
    return PagedAttentionStep(wl.batch, wl.prior_lens, wl.block_tables, wl.num_blocks, wl.num_q_heads,
                              wl.num_kv_heads, wl.head_dim, W.TORCH_DTYPES[wl.dtype], device,
                              write_batch=wl.write_batch or None, copy_pairs=wl.copy_pairs, **opts)


def host_inputs(wl):
    """Host copies of every input of the step (taken before any GPU work touches the pools)."""
    return dict(q=storage(wl.q), k_pool=storage(wl.k_pool), v_pool=storage(wl.v_pool),
                k_new=storage(wl.k_new), v_new=storage(wl.v_new))


def oracle_step(wl, h, rows=None, nthreads=0):
    """The oracle's own run of the step on host copies h (modified in place)."""
    if len(wl.copy_pairs):
        oracle.copy_blocks([h["k_pool"]], [h["v_pool"]], wl.copy_pairs)
    if wl.write_batch:
        counts = np.asarray(list(wl.batch.values()), dtype=np.int64)
        ctx_after = np.asarray(wl.prior_lens, dtype=np.int64) + counts
        wcounts = np.asarray([wl.write_batch.get(r, 0) for r in wl.batch.keys()], dtype=np.int64)
        wqsl, wctx = oracle.flatten_batch(dict(zip(wl.batch.keys(), wcounts)), ctx_after - wcounts)
        slots = oracle.slot_mapping(wl.block_tables, wqsl, wctx)
        oracle.kv_cache_write(h["k_new"], h["v_new"], h["k_pool"], h["v_pool"], slots)
    qsl, ctx = oracle.flatten_batch(wl.batch, wl.prior_lens)
    return oracle.paged_attention(h["q"], h["k_pool"], h["v_pool"], wl.block_tables, ctx, qsl, wl.scale, wl.dtype,
                                  rows=rows, nthreads=nthreads)


def max_err(gpu_out: torch.Tensor, ref: np.ndarray) -> float:
    got = gpu_out.detach().to(torch.float64).cpu().numpy()
    assert got.shape == ref.shape
    if not np.all(np.isfinite(got)):
        return float("inf")
    return float(np.max(np.abs(got - ref))) if ref.size else 0.0
