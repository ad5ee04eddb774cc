"""pkv_paged_attention_static_ws: paged attention for callers that cannot allocate device memory.

Such callers (an engine whose memory manager already holds nearly all of HBM, a plugin inside a
runtime that owns every allocation, code where allocation calls are forbidden) get the planner's
work lists and the split-K partials placed in a library-owned device array instead of a workspace
they would have to allocate. This test calls the entry point through the C ABI, twice in a row, and
checks each result against the workspace-based entry point on the same inputs (the same plan and the
same deterministic kernels, so the two must agree bit for bit) and against the CPU oracle within the
attention tolerance. It also checks that a batch needing more scratch than the array holds is
refused on the host before any launch.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_harness import TOL, max_err, storage

pytestmark = pytest.mark.gpu

_P, _I, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


def _entry():
    from paged_kv_cache_446_b200 import pkv
    lib = ctypes.CDLL(pkv.LIB_PATH)
    f = lib.pkv_paged_attention_static_ws
    f.restype = _I
    f.argtypes = [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _F, _P]
    return pkv, f


def _call(pkv, f, wl, plan_obj, block_tables, out, stream):
    qsl, ctx = plan_obj.h_query_start_loc, plan_obj.h_context_lens
    return f(qsl.ctypes.data_as(_P), ctx.ctypes.data_as(_P), ctx.shape[0], wl.num_q_heads, wl.num_kv_heads,
             wl.head_dim, pkv.DTYPE_NAME[wl.dtype], None, out.data_ptr(), wl.q.data_ptr(), wl.k_pool.data_ptr(),
             wl.v_pool.data_ptr(), block_tables.data_ptr(), block_tables.shape[1],
             plan_obj.context_lens.data_ptr(), plan_obj.query_start_loc.data_ptr(), wl.num_blocks,
             float(wl.scale), stream)


@pytest.mark.parametrize("config,small", [("c3", True), ("c5", True), ("c2", False)])
def test_static_workspace_matches_workspace_entry(config, small):
    pkv, f = _entry()
    from paged_kv_cache_446_b200 import workloads as W
    dev = torch.device("cuda:0")
    wl = W.make(config, device=dev, small=small)
    dt = W.TORCH_DTYPES[wl.dtype]
    bt = torch.from_numpy(wl.block_tables).to(dev)
    plan = pkv.AttentionPlan(wl.batch, wl.prior_lens, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, dt, dev)
    ref = pkv.paged_attention(plan, wl.q, wl.k_pool, wl.v_pool, bt, wl.scale)
    stream = torch.cuda.current_stream().cuda_stream
    # The oracle on host copies of the same inputs (every row of the small cases, sampled rows of
    # the full-size one).
    qsl, ctx = oracle.flatten_batch(wl.batch, wl.prior_lens)
    T = int(qsl[-1])
    rows = None if small else np.random.default_rng(3).choice(T, size=min(T, 8), replace=False).astype(np.int32)
    expect = oracle.paged_attention(storage(wl.q), storage(wl.k_pool), storage(wl.v_pool), wl.block_tables, ctx, qsl,
                                    wl.scale, wl.dtype, rows=rows)
    for _ in range(2):
        out = torch.full_like(wl.q, float("nan"))
        status = _call(pkv, f, wl, plan, bt, out, stream)
        assert status == 0, pkv._lib.pkv_last_error().decode()
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"{wl.name}: differs from the workspace entry point"
        got = out if rows is None else out[torch.as_tensor(rows, device=dev, dtype=torch.long)]
        err = max_err(got, expect)
        assert err <= TOL[wl.dtype], f"{wl.name}: max |err| {err} against the oracle"
    code, detail = pkv.device_error()
    assert code == 0, (code, detail)


def test_static_workspace_refuses_oversized_batch():
    pkv, f = _entry()
    from paged_kv_cache_446_b200 import workloads as W
    dev = torch.device("cuda:0")
    # 64 decode rows over 16k-token contexts cut into one-block chunks: the split-K partials far
    # exceed the static array, so the call must fail on the host with WORKSPACE_TOO_SMALL.
    R, Hq, Hkv, D = 64, 64, 8, 128
    qsl = np.arange(R + 1, dtype=np.int32)
    ctx = np.full(R, 16384, dtype=np.int32)
    opts = pkv._opts(split_blocks=1)
    one = torch.zeros(1, dtype=torch.int32, device=dev)
    status = f(qsl.ctypes.data_as(_P), ctx.ctypes.data_as(_P), R, Hq, Hkv, D, 2, ctypes.byref(opts), one.data_ptr(),
               one.data_ptr(), one.data_ptr(), one.data_ptr(), one.data_ptr(), 1024, one.data_ptr(), one.data_ptr(),
               1, 0.1, torch.cuda.current_stream().cuda_stream)
    assert status == 4
    assert "static workspace" in pkv._lib.pkv_last_error().decode()
    assert W is not None
