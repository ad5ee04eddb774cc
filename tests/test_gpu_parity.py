"""GPU parity: the sm_100a library against the CPU oracle on the same seeded inputs.

Bit-exact for slot mapping, KV append and block copies (whole pools, sentinel-filled so a stray write
shows); within the stated max |err| for attention. Small cases are checked element by element; the
full-size configurations run in the launch configuration the benchmark times and are checked on
sampled rows the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_harness import TOL, host_inputs, make_step, max_err, oracle_step, storage
from paged_kv_cache_446_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_446_b200 import pkv  # noqa: F401  (fails loudly if the library is missing)
    return torch.device("cuda:0")


@pytest.fixture(autouse=True)
def no_device_error(dev):
    from paged_kv_cache_446_b200 import pkv
    pkv.device_error()
    yield
    code, detail = pkv.device_error()
    assert code == 0, f"device error word set: code {code}, detail {detail}"


def run_and_compare(wl, dev, rows=None, **opts):
    h = host_inputs(wl)
    step = make_step(wl, dev, **opts)
    out = step.run(wl.q, wl.k_pool, wl.v_pool, wl.scale, wl.k_new, wl.v_new)
    torch.cuda.synchronize()
    ref = oracle_step(wl, h, rows=rows)
    got = out if rows is None else out[torch.as_tensor(rows, device=out.device, dtype=torch.long)]
    err = max_err(got, ref)
    assert err <= TOL[wl.dtype], f"{wl.name}: max |err| {err:.3g} > {TOL[wl.dtype]}"
    return err, step


@pytest.mark.parametrize("config", W.CONFIGS)
def test_step_small_all_outputs(dev, config):
    wl = W.make(config, device=dev, small=True)
    run_and_compare(wl, dev)


@pytest.mark.parametrize("config", W.CONFIGS)
def test_step_full_size_sampled(dev, config):
    wl = W.make(config, device=dev)
    qsl, ctx = oracle.flatten_batch(wl.batch, wl.prior_lens)
    T = int(qsl[-1])
    rng = np.random.default_rng(7)
    rows = set(rng.choice(T, size=min(T, 24), replace=False).tolist())
    # always include the longest decode row, and every prefill request's first and last row
    dec = [r for r, n in enumerate(wl.batch.values()) if n == 1]
    if dec:
        rows.add(int(qsl[max(dec, key=lambda r: ctx[r])]))
    for r, n in enumerate(wl.batch.values()):
        if n > 1:
            rows.update([int(qsl[r]), int(qsl[r + 1]) - 1])
    run_and_compare(wl, dev, rows=np.asarray(sorted(rows), np.int32))


@pytest.mark.parametrize("opts", [{"no_split": True}, {"split_blocks": 1}, {"split_blocks": 2},
                                  {"split_blocks": 5}, {}])
def test_split_count_independence(dev, opts):
    wl = W.make("c3", device=dev, small=True)
    run_and_compare(wl, dev, **opts)


def test_cuda_core_path_on_prefill_rows(dev):
    """The CUDA-core path serves chunked-prefill rows too (one row at a time, causal limit)."""
    wl = W.make("c5", device=dev, small=True)
    run_and_compare(wl, dev, cuda_core_only=True)


def sentinel_pool(shape, dtype, dev, seed):
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    bits = torch.randint(-32768, 32767, shape, generator=g, device=dev, dtype=torch.int16)
    if dtype == torch.float32:
        bits = torch.randint(-2**31, 2**31 - 1, shape, generator=g, device=dev, dtype=torch.int32)
    return bits.view(dtype)


@pytest.mark.parametrize("config,small", [("c2", True), ("c3", True), ("c5", True), ("c4", True), ("c2", False),
                                          ("c5", False)])
def test_slot_mapping_and_kv_write_bit_exact(dev, config, small):
    from paged_kv_cache_446_b200 import pkv
    wl = W.make(config, device=dev, small=small)
    shape = tuple(wl.k_pool.shape)
    dt = W.TORCH_DTYPES[wl.dtype]
    kp = sentinel_pool(shape, dt, dev, 1)
    vp = sentinel_pool(shape, dt, dev, 2)
    hk, hv = storage(kp), storage(vp)
    step = make_step(wl, dev)
    pkv.slot_mapping(step.block_tables, step.write_qsl, step.write_ctx, wl.num_blocks, step.num_write, out=step.slots)
    pkv.kv_cache_write(wl.k_new, wl.v_new, kp, vp, step.slots)
    torch.cuda.synchronize()
    counts = np.asarray(list(wl.batch.values()), dtype=np.int64)
    ctx_after = np.asarray(wl.prior_lens, dtype=np.int64) + counts
    wcounts = np.asarray([wl.write_batch.get(r, 0) for r in wl.batch.keys()], dtype=np.int64)
    wqsl, wctx = oracle.flatten_batch(dict(zip(wl.batch.keys(), wcounts)), ctx_after - wcounts)
    slots = oracle.slot_mapping(wl.block_tables, wqsl, wctx)
    assert np.array_equal(step.slots.cpu().numpy(), slots)
    oracle.kv_cache_write(storage(wl.k_new), storage(wl.v_new), hk, hv, slots)
    assert np.array_equal(storage(kp), hk)
    assert np.array_equal(storage(vp), hv)


@pytest.mark.parametrize("layers", [1, 3])
def test_copy_blocks_bit_exact(dev, layers):
    from paged_kv_cache_446_b200 import pkv
    wl = W.make("c4", device=dev, small=False, with_tensors=False)
    shape = (wl.num_blocks, wl.num_kv_heads, 16, wl.head_dim)
    kps = [sentinel_pool(shape, torch.float16, dev, 10 + i) for i in range(layers)]
    vps = [sentinel_pool(shape, torch.float16, dev, 20 + i) for i in range(layers)]
    hk = [storage(p) for p in kps]
    hv = [storage(p) for p in vps]
    pairs = torch.from_numpy(wl.copy_pairs).to(dev)
    pkv.validate_copy_pairs(wl.copy_pairs, wl.num_blocks)
    pkv.copy_blocks(kps, vps, pairs)
    torch.cuda.synchronize()
    oracle.copy_blocks(hk, hv, wl.copy_pairs)
    for i in range(layers):
        assert np.array_equal(storage(kps[i]), hk[i])
        assert np.array_equal(storage(vps[i]), hv[i])


def test_block_permutation_bit_identical(dev):
    """Relabelling physical blocks (pool and tables together) leaves every output bit unchanged."""
    wl = W.make("c3", device=dev, small=True)
    wl.write_batch = {}
    step = make_step(wl, dev)
    base = step.run(wl.q, wl.k_pool, wl.v_pool, wl.scale).clone()
    perm = torch.randperm(wl.num_blocks, generator=torch.Generator().manual_seed(3))
    kp = torch.empty_like(wl.k_pool)
    vp = torch.empty_like(wl.v_pool)
    kp[perm.to(dev)] = wl.k_pool
    vp[perm.to(dev)] = wl.v_pool
    bt = wl.block_tables.copy()
    pn = perm.numpy()
    bt[bt >= 0] = pn[bt[bt >= 0]]
    wl.block_tables = bt
    out = make_step(wl, dev).run(wl.q, kp, vp, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, base)


def custom(dev, dtype, Hq, Hkv, D, specs, seed=5):
    """A workload with explicit (prior, num_tokens) rows over a shuffled pool."""
    rng = np.random.default_rng(seed)
    ctx = np.asarray([p + n for p, n in specs], np.int64)
    need = [int(-(-c // 16)) for c in ctx]
    NB = max(1, int(math.ceil(1.2 * sum(need))) + 1)
    perm = rng.permutation(NB).astype(np.int32)
    bt = np.full((len(specs), max(max(need), 1)), -1, np.int32)
    pos = 0
    for r, k in enumerate(need):
        bt[r, :k] = perm[pos:pos + k]
        pos += k
    batch = {r: n for r, (_, n) in enumerate(specs)}
    wl = W.Workload(name="custom", dtype=dtype, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                    scale=float(np.float32(1 / math.sqrt(D))), batch=batch,
                    prior_lens=np.asarray([p for p, _ in specs], np.int32), block_tables=bt, num_blocks=NB,
                    write_batch={}, copy_pairs=np.zeros((0, 2), np.int32), seed=seed)
    W._draw_tensors(wl, dev)
    return wl


@pytest.mark.parametrize("dtype,Hq,Hkv,D,specs", [
    ("f16", 8, 8, 128, [(0, 1)]),                                  # context of one token
    ("bf16", 32, 2, 128, [(31, 1), (16, 1), (200, 1)]),            # group of 16 query heads
    ("f16", 16, 8, 64, [(100, 1), (15, 1), (47, 3)]),              # head_dim 64, 16-bit
    ("f32", 16, 4, 128, [(90, 1), (7, 2)]),                        # fp32, head_dim 128
    ("bf16", 12, 4, 128, [(50, 1), (3, 1)]),                       # group of 3 (padded to 4)
    ("f16", 8, 8, 128, [(0, 0), (20, 1), (0, 0), (63, 1)]),       # requests with no rows this step
    ("bf16", 64, 8, 128, [(16 * 2080 - 1, 1)]),                    # 33280-token context
    ("f16", 8, 2, 128, [(0, 17), (5, 130)]),                       # prefill rows, ragged tiles
])
def test_edge_cases(dev, dtype, Hq, Hkv, D, specs):
    run_and_compare(custom(dev, dtype, Hq, Hkv, D, specs), dev)


def test_empty_batch(dev):
    from paged_kv_cache_446_b200 import pkv
    plan = pkv.AttentionPlan({}, [], 8, 8, 128, torch.float16, dev)
    q = torch.empty(0, 8, 128, dtype=torch.float16, device=dev)
    pool = torch.zeros(1, 8, 16, 128, dtype=torch.float16, device=dev)
    bt = torch.zeros(1, 1, dtype=torch.int32, device=dev)
    out = pkv.paged_attention(plan, q, pool, pool, bt, 0.1)
    assert out.shape == (0, 8, 128)


def test_device_error_on_out_of_range_table_entry(dev):
    """A table entry outside the pool is skipped by the kernel and reported through the error word."""
    from paged_kv_cache_446_b200 import pkv
    wl = custom(dev, "f16", 8, 8, 128, [(40, 1), (10, 1)])
    wl.block_tables[1, 0] = wl.num_blocks + 5
    make_step(wl, dev).run(wl.q, wl.k_pool, wl.v_pool, wl.scale)
    code, detail = pkv.device_error()
    assert code == 6 and detail >= 0


def test_device_lengths_beyond_the_table_are_reported(dev):
    """The prefill tiles take each request's context from the device lengths. When those exceed
    what the host plan (and the table's width) covers, the entries past the table are not read:
    the kernel zero-fills those keys and records a range error."""
    from paged_kv_cache_446_b200 import pkv
    wl = custom(dev, "bf16", 64, 8, 128, [(300, 80)])
    assert wl.block_tables.shape[1] == 24                  # ceil(380 / 16) blocks: the table's width
    plan = pkv.AttentionPlan(wl.batch, wl.prior_lens, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                             W.TORCH_DTYPES[wl.dtype], dev, tc_min_rows=2)
    assert plan.plan.num_tiles > 0
    bt = torch.from_numpy(wl.block_tables).to(dev)
    plan.context_lens.add_(64)                             # 444 tokens: 28 blocks on the device
    out = pkv.paged_attention(plan, wl.q, wl.k_pool, wl.v_pool, bt, wl.scale)
    torch.cuda.synchronize()
    code, detail = pkv.device_error()
    assert code == 6 and detail >= 24, (code, detail)
    assert torch.isfinite(out.float()).all()


PREFILL_CASES = [
    ("bf16", 64, 8, 128, [(0, 512)]),                              # first 512-row chunk, G = 8
    ("bf16", 64, 8, 128, [(300, 80), (0, 1), (17, 33)]),           # mixed rows, ragged tiles
    ("f16", 32, 32, 128, [(0, 200), (129, 130)]),                  # G = 1: 128 rows per tile
    ("bf16", 32, 2, 128, [(5, 40)]),                               # G = 16: 8 rows per tile
    ("f16", 16, 8, 128, [(1000, 3)]),                              # few rows, long prior
    ("bf16", 8, 8, 128, [(0, 2)]),                                 # two rows
    ("f16", 64, 16, 128, [(4096 - 7, 45), (250, 1)]),              # prior not block aligned
]


@pytest.mark.parametrize("dtype,Hq,Hkv,D,specs", PREFILL_CASES)
def test_prefill_tiles_tcgen05(dev, dtype, Hq, Hkv, D, specs):
    wl = custom(dev, dtype, Hq, Hkv, D, specs, seed=11)
    _, step = run_and_compare(wl, dev, tc_min_rows=2)
    assert step.plan.plan.num_tiles > 0, "expected the tcgen05 tile path"


@pytest.mark.parametrize("dtype,Hq,Hkv,D,specs", PREFILL_CASES[:4])
def test_prefill_tiles_match_cuda_core_path(dev, dtype, Hq, Hkv, D, specs):
    """The tcgen05 tiles and the CUDA-core kernel agree on the same prefill rows."""
    wl = custom(dev, dtype, Hq, Hkv, D, specs, seed=12)
    a = make_step(wl, dev, tc_min_rows=2).run(wl.q, wl.k_pool, wl.v_pool, wl.scale).clone()
    b = make_step(wl, dev, cuda_core_only=True).run(wl.q, wl.k_pool, wl.v_pool, wl.scale)
    torch.cuda.synchronize()
    err = (a.double() - b.double()).abs().max().item()
    assert err <= TOL[wl.dtype], err


@pytest.mark.parametrize("hpi", [1, 3, 4, 8])
def test_heads_per_item(dev, hpi):
    """A query group served by several work items (each re-reading the same K/V blocks) gives the
    same result."""
    wl = W.make("c5", device=dev, small=True)
    run_and_compare(wl, dev, heads_per_item=hpi, cuda_core_only=True)


# Speculative verify steps: each request submits k draft tokens plus one as k+1 query rows.
VERIFY_CASES = [
    ("f16", 40, 40, 128, [(700, 5), (33, 5), (1500, 5), (15, 2)]),   # G = 1: 5 rows per item
    ("bf16", 32, 8, 128, [(900, 4), (63, 3), (2000, 8), (5, 1)]),    # G = 4: 2 rows per item
    ("f16", 16, 8, 128, [(31, 4), (32, 4), (47, 8), (400, 6)]),      # G = 2: 4 rows per item
    ("bf16", 64, 8, 128, [(1200, 4), (16, 2)]),                      # G = 8: 1 row per item
    ("f32", 8, 8, 128, [(300, 8), (17, 7), (0, 3)]),                 # fp32 (CUDA cores only)
    ("f16", 16, 16, 64, [(250, 6), (9, 5)]),                         # head_dim 64
]


@pytest.mark.parametrize("opts", [{"tc_min_rows": 9}, {"tc_min_rows": 9, "split_blocks": 1},
                                  {"tc_min_rows": 9, "split_blocks": 3}, {"cuda_core_only": True, "rows_per_item": 1},
                                  {}], ids=["rows", "rows-split1", "rows-split3", "one-row", "default"])
@pytest.mark.parametrize("dtype,Hq,Hkv,D,specs", VERIFY_CASES)
def test_verify_rows(dev, dtype, Hq, Hkv, D, specs, opts):
    """Multi-token rows served by CUDA-core items that pack consecutive rows of a request (each
    with its own causal limit) -- chunked so that some chunks lie wholly past the earlier rows'
    limits -- one row per item, or the default routing, all against the oracle."""
    wl = custom(dev, dtype, Hq, Hkv, D, specs, seed=21)
    _, step = run_and_compare(wl, dev, **opts)
    p = step.plan.plan
    G = Hq // Hkv
    if opts.get("tc_min_rows") and p.num_items:
        cap = p.part_stride
        assert p.rows_per_item == min(max(n for _, n in specs), max(1, cap // min(G, cap)))


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("opts", [{}, {"split_blocks": 1}, {"split_blocks": 5}, {"no_split": True}],
                         ids=["auto-split", "split1", "split5", "nosplit"])
@pytest.mark.parametrize("config", ["c2", "c3", "c4", "c5", "c6"])
def test_decode_kernels(dev, config, opts, kernel):
    """The FMA and warp-MMA kernels for CUDA-core rows, forced, on each 16-bit configuration
    (small), chunked in several ways, against the oracle."""
    wl = W.make(config, device=dev, small=True)
    _, step = run_and_compare(wl, dev, decode_kernel=kernel, tc_min_rows=9, **opts)
    assert step.plan.plan.decode_kernel == kernel


@pytest.mark.parametrize("dtype,Hq,Hkv,D,specs", [
    ("bf16", 64, 8, 128, [(16 * 2080 - 1, 1), (3, 1), (100, 16)]),    # long context; 16 rows
    ("f16", 32, 2, 128, [(31, 1), (16, 1), (200, 2)]),                # group of 16: 16 slots per row
    ("bf16", 96, 4, 128, [(70, 1), (5, 3)]),                          # group of 24: split over items
    ("f16", 8, 8, 128, [(0, 1), (15, 1), (16, 1), (17, 9)]),          # tiny contexts, G = 1
])
def test_mma_kernel_edges(dev, dtype, Hq, Hkv, D, specs):
    wl = custom(dev, dtype, Hq, Hkv, D, specs, seed=23)
    _, step = run_and_compare(wl, dev, decode_kernel=2, tc_min_rows=64)
    assert step.plan.plan.decode_kernel == 2



@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_prefill_reference_raised_mid_tile(dev, dtype):
    """Keys whose scores jump by far more than the rescale threshold inside a 128-key tile (its
    second half) and from tile to tile, so the prefill softmax raises a row's reference after
    part of the tile's P is stored and rescales O repeatedly."""
    wl = custom(dev, dtype, 16, 8, 128, [(700, 40), (130, 9)], seed=31)
    k = wl.k_pool
    for r in range(len(wl.batch)):
        ctx = int(wl.prior_lens[r]) + wl.batch[r]
        for p in range(ctx):
            f = 1.0 + (5.0 if p % 128 >= 64 else 0.0) + 1.5 * (p // 128)
            blk = int(wl.block_tables[r, p // 16])
            k[blk, :, p % 16, :] *= f
    _, step = run_and_compare(wl, dev, tc_min_rows=2)
    assert step.plan.plan.num_tiles > 0


def test_attend_one_call(dev):
    """pkv.attend plans and runs a {request_id: num_tokens} batch in one call (no KV append)."""
    from paged_kv_cache_446_b200 import pkv
    wl = custom(dev, "bf16", 32, 8, 128, [(300, 1), (0, 40), (17, 5), (64, 1)], seed=41)
    h = host_inputs(wl)
    bt = torch.from_numpy(wl.block_tables).to(dev)
    out = pkv.attend(wl.batch, wl.prior_lens, wl.q, wl.k_pool, wl.v_pool, bt, wl.scale)
    torch.cuda.synchronize()
    err = max_err(out, oracle_step(wl, h))
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("opts", [{}, {"split_blocks": 1}, {"no_split": True}, {"share_prefixes": False}],
                         ids=["auto", "split1", "nosplit", "no-sharing"])
@pytest.mark.parametrize("dtype,Hq,Hkv", [("f16", 32, 8), ("bf16", 64, 8), ("bf16", 16, 16)])
def test_shared_prefix_items(dev, dtype, Hq, Hkv, opts, kernel):
    """Runs of decode requests sharing their leading blocks (one item set reads the shared blocks
    for all of them, merged by log-sum-exp with each request's own blocks) against the oracle."""
    from test_abi_host import shared_prefix_batch
    rng = np.random.default_rng(61)
    ctx, tables = shared_prefix_batch(rng, [(8, 5), (3, 12), (2, 1), (5, 4)], lone=4)
    R = len(ctx)
    NB = int(tables.max()) + 1
    wl = W.Workload(name="shared", dtype=dtype, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=128,
                    scale=float(np.float32(1 / math.sqrt(128))), batch={r: 1 for r in range(R)},
                    prior_lens=(ctx - 1).astype(np.int32), block_tables=tables, num_blocks=NB,
                    write_batch={}, copy_pairs=np.zeros((0, 2), np.int32), seed=61)
    W._draw_tensors(wl, dev)
    _, step = run_and_compare(wl, dev, decode_kernel=kernel, **opts)
    slots = 16 if kernel == 2 else 8
    if not opts and slots // min(Hq // Hkv, slots) >= 2:
        assert step.plan.plan.rows_per_item > 1     # shared items pack several requests' rows


@pytest.mark.parametrize("seed", range(12))
def test_random_mixed_batches(dev, seed):
    """Seeded random batches: decode, verify and prefill rows mixed, random group sizes, dtypes,
    chunkings and kernels, requests with no rows, against the oracle."""
    rng = np.random.default_rng(700 + seed)
    dtype = ["f16", "bf16", "f32"][seed % 3]
    Hkv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.choice([1, 2, 3, 4, 8, 16]))
    D = 64 if (dtype == "f32" and seed % 2) else 128
    R = int(rng.integers(1, 10))
    specs = []
    for _ in range(R):
        n = int(rng.choice([0, 1, 1, 1, 2, 5, 16, 70]))
        prior = int(rng.integers(0 if n else 1, 700))
        specs.append((prior, n))
    if all(n == 0 for _, n in specs):
        specs[0] = (specs[0][0], 1)
    opts = {}
    if rng.random() < 0.5:
        opts["split_blocks"] = int(rng.choice([1, 2, 7]))
    if rng.random() < 0.3:
        opts["tc_min_rows"] = int(rng.choice([2, 9, 64]))
    if dtype != "f32" and D == 128 and rng.random() < 0.3:
        opts["decode_kernel"] = int(rng.choice([1, 2]))
    wl = custom(dev, dtype, Hkv * G, Hkv, D, specs, seed=700 + seed)
    run_and_compare(wl, dev, **opts)


def test_pool_too_large_for_tensor_maps_is_refused(dev):
    """A pool whose rows (blocks x KV heads x 16) do not fit a 32-bit tensor-map coordinate is
    refused at launch with a CUDA status, before any kernel runs."""
    import ctypes
    from paged_kv_cache_446_b200 import pkv
    wl = custom(dev, "bf16", 16, 8, 128, [(40, 1), (10, 1)], seed=71)
    step = make_step(wl, dev)
    p = step.plan
    huge_nb = (1 << 31) // (8 * 16) + 1
    status = pkv._attention(pkv._ptr(wl.q), pkv._ptr(wl.q), pkv._ptr(wl.k_pool), pkv._ptr(wl.v_pool),
                            pkv._ptr(step.block_tables), step.block_tables.shape[1], pkv._ptr(p.context_lens),
                            pkv._ptr(p.query_start_loc), huge_nb, ctypes.c_float(wl.scale), ctypes.byref(p.plan),
                            pkv._ptr(p.workspace), p.workspace.numel(), pkv._stream(None))
    torch.cuda.synchronize()
    assert status == 3


@pytest.mark.parametrize("decode_sms", [1, 16, 74, 147])
def test_overlapped_mixed_batch(dev, decode_sms):
    """A mixed batch served by one persistent launch: decode_sms CTAs of the tcgen05 kernel start on
    the split-K items, the rest on the tiles, each turning to the other queue when its own empties.
    Within tolerance of the oracle, and bit for bit the output of the two kernels run one after the
    other (every output element is computed by the same item or tile either way)."""
    wl = W.make("c5", device=dev, small=True)
    _, step = run_and_compare(wl, dev, decode_sms=decode_sms)
    p = step.plan.plan
    assert p.num_tiles > 0 and p.num_items > 0 and p.decode_sms == decode_sms
    a = step.run(wl.q, wl.k_pool, wl.v_pool, wl.scale, wl.k_new, wl.v_new).clone()
    b = make_step(wl, dev, decode_sms=-1).run(wl.q, wl.k_pool, wl.v_pool, wl.scale, wl.k_new, wl.v_new)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype,Hq,Hkv,specs,rows_per_item,slots", [
    # 16 query heads per KV head: 16-slot items, served by warps 0-7 inside the register split
    ("bf16", 32, 2, [(300, 70), (0, 130)] + [(400 + 97 * i, 1) for i in range(6)], 0, 16),
    # verify rows of 2 tokens at G = 4: 8-slot items of two rows, served by all twelve warps
    ("f16", 16, 4, [(250, 64), (33, 48)] + [(300 + 211 * i, 2) for i in range(5)], 2, 8),
])
@pytest.mark.parametrize("decode_sms", [3, 37])
def test_overlapped_mixed_batch_item_forms(dev, dtype, Hq, Hkv, specs, rows_per_item, slots, decode_sms):
    """One persistent launch over tiles and split-K items in both item forms the launch can take,
    with short split chunks so every CTA sees many items: within tolerance of the oracle and bit
    for bit the two kernels run one after the other."""
    wl = custom(dev, dtype, Hq, Hkv, 128, specs, seed=41 + decode_sms)
    opts = dict(decode_sms=decode_sms, split_blocks=3, rows_per_item=rows_per_item)
    _, step = run_and_compare(wl, dev, **opts)
    p = step.plan.plan
    assert p.num_tiles > 0 and p.num_items > 0 and p.decode_sms == decode_sms and p.decode_kernel == 2
    assert max(1, p.rows_per_item) * min(p.heads_per_item, Hq // Hkv) == slots
    a = step.run(wl.q, wl.k_pool, wl.v_pool, wl.scale).clone()
    b = make_step(wl, dev, **dict(opts, decode_sms=-1)).run(wl.q, wl.k_pool, wl.v_pool, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("config", ["c2", "c4", "c5"])
def test_plan_reused_across_launches(dev, config):
    """One plan run many times in a row (as every layer of a model step does): the split-K kernel's
    item ticket counter resets itself at the end of each launch, so every launch serves every item
    and the outputs agree bit for bit."""
    from paged_kv_cache_446_b200 import pkv
    wl = W.make(config, device=dev, small=True)
    bt = torch.from_numpy(wl.block_tables).to(dev)
    plan = pkv.AttentionPlan(wl.batch, wl.prior_lens, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                             W.TORCH_DTYPES[wl.dtype], dev, decode_sms=8)
    outs = []
    for _ in range(4):
        out = torch.full_like(wl.q, float("nan"))
        pkv.paged_attention(plan, wl.q, wl.k_pool, wl.v_pool, bt, wl.scale, out=out)
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.isfinite(outs[0].float()).all()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
