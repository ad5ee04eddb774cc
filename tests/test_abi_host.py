"""Host-side checks of the C ABI (no GPU): exported symbols, argument errors, validators, planner."""
import ctypes
import os
import re

import numpy as np
import pytest

from paged_kv_cache_446_b200 import build as pkv_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkv.h")


@pytest.fixture(scope="module")
def pkv():
    pkv_build.build()
    from paged_kv_cache_446_b200 import pkv as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_function(pkv):
    lib = ctypes.CDLL(pkv.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 12
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, f"declared in pkv.h but not exported: {missing}"


def test_status_strings(pkv):
    for code in range(8):
        assert pkv._lib.pkv_status_string(code)
    assert "sm_100a" in pkv.version()


def test_validators(pkv):
    bt = np.array([[0, 3, 6], [1, 2, -1], [4, -1, -1]], np.int32)       # the block-pool figure
    ctx = np.array([40, 20, 9], np.int32)
    pkv.validate_tables(bt, ctx, 9)
    with pytest.raises(pkv.PkvError):
        pkv.validate_tables(bt, np.array([40, 40, 9], np.int32), 9)    # second table too short
    with pytest.raises(pkv.PkvError):
        pkv.validate_tables(bt, ctx, 6)                                # id 6 outside a 6-block pool
    pkv.validate_slots(np.array([0, 17, -1, 143], np.int64), 9)
    with pytest.raises(pkv.PkvError):
        pkv.validate_slots(np.array([0, 17, 17], np.int64), 9)
    with pytest.raises(pkv.PkvError):
        pkv.validate_slots(np.array([144], np.int64), 9)
    pkv.validate_copy_pairs(np.array([[4, 5], [4, 7], [2, 2]], np.int32), 9)
    with pytest.raises(pkv.PkvError):
        pkv.validate_copy_pairs(np.array([[4, 5], [3, 5]], np.int32), 9)
    with pytest.raises(pkv.PkvError):
        pkv.validate_copy_pairs(np.array([[4, 5], [5, 6]], np.int32), 9)
    with pytest.raises(pkv.PkvError):
        pkv.validate_copy_pairs(np.array([[4, 9]], np.int32), 9)


def test_argument_errors_before_any_launch(pkv):
    lib = pkv._lib
    # block_size other than 16, bad dtype, null pointers: rejected on the host.
    assert lib.pkv_kv_cache_write(1, 1, 1, 1, 1, 4, 8, 2, 64, 8, 1, None) == 2
    assert lib.pkv_kv_cache_write(1, 1, 1, 1, 1, 4, 8, 2, 64, 16, 7, None) == 1
    assert lib.pkv_kv_cache_write(None, 1, 1, 1, 1, 4, 8, 2, 64, 16, 1, None) == 1
    assert lib.pkv_copy_blocks(None, None, 1, 1, 1, 8, 2, 64, 32, 1, None) == 2
    assert lib.pkv_slot_mapping(None, 4, 1, 1, 2, 8, 1, 3, None) == 1
    plan = pkv.Plan()
    assert lib.pkv_paged_attention(1, 1, 1, 1, 1, 4, 1, 1, 8, ctypes.c_float(0.1), ctypes.byref(plan), 1, 1024, None) == 1
    assert "plan" in lib.pkv_last_error().decode()


@pytest.mark.parametrize("bad", ["decreasing", "ctx_short", "heads", "head_dim", "empty_ctx"])
def test_planner_rejects(pkv, bad):
    qsl = np.array([0, 1, 3], np.int32)
    ctx = np.array([5, 9], np.int32)
    Hq, Hkv, D = 8, 2, 128
    if bad == "decreasing":
        qsl = np.array([0, 2, 1], np.int32)
    elif bad == "ctx_short":
        ctx = np.array([5, 1], np.int32)
    elif bad == "heads":
        Hq = 7
    elif bad == "head_dim":
        D = 96
    elif bad == "empty_ctx":
        qsl = np.array([0, 0, 2], np.int32)
        ctx = np.array([0, 0], np.int32)
    with pytest.raises(pkv.PkvError):
        pkv.plan_host(qsl, ctx, Hq, Hkv, D, "f16")


def parse_meta(plan, meta):
    items = np.frombuffer(meta[plan.off_items:plan.off_items + 32 * plan.num_items].tobytes(), np.int32)
    tiles = np.frombuffer(meta[plan.off_tiles:plan.off_tiles + 16 * plan.num_tiles].tobytes(), np.int32)
    merges = np.frombuffer(meta[plan.off_merge:plan.off_merge + 48 * plan.num_merge_rows].tobytes(), np.int32)
    return items.reshape(-1, 8), tiles.reshape(-1, 4), merges.reshape(-1, 12)


def check_plan(pkv, plan, meta, qsl, ctx, Hq, Hkv, opts, dtype, tables=None):
    """Every (row, query head, visible KV block) is covered by exactly one work item or tile, each
    item shows a row exactly the keys the row sees, and every partial result an item writes is read
    by exactly one merge slot, for that same (row, head)."""
    items, tiles, merges = parse_meta(plan, meta)
    R = len(ctx)
    G = Hq // Hkv
    hpi = plan.heads_per_item
    req_of_row = np.repeat(np.arange(R), np.diff(qsl))

    def true_limit(row):
        r = req_of_row[row]
        return r, int(ctx[r] - (qsl[r + 1] - qsl[r]) + (row - qsl[r]) + 1)

    cover, written = {}, {}
    max_rows = 0
    for row0, req, packed, head0, b0, b1, limit, part in items:
        kvh, nrows = packed & 0xFFFF, packed >> 16
        nh = min(hpi, G - head0)
        assert 1 <= nrows and nrows * nh <= plan.part_stride <= 16
        max_rows = max(max_rows, nrows)
        assert 0 <= b0 < b1
        for jr in range(nrows):
            row = row0 + jr
            r, L = true_limit(row)
            for b in range(b0, b1):
                seen_by_kernel = min(max(limit + jr - 16 * b, 0), 16)
                seen_by_row = min(max(L - 16 * b, 0), 16)
                assert seen_by_kernel == seen_by_row, (row, b, limit, jr, L)
                if seen_by_row == 0:
                    continue
                if tables is not None:
                    assert tables[req, b] == tables[r, b], "item reads another request's block"
                elif nrows > 1 or req != r:
                    assert req == r
                for h in range(head0, head0 + nh):
                    key = (row, kvh * G + h, b)
                    cover[key] = cover.get(key, 0) + 1
            if part >= 0:
                for hh in range(nh):
                    written[(part, jr * nh + hh)] = (row, kvh * G + head0 + hh)
    assert plan.rows_per_item == max_rows
    if "rows_per_item" in opts:
        assert max_rows <= opts["rows_per_item"]
    mma_ok = dtype != "f32" and opts.get("decode_kernel") != 1
    tc_min = opts.get("tc_min_rows") or (max(2, 16 // G + 1) if mma_ok else 2)
    tile_rows = 2 * (128 // G)      # two 128-row MMA tiles per CTA
    for req, kvh, tok0, _ in tiles:
        nreq = qsl[req + 1] - qsl[req]
        assert nreq >= tc_min
        for j in range(tok0, min(nreq, tok0 + tile_rows)):
            limit = ctx[req] - nreq + j + 1
            for h in range(G):
                for b in range(-(-limit // 16)):
                    key = (qsl[req] + j, kvh * G + h, b)
                    cover[key] = cover.get(key, 0) + 1
    expect = {}
    for r in range(R):
        nreq = qsl[r + 1] - qsl[r]
        for j in range(nreq):
            limit = ctx[r] - nreq + j + 1
            for h in range(Hq):
                for b in range(-(-limit // 16)):
                    expect[(qsl[r] + j, h, b)] = 1
    assert cover == expect
    read = {}
    for row, qh0, nslots, first, count, hpr, xf, xc, xs, *_ in merges:
        for g in range(nslots):
            target = (row + g // hpr, qh0 + g % hpr)
            srcs = [(first + i, g) for i in range(count)] + ([(xf + i, xs + g) for i in range(xc)] if xf >= 0 else [])
            assert srcs
            for src in srcs:
                assert src not in read
                read[src] = target
    assert read == written
    # the merge grid's stride: the largest merge row
    assert plan.merge_slots == (int(merges[:, 2].max()) if len(merges) else 0)
    if opts.get("no_split") and tables is None:
        assert plan.num_merge_rows == 0


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("opts", [{}, {"split_blocks": 1}, {"split_blocks": 3}, {"no_split": True},
                                  {"cuda_core_only": True}, {"heads_per_item": 4}, {"heads_per_item": 3},
                                  {"cuda_core_only": True, "split_blocks": 2}, {"tc_min_rows": 9},
                                  {"cuda_core_only": True, "rows_per_item": 1},
                                  {"cuda_core_only": True, "rows_per_item": 3, "heads_per_item": 2},
                                  {"decode_kernel": 1}, {"decode_kernel": 2, "tc_min_rows": 9},
                                  {"decode_kernel": 2, "heads_per_item": 16, "split_blocks": 2}])
def test_planner_covers_every_block_once(pkv, seed, opts):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 12))
    n = rng.choice([0, 1, 1, 1, 2, 4, 5, 8, 37, 130], size=R)
    prior = rng.integers(0, 300, size=R)
    ctx = (prior + n).astype(np.int32)
    ctx[(n == 0) & (rng.random(R) < 0.5)] = 0
    qsl = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    Hq, Hkv = [(8, 8), (32, 8), (64, 8), (32, 2), (6, 3)][seed % 5]
    dtype = ["f16", "bf16", "f32"][seed % 3]
    if opts.get("decode_kernel") == 2 and dtype == "f32":
        with pytest.raises(pkv.PkvError):
            pkv.plan_host(qsl, ctx, Hq, Hkv, 128, dtype, **opts)
        return
    plan, meta = pkv.plan_host(qsl, ctx, Hq, Hkv, 128, dtype, **opts)
    if plan.num_items:
        assert plan.decode_kernel in (1, 2) and 1 <= plan.part_stride <= (16 if plan.decode_kernel == 2 else 8)
        if "decode_kernel" in opts:
            assert plan.decode_kernel == opts["decode_kernel"]
    check_plan(pkv, plan, meta, qsl, ctx, Hq, Hkv, opts, dtype)


def shared_prefix_batch(rng, groups, lone):
    """Decode requests in runs that share leading blocks (forks of a prompt), plus lone requests,
    shuffled as whole runs; tables over a pool of distinct ids except for the shared blocks."""
    runs = []
    next_id = 0
    for size, shared in groups:
        ids = list(range(next_id, next_id + shared))
        next_id += shared
        run = []
        for _ in range(size):
            own = int(rng.integers(0, 40))
            run.append((ids, own))
        runs.append(run)
    for _ in range(lone):
        runs.append([([], int(rng.integers(1, 200)))])
    order = rng.permutation(len(runs))
    reqs = [req for i in order for req in runs[i]]
    ctxs, rows = [], []
    for ids, own in reqs:
        c = 16 * len(ids) + own
        c = max(c, 1)
        nb = -(-c // 16)
        row = list(ids) + list(range(next_id, next_id + nb - len(ids)))
        next_id += nb - len(ids)
        ctxs.append(c)
        rows.append(row)
    width = max(len(r) for r in rows)
    tables = np.full((len(rows), width), -1, np.int32)
    for i, row in enumerate(rows):
        tables[i, :len(row)] = row
    return np.array(ctxs, np.int32), tables


@pytest.mark.parametrize("seed", range(5))
@pytest.mark.parametrize("opts", [{}, {"split_blocks": 1}, {"split_blocks": 5}, {"no_split": True},
                                  {"decode_kernel": 1}, {"heads_per_item": 2}, {"min_shared_blocks": 2}])
def test_planner_shared_prefixes(pkv, seed, opts):
    """Runs of decode requests that share leading blocks read them through shared items; coverage,
    visibility, table consistency and merge wiring all hold."""
    rng = np.random.default_rng(100 + seed)
    ctx, tables = shared_prefix_batch(rng, [(8, 5), (3, 12), (2, 1), (5, 4)], lone=4)
    R = len(ctx)
    qsl = np.arange(R + 1, dtype=np.int32)
    Hq, Hkv = [(32, 8), (64, 8), (8, 8), (32, 2), (6, 3)][seed % 5]
    dtype = ["f16", "bf16", "f32"][seed % 3]
    if opts.get("decode_kernel") == 2 and dtype == "f32":
        return
    plan, meta = pkv.plan_host(qsl, ctx, Hq, Hkv, 128, dtype, shared_tables=tables, **opts)
    check_plan(pkv, plan, meta, qsl, ctx, Hq, Hkv, opts, dtype, tables=tables)
    base, _ = pkv.plan_host(qsl, ctx, Hq, Hkv, 128, dtype, **opts)
    items, _, _ = parse_meta(plan, meta)
    if plan.heads_per_item * 2 <= (16 if plan.decode_kernel == 2 else 8):
        assert max(it[2] >> 16 for it in items) > 1          # shared items pack several requests' rows
    assert plan.kv_bytes == base.kv_bytes


def test_workspace_size_matches_plan(pkv):
    from paged_kv_cache_446_b200 import workloads as W
    for c in W.CONFIGS:
        wl = W.make(c, with_tensors=False)
        qsl, ctx = pkv.flatten_batch(wl.batch, wl.prior_lens)
        plan, _ = pkv.plan_host(qsl, ctx, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.dtype, with_meta=False,
                                num_sms=148)
        size = ctypes.c_size_t(0)
        o = pkv._opts(num_sms=148)
        assert pkv._ws_size(pkv._np_ptr(qsl), pkv._np_ptr(ctx), ctx.shape[0], wl.num_q_heads, wl.num_kv_heads,
                            wl.head_dim, pkv.DTYPE_NAME[wl.dtype], ctypes.byref(o), ctypes.byref(size)) == 0
        assert size.value == plan.ws_bytes
        # Algorithmic KV bytes: every (request, KV head, context token) once as K and once as V.
        eb = 4 if wl.dtype == "f32" else 2
        assert plan.kv_bytes == int(ctx.astype(np.int64).sum()) * wl.num_kv_heads * 2 * wl.head_dim * eb


def test_plan_async_refuses_before_any_copy(pkv):
    """pkv_attention_plan_async checks its buffers on the host: without room for the work lists it
    enqueues nothing, reports the sizes it needs and leaves the plan unlaunchable; a half-given
    batch-description pair is an argument error."""
    from paged_kv_cache_446_b200 import workloads as W
    wl = W.make("c3", small=True, with_tensors=False)
    qsl, ctx = pkv.flatten_batch(wl.batch, wl.prior_lens)
    ref, _ = pkv.plan_host(qsl, ctx, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.dtype, with_meta=False,
                           num_sms=148)
    o = pkv._opts(num_sms=148)
    plan = pkv.Plan()
    args = (qsl.ctypes.data, ctx.ctypes.data, ctx.shape[0], wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
            pkv.DTYPE_NAME[wl.dtype], ctypes.byref(o))
    meta = np.zeros(ref.meta_bytes, np.uint8)
    # no device workspace: refused with the sizes filled in
    assert pkv._plan_async(*args, meta.ctypes.data, meta.nbytes, None, 0, None, None, ctypes.byref(plan), None) == 4
    assert plan.magic == 0 and plan.meta_bytes == ref.meta_bytes and plan.ws_bytes == ref.ws_bytes
    # host image one byte short: refused (the device pointer is never touched)
    assert pkv._plan_async(*args, meta.ctypes.data, meta.nbytes - 1, 1 << 20, ref.ws_bytes, None, None,
                           ctypes.byref(plan), None) == 4
    assert plan.magic == 0
    # only one of the batch-description buffers
    desc = np.zeros(2 * ctx.shape[0] + 1, np.int32)
    assert pkv._plan_async(*args, meta.ctypes.data, meta.nbytes, 1 << 20, ref.ws_bytes, desc.ctypes.data, None,
                           ctypes.byref(plan), None) == 1
    assert "h_desc" in pkv._lib.pkv_last_error().decode()


@pytest.mark.parametrize("config", ["c3", "c4", "c5"])
def test_plan_image_independent_of_buffer_contents(pkv, config):
    """The planner writes the work lists in place into the caller's image and zeroes every gap:
    planning into a buffer full of stale bytes gives the same image as planning into zeros."""
    from paged_kv_cache_446_b200 import workloads as W
    wl = W.make(config, small=True, with_tensors=False)
    qsl, ctx = pkv.flatten_batch(wl.batch, wl.prior_lens)
    o = pkv._opts(num_sms=148, shared_tables=np.ascontiguousarray(wl.block_tables, dtype=np.int32))
    plan = pkv.Plan()
    assert pkv._plan_host(qsl.ctypes.data, ctx.ctypes.data, ctx.shape[0], wl.num_q_heads, wl.num_kv_heads,
                          wl.head_dim, pkv.DTYPE_NAME[wl.dtype], ctypes.byref(o), None, 0, ctypes.byref(plan)) == 0
    images = []
    for fill in (0x00, 0xAB):
        meta = np.full(plan.meta_bytes + 512, fill, np.uint8)
        assert pkv._plan_host(qsl.ctypes.data, ctx.ctypes.data, ctx.shape[0], wl.num_q_heads, wl.num_kv_heads,
                              wl.head_dim, pkv.DTYPE_NAME[wl.dtype], ctypes.byref(o), meta.ctypes.data, meta.nbytes,
                              ctypes.byref(plan)) == 0
        assert (meta[plan.meta_bytes:] == fill).all()          # nothing written past the image
        images.append(meta[:plan.meta_bytes].copy())
    assert np.array_equal(images[0], images[1])
    assert plan.num_items > 0


@pytest.mark.parametrize("config,num_sms", [("c2", 148), ("c3", 148), ("c4", 148), ("c6", 148), ("c3", 2),
                                            ("c5", 3), ("c6", 1)])
def test_fma_items_dealt_longest_first_in_a_snake(pkv, config, num_sms):
    """The FMA kernel's persistent warps run positions w, w + W, w + 2W, ... (W = 8 per SM): the
    planner sorts the items longest first and deals every second round of W in reverse, so reading
    the positions back in dealing order gives block counts that never increase, and the warps'
    totals come out within a few percent of each other (or within one item of the mean)."""
    from paged_kv_cache_446_b200 import workloads as W
    wl = W.make(config, with_tensors=False)
    qsl, ctx = pkv.flatten_batch(wl.batch, wl.prior_lens)
    plan, meta = pkv.plan_host(qsl, ctx, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.dtype, num_sms=num_sms,
                               shared_tables=wl.block_tables, decode_kernel=1, tc_min_rows=1 << 20)
    assert plan.decode_kernel == 1
    items, _, _ = parse_meta(plan, meta)
    lens = items[:, 5] - items[:, 4]
    n, deal = len(lens), num_sms * 8
    dealt = []
    for k in range(n):
        r, w = divmod(k, deal)
        in_round = min(deal, n - r * deal)
        dealt.append(lens[k] if r % 2 == 0 else lens[r * deal + in_round - 1 - w])
    assert all(a >= b for a, b in zip(dealt, dealt[1:]))
    per_warp = np.zeros(deal)
    np.add.at(per_warp, np.arange(n) % deal, lens + 1)
    assert per_warp.max() <= max(1.1 * per_warp.mean(), per_warp.mean() + lens.max() + 1) or n <= 3 * deal


@pytest.mark.parametrize("config,num_sms", [("c2", 148), ("c3", 148), ("c4", 148), ("c5", 148), ("c6", 148),
                                            ("c3", 2), ("c6", 1)])
def test_mma_items_longest_first_for_greedy_warps(pkv, config, num_sms):
    """The warp-MMA kernel's warps take items greedily (warp w starts with item w, then each takes
    the next unclaimed item from a ticket counter): the planner lists the items longest first, and a
    greedy simulation of W = 8 warps per SM over that list ends within a few percent of the mean
    load (or within one item of it)."""
    import heapq
    from paged_kv_cache_446_b200 import workloads as W
    wl = W.make(config, with_tensors=False)
    qsl, ctx = pkv.flatten_batch(wl.batch, wl.prior_lens)
    plan, meta = pkv.plan_host(qsl, ctx, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.dtype, num_sms=num_sms,
                               shared_tables=wl.block_tables)
    assert plan.decode_kernel == 2
    items, _, _ = parse_meta(plan, meta)
    lens = (items[:, 5] - items[:, 4]).astype(np.int64)
    assert all(a >= b for a, b in zip(lens, lens[1:]))
    W_ = num_sms * 8
    heap = [(0, w) for w in range(W_)]
    for ln in lens:
        t, w = heapq.heappop(heap)
        heapq.heappush(heap, (t + int(ln) + 1, w))
    finish = max(t for t, _ in heap)
    mean = (lens + 1).sum() / W_
    assert finish <= max(1.1 * mean, mean + lens.max() + 1)


def test_mixed_split_choice(pkv):
    """The split of a mixed batch's SMs between split-K items and tcgen05 tiles: a batch with both
    gets 1 .. S-1 item CTAs from the planner (none when one part is missing), the same batch with
    twice the decode context does not get fewer, and an explicit split is honoured (clamped to
    S - 1; -1 runs the two kernels one after the other)."""
    from paged_kv_cache_446_b200 import workloads as W
    wl = W.make("c5", with_tensors=False)
    prior = np.asarray(wl.prior_lens)
    is_dec = np.array([n == 1 for n in wl.batch.values()])

    def split(prior_lens, num_sms=148, **opts):
        qsl, ctx = pkv.flatten_batch(wl.batch, prior_lens)
        p, _ = pkv.plan_host(qsl, ctx, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.dtype, with_meta=False,
                             num_sms=num_sms, **opts)
        assert p.num_tiles > 0 and p.num_items > 0
        return p.decode_sms

    base = split(prior)
    assert 1 <= base <= 147
    doubled = prior.copy()
    doubled[is_dec] *= 2
    assert split(doubled) >= base
    assert 1 <= split(prior, num_sms=132) <= 131
    assert split(prior, decode_sms=10) == 10
    assert split(prior, decode_sms=500) == 147
    assert split(prior, decode_sms=-1) == 0
    for part, cfg in (("prefill", "c5"), ("all", "c2")):
        w = W.make(cfg, with_tensors=False, part=part) if part != "all" else W.make(cfg, with_tensors=False)
        qsl, ctx = pkv.flatten_batch(w.batch, w.prior_lens)
        p, _ = pkv.plan_host(qsl, ctx, w.num_q_heads, w.num_kv_heads, w.head_dim, w.dtype, with_meta=False,
                             num_sms=148)
        assert p.decode_sms == 0


def test_single_read_flag(pkv):
    """PKV_PLAN_SINGLE_READ (the split-K kernel may let its K/V leave L2 first) is set only when
    every K/V block the items read is read by one item: not with shared-prefix groups, not when a
    KV head's query group spans several items, not when a request's rows do."""
    from paged_kv_cache_446_b200 import workloads as W

    def flags(cfg, **opts):
        wl = W.make(cfg, with_tensors=False)
        qsl, ctx = pkv.flatten_batch(wl.batch, wl.prior_lens)
        p, _ = pkv.plan_host(qsl, ctx, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.dtype, with_meta=False,
                             num_sms=148, shared_tables=wl.block_tables, **opts)
        return p.flags & 1

    assert flags("c2") == 1 and flags("c3") == 1 and flags("c6") == 1
    assert flags("c4") == 0                          # shared-prefix groups
    assert flags("c3", heads_per_item=2) == 0        # G = 4 over two items per KV head
    assert flags("c6", rows_per_item=2) == 0         # 5 verify rows over three items
