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
    merges = np.frombuffer(meta[plan.off_merge:plan.off_merge + 32 * plan.num_merge_rows].tobytes(), np.int32)
    return items.reshape(-1, 8), tiles.reshape(-1, 4), merges.reshape(-1, 8)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("opts", [{}, {"split_blocks": 1}, {"split_blocks": 3}, {"no_split": True},
                                  {"cuda_core_only": True}, {"heads_per_item": 4}, {"heads_per_item": 3},
                                  {"cuda_core_only": True, "split_blocks": 2}, {"tc_min_rows": 9},
                                  {"cuda_core_only": True, "rows_per_item": 1},
                                  {"cuda_core_only": True, "rows_per_item": 3, "heads_per_item": 2},
                                  {"decode_kernel": 1}, {"decode_kernel": 2, "tc_min_rows": 9},
                                  {"decode_kernel": 2, "heads_per_item": 16, "split_blocks": 2}])
def test_planner_covers_every_block_once(pkv, seed, opts):
    """Every (row, query head, visible KV block) is covered by exactly one work item or tile."""
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
    items, tiles, merges = parse_meta(plan, meta)
    G = Hq // Hkv
    hpi = plan.heads_per_item
    cover = {}
    max_rows = 0
    for row, req, packed, head0, b0, b1, limit, part in items:
        kvh, nrows = packed & 0xFFFF, packed >> 16
        assert 1 <= nrows and nrows * min(hpi, G - head0) <= plan.part_stride <= 16
        max_rows = max(max_rows, nrows)
        nreq = qsl[req + 1] - qsl[req]
        assert qsl[req] <= row and row + nrows <= qsl[req + 1]
        j = row - qsl[req]
        assert limit == ctx[req] - nreq + j + 1
        assert 0 <= b0 < b1 <= -(-(limit + nrows - 1) // 16)
        for jr in range(nrows):
            visible = -(-(limit + jr) // 16)
            for h in range(head0, min(G, head0 + hpi)):
                for b in range(b0, min(b1, visible)):
                    key = (row + jr, kvh * G + h, b)
                    cover[key] = cover.get(key, 0) + 1
    assert plan.rows_per_item == max_rows
    if "rows_per_item" in opts:
        assert max_rows <= opts["rows_per_item"]
    tile_rows = 2 * (128 // G)      # two 128-row MMA tiles per CTA
    mma_ok = dtype != "f32" and opts.get("decode_kernel") != 1
    tc_min = opts.get("tc_min_rows") or (max(2, 16 // G + 1) if mma_ok else 2)
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
    # Partials: every partial slot belongs to exactly one merge row, and chunked items point into it.
    owners = {}
    for row, qh0, nslots, first, count, hpr, *_ in merges:
        for p in range(first, first + count):
            assert p not in owners
            owners[p] = (row, qh0, nslots, hpr)
    assert len(owners) == plan.num_partials
    for row, req, packed, head0, b0, b1, limit, part in items:
        kvh, nrows = packed & 0xFFFF, packed >> 16
        if part >= 0:
            nh = min(hpi, G - head0)
            assert owners[part] == (row, kvh * G + head0, nh * nrows, nh)
    if opts.get("no_split"):
        assert plan.num_merge_rows == 0


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
