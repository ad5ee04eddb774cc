// C ABI entry points (include/pkv.h): argument checks, the host planner and kernel launches.
#include <algorithm>
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <cuda.h>

#include "internal.h"
#include "pkv.h"

namespace pkv {

__device__ DeviceError g_device_error;

namespace {

thread_local std::string t_last_error;

pkv_status fail(pkv_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
pkv_status fail(pkv_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return s;
}

pkv_status cuda_fail(cudaError_t e, const char* what) {
    return fail(PKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int elem_bytes(pkv_dtype dt) { return dt == PKV_F32 ? 4 : 2; }
bool dtype_ok(int dt) { return dt == PKV_F32 || dt == PKV_F16 || dt == PKV_BF16; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t align256(int64_t x) { return (x + 255) / 256 * 256; }

int current_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

// Work lists of one batch, before they are written into the metadata image. One instance per host
// thread is reused across calls so the vectors keep their capacity (fresh large allocations would
// be served from newly mapped pages and fault on every call).
struct PlanLists {
    std::vector<DecodeItem> items;
    std::vector<PrefillTile> tiles;
    std::vector<MergeRow> merges;
    std::vector<size_t> start;
    std::vector<int> req_keys;
    std::vector<int> shared_first;
    struct Cursor { uint32_t round, index; };
    std::vector<Cursor> cursor;
    int num_partials = 0;
    size_t num_items = 0, num_merges = 0;
    // Set when the planner wrote the whole image straight into the caller's buffer.
    const unsigned char* direct = nullptr;
    void reset() {
        items.clear();
        tiles.clear();
        merges.clear();
        start.clear();
        req_keys.clear();
        num_partials = 0;
        num_items = num_merges = 0;
        direct = nullptr;
    }
};

PlanLists& thread_lists() {
    static thread_local PlanLists lists;
    lists.reset();
    return lists;
}

// Query rows per tcgen05 CTA: two 128-row MMA tiles, each (128 / G) consecutive query rows x G heads.
int tile_tokens(int group) { return 2 * (128 / group); }

// When the last tile ends if the tiles (longest first, as the ticket counter hands them out) each
// go to the CTA that frees first: `ctas` CTAs, `late` of which free only at t_late. Durations and
// loads are whole ticks. Tiles of equal length form runs (ticks, count) and CTAs of equal load form
// groups (load, count), kept in `load` sorted by decreasing load (the least loaded group last), so
// a run is dealt to whole groups at once and the cost grows with the distinct lengths and loads,
// not with the tiles.
int64_t greedy_end(const std::vector<std::pair<int64_t, int>>& runs, int ctas, int late, int64_t t_late,
                   std::vector<std::pair<int64_t, int>>& load) {
    load.clear();
    if (late > 0) load.push_back({t_late, late});
    if (ctas > late) load.push_back({0, ctas - late});
    int64_t end = late > 0 ? t_late : 0;
    const auto add = [&](int64_t l, int k) {  // k CTAs at load l, merged into an equal group if any
        auto it = std::lower_bound(load.begin(), load.end(), l,
                                   [](const std::pair<int64_t, int>& g, int64_t v) { return g.first > v; });
        if (it != load.end() && it->first == l) it->second += k;
        else load.insert(it, {l, k});
    };
    for (const auto& run : runs) {
        for (int n = run.second; n > 0;) {
            std::pair<int64_t, int>& g = load.back();
            const int64_t l = g.first;
            const int k = std::min(g.second, n);
            n -= k;
            if ((g.second -= k) == 0) load.pop_back();
            add(l + run.first, k);
            end = std::max(end, l + run.first);
        }
    }
    return end;
}

// CTAs of the tile kernel that should start on the split-K items of a mixed batch (0: run the two
// kernels one after the other). Model, with rates measured on B200 for these kernels: a tile CTA
// spends ~1.95 us per 128-key tile while items stream beside it; an SM serving items streams their
// K/V at ~115 GB/s while the others run tiles (items of at most 8 (row, head) slots, on all twelve
// warps; ~85 GB/s for items of up to 16 slots, on eight); the items alone stream at ~6.6 TB/s on
// the whole GPU.
// With nd SMs on items, the tiles are dealt greedily to the other S - nd CTAs (greedy_end: long
// tiles come in few sizes, so the step's length moves in steps as nd changes, not smoothly). If the
// nd SMs have not streamed every item when the tiles end, the rest runs on the whole GPU and the
// step ends about half an item later than the bytes alone say (each of the S x 12 (or 8) item
// warps finishes its last item at its own time). If they have, they turn to the tiles still unclaimed, which the
// greedy schedule models as nd CTAs freeing late. Candidates near the balanced share (both queues
// ending together) are simulated. Past the share the estimate is flat (the items end first and
// the tiles set the step) and just below it the step grows fast, so the pick is the middle of the
// run of candidates within 0.3 % of the best, not its low end. The step length moves in steps:
// on the 70B-shaped mixed batch with eight item warps per SM, 52 item SMs measured 1.209 ms and 53
// measured 1.247 ms (128 tiles of ~500 us and 128 of ~250 us pack evenly onto 96 tile CTAs, not
// onto 95); with twelve, 44-52 measured within 0.4 % of each other and 40 2 % slower.
int mixed_split(const std::vector<PrefillTile>& tiles, int64_t item_bytes, int64_t num_items, int item_slots,
                int num_sms) {
    constexpr double kKeyTileSec = 1.95e-6, kGpuBytesPerSec = 6.6e12;
    const double kSmBytesPerSec = item_slots <= 8 ? 115e9 : 85e9;
    const double warps_per_sm = item_slots <= 8 ? 12.0 : 8.0;
    if (tiles.empty() || num_items <= 0) return 0;
    static thread_local std::vector<std::pair<int64_t, int>> runs;
    static thread_local std::vector<std::pair<int64_t, int>> load;
    // Ticks of 1/96 of the longest tile: coarse enough that equal loads recur (the simulation then
    // takes ~85 us of host time on that batch), fine enough that a CTA's few tiles add up to within
    // ~1 % (at 1/64 the choice there moved to 50).
    int max_kt = 1;
    for (const PrefillTile& t : tiles) max_kt = std::max(max_kt, t.key_tiles);
    const double tick = max_kt * kKeyTileSec / 96.0;
    runs.clear();
    double tile_work = 0.0;
    for (const PrefillTile& t : tiles) {
        const int64_t d = std::max<int64_t>(1, std::llround(t.key_tiles * kKeyTileSec / tick));
        tile_work += d * tick;
        if (!runs.empty() && runs.back().first == d) ++runs.back().second;
        else runs.push_back({d, 1});
    }
    const double items = (double)item_bytes;
    const double item_work = items / kSmBytesPerSec;  // SM-seconds on item-first SMs
    const double tail = 0.5 * (items / num_items) * (num_sms * warps_per_sm) / kGpuBytesPerSec;
    const double serial = greedy_end(runs, num_sms, 0, 0, load) * tick + items / kGpuBytesPerSec;
    const int bal = (int)std::lround(num_sms * item_work / std::max(tile_work + item_work, 1e-30));
    const int lo = std::max(1, bal - 12), hi = std::min(num_sms - 1, bal + 12);
    static thread_local std::vector<double> est;
    est.assign((size_t)std::max(hi - lo + 1, 0), 0.0);
    double best = serial;
    for (int nd = lo; nd <= hi; ++nd) {
        const double t = greedy_end(runs, num_sms - nd, 0, 0, load) * tick;
        const double streamed = nd * kSmBytesPerSec * t;
        est[nd - lo] = streamed >= items ? greedy_end(runs, num_sms, nd, std::llround(item_work / nd / tick), load) * tick
                                         : t + (items - streamed) / kGpuBytesPerSec + tail;
        best = std::min(best, est[nd - lo]);
    }
    if (best >= serial) return 0;  // one kernel after the other
    // The middle of the longest run of candidates within 0.3 % of the best.
    int run_lo = -1, best_lo = lo, best_len = 0;
    for (int nd = lo; nd <= hi + 1; ++nd) {
        const bool near = nd <= hi && est[nd - lo] <= best * 1.003;
        if (near && run_lo < 0) run_lo = nd;
        if (!near && run_lo >= 0) {
            if (nd - run_lo > best_len) {
                best_len = nd - run_lo;
                best_lo = run_lo;
            }
            run_lo = -1;
        }
    }
    return best_lo + (best_len - 1) / 2;
}

// out_meta / out_cap: when given and large enough, the work lists are written straight into that
// image (the layout write_meta produces), skipping the intermediate lists.
pkv_status plan_lists(const int32_t* qsl, const int32_t* ctx, int R, int Hq, int Hkv, int D, pkv_dtype dt,
                      const pkv_plan_options* opts, int num_sms, PlanLists* L, pkv_plan* plan,
                      unsigned char* out_meta = nullptr, size_t out_cap = 0) {
    if (!qsl || (R > 0 && !ctx) || !plan) return fail(PKV_ERR_INVALID_ARG, "null planner argument");
    if (R < 0) return fail(PKV_ERR_INVALID_ARG, "num_reqs < 0");
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Hkv > 32767)
        return fail(PKV_ERR_INVALID_ARG, "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)", Hq, Hkv);
    if (D != 64 && D != 128) return fail(PKV_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", D);
    if (!dtype_ok(dt)) return fail(PKV_ERR_INVALID_ARG, "bad dtype %d", (int)dt);
    const int G = Hq / Hkv;
    if (qsl[0] != 0) return fail(PKV_ERR_INVALID_ARG, "query_start_loc[0] = %d, expected 0", qsl[0]);
    for (int r = 0; r < R; ++r) {
        const int n = qsl[r + 1] - qsl[r];
        if (n < 0) return fail(PKV_ERR_INVALID_ARG, "query_start_loc decreases at request %d", r);
        if (ctx[r] < n) return fail(PKV_ERR_INVALID_ARG, "request %d: context_len %d < num_tokens %d", r, ctx[r], n);
        if (n > 0 && ctx[r] < 1) return fail(PKV_ERR_INVALID_ARG, "request %d: empty context with query rows", r);
    }
    pkv_plan_options o{};
    if (opts) o = *opts;
    const bool tc_ok = !o.cuda_core_only && prefill_tc_supported((int)dt, D, G);
    const int eb = elem_bytes(dt);
    if (o.decode_kernel < 0 || o.decode_kernel > 2) return fail(PKV_ERR_INVALID_ARG, "decode_kernel %d", o.decode_kernel);
    const bool mma_ok = decode_mma_supported((int)dt, D);
    // Multi-row requests whose rows x heads fit one 16-slot MMA item stream each K/V block once
    // there, as a tcgen05 tile would, and faster (measured on speculative verify steps); larger
    // ones go to the tiles.
    const int tc_min = o.tc_min_rows >= 2 ? o.tc_min_rows : (mma_ok && o.decode_kernel != 1 ? std::max(2, kMmaSlots / G + 1) : 2);
    if (o.decode_kernel == 2 && !mma_ok)
        return fail(PKV_ERR_UNSUPPORTED, "the MMA decode kernel needs f16/bf16 and head_dim 128");
    // Kernel for the CUDA-core rows: warp-level MMAs over 16 (row, head) slots wherever the type
    // and head size allow (measured as fast or faster than the FMA kernel for groups of 1 to 8
    // and for packed rows); the FMA kernel otherwise.
    const int kind = o.decode_kernel ? o.decode_kernel : (mma_ok ? 2 : 1);
    const int slot_cap = kind == 2 ? kMmaSlots : kMaxGroupPerItem;
    const int hpi = (o.heads_per_item > 0 && o.heads_per_item <= slot_cap) ? o.heads_per_item : std::min(G, slot_cap);
    // Rows per CUDA-core item: as many consecutive rows of a request as fit the item's slots.
    const int rows_cap = slot_cap / hpi;
    const int rpi = o.rows_per_item > 0 ? std::min(o.rows_per_item, rows_cap) : rows_cap;

    // CUDA-core work: nrows consecutive rows whose first sees keys < limit, over the blocks
    // [bs, be). kind 0: ordinary rows (partials only when split into several chunks); kind 1: the
    // shared-prefix blocks of a group of requests (rows j .. j+nrows-1 of the group, always
    // partials); kind 2: one group member's own blocks (always merged with its group's partials).
    struct CoreRow { int row, req, limit, nrows, bs, be, kind, group, j; };
    static thread_local std::vector<CoreRow> core_rows;
    core_rows.clear();
    core_rows.reserve(R > 0 ? (size_t)qsl[R] : 0);
    int64_t kv_bytes = 0, flops = 0, tile_kv = 0, tile_flops = 0;
    int decode_rows = 0, prefill_rows = 0, max_blocks = 0;
    bool rows_split = false;  // some request's rows span several items (each reads the same blocks)
    for (int r = 0; r < R; ++r) {
        const int n = qsl[r + 1] - qsl[r];
        if (n == 0) continue;
        const int P = ctx[r] - n;
        max_blocks = std::max<int>(max_blocks, (int)ceil_div(ctx[r], kBlockSize));
        const int64_t req_kv = (int64_t)ctx[r] * Hkv * 2 * D * eb;
        // keys attended: sum_j (P + j + 1)
        const int64_t req_flops = 4LL * D * Hq * ((int64_t)n * P + (int64_t)n * (n + 1) / 2);
        kv_bytes += req_kv;
        flops += req_flops;
        if (n > 1 && tc_ok && n >= tc_min) {
            tile_kv += req_kv;
            tile_flops += req_flops;
            prefill_rows += n;
            const int tt = tile_tokens(G);
            for (int h = 0; h < Hkv; ++h)
                for (int t0 = 0; t0 < n; t0 += tt) {
                    const int last = std::min(n, t0 + tt);
                    const int keys = P + last;  // keys visible to the tile's last row
                    L->tiles.push_back(PrefillTile{r, h, t0, (int)ceil_div(keys, 128)});
                }
        } else {
            if (n == 1) ++decode_rows;
            if (n > rpi) rows_split = true;
            for (int j = 0; j < n; j += rpi) {
                const int nr = std::min(rpi, n - j);
                core_rows.push_back(CoreRow{qsl[r] + j, r, P + j + 1, nr, 0, (int)ceil_div(P + j + nr, kBlockSize), 0, -1, 0});
            }
        }
    }
    // Shared prefixes (cascade): consecutive decode requests whose block tables begin with the
    // same physical blocks (parallel samples, beam candidates, requests reusing a cached prompt)
    // read those blocks once for all of them: one set of items over the shared blocks for all their
    // rows, one per request over its own blocks, combined by the log-sum-exp merge. Needs the host
    // copy of the tables.
    struct Group { int r0, r1, k, first_core; };  // requests [r0, r1), k shared blocks
    static thread_local std::vector<Group> grps;
    grps.clear();
    if (o.h_block_tables && o.block_table_stride > 0 && rpi >= 2) {  // an item must hold >= 2 rows
        const int minb = o.min_shared_blocks > 0 ? o.min_shared_blocks : 4;
        const int stride = o.block_table_stride;
        auto decode_row = [&](int r) { return qsl[r + 1] - qsl[r] == 1; };
        for (int r = 0; r < R;) {
            if (!decode_row(r)) { ++r; continue; }
            int k = std::min(ctx[r] / kBlockSize, stride);
            int e = r + 1;
            while (e < R && decode_row(e)) {
                const int kk = std::min(k, ctx[e] / kBlockSize);
                const int32_t* a = o.h_block_tables + (size_t)r * stride;
                const int32_t* b = o.h_block_tables + (size_t)e * stride;
                int cp = 0;
                while (cp < kk && a[cp] == b[cp]) ++cp;
                if (cp < minb) break;
                k = cp;
                ++e;
            }
            if (e - r >= 2 && k >= minb) {
                grps.push_back(Group{r, e, k, 0});
                r = e;
            } else {
                ++r;
            }
        }
    }
    if (!grps.empty()) {
        // Group members' rows: their own blocks only. Then the groups' shared rows, first.
        std::vector<int> member_group(R, -1);
        for (int gi = 0; gi < (int)grps.size(); ++gi)
            for (int r = grps[gi].r0; r < grps[gi].r1; ++r) member_group[r] = gi;
        for (CoreRow& c : core_rows) {
            const int gi = member_group[c.req];
            if (gi < 0) continue;
            c.kind = 2;
            c.group = gi;
            c.j = c.req - grps[gi].r0;
            c.bs = grps[gi].k;
        }
        std::vector<CoreRow> shared;
        for (int gi = 0; gi < (int)grps.size(); ++gi) {
            Group& g = grps[gi];
            g.first_core = (int)shared.size();
            const int m = g.r1 - g.r0;
            for (int j = 0; j < m; j += rpi)
                shared.push_back(CoreRow{qsl[g.r0] + j, g.r0, g.k * kBlockSize, std::min(rpi, m - j), 0, g.k, 1, gi, j});
        }
        core_rows.insert(core_rows.begin(), shared.begin(), shared.end());
    }

    // Chunk length: enough items per resident warp that the snake-dealt longest-first order (below)
    // ends evenly, but never below 16 blocks. A split item of s (row, head) slots writes s partials
    // that s merge warps read back, so items of one or two slots are cut finer: 6 items per warp
    // for s <= 2, 4 otherwise. Measured on the decode batches with the snake dealing against
    // fixed lengths: one-slot rows (13B-shaped decode) best at 24 blocks (18: +0.9 %, 36: +0.8 %),
    // 4-slot GQA rows at 39 (26: +1.7 %), 5-slot verify rows at 39 (24: +1.7 %, 52: +6 %);
    // parallel sampling gains 4 % from the 16-block floor (8 before).
    const int groups = (int)ceil_div(G, hpi);
    int64_t total_blocks = 0;
    int max_slots = 1;
    for (const CoreRow& c : core_rows) {
        total_blocks += (int64_t)(c.be - c.bs) * Hkv * groups;
        max_slots = std::max(max_slots, std::min(hpi, G) * c.nrows);
    }
    int chunk;
    if (o.no_split) chunk = 1 << 30;
    else if (o.split_blocks > 0) chunk = o.split_blocks;
    else {
        const int64_t workers = (int64_t)std::max(num_sms, 1) * 8;
        const int per_worker = max_slots <= 2 ? 6 : 4;
        chunk = (int)std::min<int64_t>(std::max<int64_t>(ceil_div(total_blocks, workers * per_worker), 16), 1 << 20);
    }
    auto pieces_of = [&](const CoreRow& c) { return (int)ceil_div(c.be - c.bs, chunk); };
    auto with_partials = [&](const CoreRow& c, int pieces) { return c.kind != 0 || pieces > 1; };
    // Items are placed directly at their position in a stable order by length, longest first. For
    // the FMA kernel, whose persistent warps run fixed positions (warp w runs w, w + W, w + 2W, ...),
    // they are dealt in a snake: each odd round of W items is dealt in reverse, so the warps that
    // took the longest items of one round take the shortest of the next and the warps' totals even
    // out (W = 8 resident warps per SM; a launch with another count still runs every item). Pass 1
    // counts the items of each length from the row lengths alone; pass 2 writes every item to its
    // slot.
    size_t n_items = 0, n_merge = 0;
    int max_len = 0;
    for (const CoreRow& c : core_rows) {
        const int pieces = pieces_of(c);
        n_items += (size_t)pieces * Hkv * groups;
        if (c.kind == 2 || (c.kind == 0 && pieces > 1)) n_merge += (size_t)Hkv * groups;
        max_len = std::max(max_len, std::min(c.be - c.bs, chunk));
    }
    std::vector<size_t>& start = L->start;
    start.assign((size_t)max_len + 2, 0);
    for (const CoreRow& c : core_rows) {
        const int pieces = pieces_of(c);
        if (pieces == 0) continue;
        const size_t per = (size_t)Hkv * groups;
        start[std::min(c.be - c.bs, chunk)] += per * (pieces > 1 ? pieces - 1 : 1);
        if (pieces > 1) start[(c.be - c.bs) - (pieces - 1) * chunk] += per;
    }
    size_t acc = 0;
    for (int len = max_len; len >= 1; --len) {
        const size_t cnt = start[len];
        start[len] = acc;
        acc += cnt;
    }
    // Dealing cursors: the items of length `len` take the sorted positions start[len], +1, ...;
    // each cursor keeps its position as (round, index in the round) so the snake needs no
    // division per item.
    // The warp-MMA kernel takes items greedily from a ticket counter: plain longest-first order
    // (one round). The FMA kernel's warps run fixed positions: the snake over its W warps.
    const uint32_t deal = kind == 2 ? (uint32_t)std::max<size_t>(n_items, 1) : (uint32_t)std::max(num_sms, 1) * 8;
    const uint32_t n_items32 = (uint32_t)n_items;  // the plan counts items in int32
    std::vector<PlanLists::Cursor>& cursor = L->cursor;
    cursor.resize((size_t)max_len + 2);
    for (int len = 1; len <= max_len; ++len)
        cursor[len] = PlanLists::Cursor{(uint32_t)(start[len] / deal), (uint32_t)(start[len] % deal)};
    auto place = [&](int len) -> size_t {
        PlanLists::Cursor& q = cursor[len];
        const size_t at = (size_t)q.round * deal +
                          ((q.round & 1) ? std::min(deal, n_items32 - q.round * deal) - 1 - q.index : q.index);
        if (++q.index == deal) {
            q.index = 0;
            ++q.round;
        }
        return at;
    };
    // Image layout (header, items, tiles, merges; 256-byte aligned), known from the counts.
    const int64_t off_items = 256;
    const int64_t off_tiles = align256(off_items + (int64_t)n_items * sizeof(DecodeItem));
    const int64_t off_merge = align256(off_tiles + (int64_t)L->tiles.size() * sizeof(PrefillTile));
    const int64_t meta_bytes = align256(off_merge + (int64_t)n_merge * sizeof(MergeRow));
    const bool direct = out_meta && out_cap >= (size_t)meta_bytes;
    DecodeItem* items;
    MergeRow* merges;
    if (direct) {
        items = reinterpret_cast<DecodeItem*>(out_meta + off_items);
        merges = reinterpret_cast<MergeRow*>(out_meta + off_merge);
    } else {
        L->items.resize(n_items);
        L->merges.resize(n_merge);
        items = L->items.data();
        merges = L->merges.data();
    }
    L->num_items = n_items;
    L->num_merges = n_merge;
    if (direct) L->direct = out_meta;
    size_t mi = 0;
    int partials = 0;
    // First partial entry of each (shared row, KV head, head group): members' merges point there.
    std::vector<int>& shared_first = L->shared_first;
    shared_first.clear();
    for (int ci = 0; ci < (int)core_rows.size(); ++ci) {
        const CoreRow& c = core_rows[ci];
        const int pieces = pieces_of(c);
        for (int h = 0; h < Hkv; ++h)
            for (int g0 = 0; g0 < G; g0 += hpi) {
                const int nh = std::min(hpi, G - g0);
                int first = -1;
                if (with_partials(c, pieces)) {
                    first = partials;
                    partials += pieces;
                }
                if (c.kind == 1) {
                    shared_first.push_back(first);
                } else if (c.kind == 2 || pieces > 1) {
                    int xf = -1, xc = 0, xs = 0;
                    if (c.kind == 2) {
                        const Group& g = grps[c.group];
                        const CoreRow& sc = core_rows[g.first_core + c.j / rpi];
                        xf = shared_first[((size_t)(g.first_core + c.j / rpi) * Hkv + h) * groups + g0 / hpi];
                        xc = pieces_of(sc);
                        xs = (c.j - sc.j) * nh;
                    }
                    merges[mi++] = MergeRow{c.row, h * G + g0, nh * c.nrows, first, first >= 0 ? pieces : 0, nh, xf, xc, xs,
                                            {0, 0, 0}};
                }
                for (int p = 0; p < pieces; ++p) {
                    const int b0 = c.bs + p * chunk, b1 = std::min(c.be, b0 + chunk);
                    items[place(b1 - b0)] = DecodeItem{c.row, c.req, (int16_t)h, (int16_t)c.nrows, g0, b0, b1, c.limit,
                                                       first >= 0 ? first + p : -1};
                }
            }
    }
    L->num_partials = partials;
    // Tiles: longest requests first; a (request, KV head)'s tiles stay adjacent (longest first) so
    // the CTAs running at the same time share that head's K/V through L2.
    std::vector<int>& req_keys = L->req_keys;
    req_keys.assign(R > 0 ? R : 1, 0);
    for (const PrefillTile& t : L->tiles) req_keys[t.req] = std::max(req_keys[t.req], t.key_tiles);
    std::stable_sort(L->tiles.begin(), L->tiles.end(), [&](const PrefillTile& a, const PrefillTile& b) {
        if (req_keys[a.req] != req_keys[b.req]) return req_keys[a.req] > req_keys[b.req];
        if (a.req != b.req) return a.req < b.req;
        if (a.kv_head != b.kv_head) return a.kv_head < b.kv_head;
        return a.tok0 > b.tok0;
    });

    std::memset(plan, 0, sizeof *plan);
    plan->magic = PKV_PLAN_MAGIC;
    plan->num_reqs = R;
    plan->num_q_tokens = R > 0 ? qsl[R] : 0;
    plan->num_q_heads = Hq;
    plan->num_kv_heads = Hkv;
    plan->head_dim = D;
    plan->dtype = (int32_t)dt;
    plan->num_decode_rows = decode_rows;
    plan->num_prefill_rows = prefill_rows;
    plan->num_items = (int32_t)n_items;
    plan->num_tiles = (int32_t)L->tiles.size();
    plan->num_merge_rows = (int32_t)n_merge;
    plan->num_partials = L->num_partials;
    plan->split_blocks = chunk;
    plan->max_blocks = max_blocks;
    plan->heads_per_item = hpi;
    int max_rows = 0;
    for (const CoreRow& c : core_rows) max_rows = std::max(max_rows, c.nrows);
    plan->rows_per_item = max_rows;
    plan->decode_kernel = n_items == 0 ? 0 : kind;
    // Partial entries hold as many (row, head) slots as the largest item has.
    const int part_stride = std::max(1, std::min(slot_cap, hpi * std::max(max_rows, 1)));
    plan->part_stride = part_stride;
    int merge_slots = 0;
    for (size_t i = 0; i < n_merge; ++i) merge_slots = std::max(merge_slots, merges[i].num_slots);
    plan->merge_slots = merge_slots;
    plan->off_items = off_items;  // the first 256 bytes are reserved
    plan->off_tiles = off_tiles;
    plan->off_merge = off_merge;
    plan->meta_bytes = meta_bytes;
    int64_t off = meta_bytes;
    plan->off_part_o = off;
    off = align256(off + (int64_t)L->num_partials * part_stride * D * 4);
    plan->off_part_ml = off;
    off = align256(off + (int64_t)L->num_partials * part_stride * 2 * 4);
    plan->ws_bytes = off;
    plan->kv_bytes = kv_bytes;
    plan->attn_flops = flops;
    // K/V the CUDA-core kernel must read: a shared prefix once per group, not once per member.
    int64_t shared_saved_tokens = 0;
    for (const Group& g : grps) shared_saved_tokens += (int64_t)(g.r1 - g.r0 - 1) * g.k * kBlockSize;
    plan->core_kv_bytes = kv_bytes - tile_kv - shared_saved_tokens * Hkv * 2 * D * eb;
    plan->tile_kv_bytes = tile_kv;
    plan->tile_flops = tile_flops;
    if (grps.empty() && ceil_div(G, hpi) == 1 && !rows_split) plan->flags |= PKV_PLAN_SINGLE_READ;
    // Mixed batch: the tcgen05 kernel's persistent CTAs (one per SM) also serve the warp-MMA items;
    // decode_sms of them start on items, the rest on tiles, and each turns to the other queue when
    // its own empties.
    plan->decode_sms = 0;
    if (o.decode_sms >= 0 && kind == 2 && n_items > 0 && !L->tiles.empty() && num_sms >= 2) {
        int nd = o.decode_sms;
        if (nd == 0) nd = mixed_split(L->tiles, plan->core_kv_bytes, (int64_t)n_items, max_slots, num_sms);
        if (nd > 0) plan->decode_sms = std::min(nd, num_sms - 1);
    }
    return PKV_OK;
}

// The work-list image: each list at its offset, the header and the alignment gaps zeroed.
// Fills the image around the items and merges (header, gaps, tiles) -- and the items and merges
// themselves unless the planner already wrote them in place.
void write_meta(const PlanLists& L, const pkv_plan& plan, unsigned char* meta) {
    if (L.direct && L.direct != meta) {
        std::memcpy(meta, L.direct, (size_t)plan.meta_bytes);
        return;
    }
    const bool in_place = L.direct == meta;
    const size_t end_items = plan.off_items + L.num_items * sizeof(DecodeItem);
    const size_t end_tiles = plan.off_tiles + L.tiles.size() * sizeof(PrefillTile);
    const size_t end_merge = plan.off_merge + L.num_merges * sizeof(MergeRow);
    std::memset(meta, 0, (size_t)plan.off_items);
    if (!in_place && L.num_items) std::memcpy(meta + plan.off_items, L.items.data(), L.num_items * sizeof(DecodeItem));
    std::memset(meta + end_items, 0, (size_t)plan.off_tiles - end_items);
    if (!L.tiles.empty()) std::memcpy(meta + plan.off_tiles, L.tiles.data(), L.tiles.size() * sizeof(PrefillTile));
    std::memset(meta + end_tiles, 0, (size_t)plan.off_merge - end_tiles);
    if (!in_place && L.num_merges) std::memcpy(meta + plan.off_merge, L.merges.data(), L.num_merges * sizeof(MergeRow));
    std::memset(meta + end_merge, 0, (size_t)plan.meta_bytes - end_merge);
}

// Per-thread kernel timing state (pkv_profile_start / pkv_profile_stop).
struct Profiler {
    bool on = false;
    std::vector<cudaEvent_t> ev;  // 2 per record
    std::vector<int> kind;
    int used = 0;
    int launches[PKV_KERNEL_KINDS] = {0};
    int dropped = 0;
};
thread_local Profiler t_prof;

// Brackets one launch with events when profiling is on.
struct ProfileScope {
    int slot = -1;
    cudaStream_t s;
    ProfileScope(int k, cudaStream_t stream) : s(stream) {
        if (!t_prof.on) return;
        t_prof.launches[k]++;
        if (t_prof.used * 2 + 1 >= (int)t_prof.ev.size()) {
            t_prof.dropped++;
            return;
        }
        slot = t_prof.used++;
        t_prof.kind[slot] = k;
        cudaEventRecord(t_prof.ev[2 * slot], s);
    }
    ~ProfileScope() {
        if (slot >= 0) cudaEventRecord(t_prof.ev[2 * slot + 1], s);
    }
};

}  // namespace

void set_last_error(const char* msg) { t_last_error = msg ? msg : ""; }

unsigned long long current_context_id() {
    typedef CUresult (*GetCurrent)(CUcontext*);
    typedef CUresult (*GetId)(CUcontext, unsigned long long*);
    static std::once_flag once;
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(p);
    });
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}



DeviceError* device_error_word() {
    static std::mutex mu;
    static DeviceError* addr[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<DeviceError*>(p);
    }
    return addr[dev];
}

}  // namespace pkv

using namespace pkv;

extern "C" {

const char* pkv_status_string(pkv_status s) {
    switch (s) {
        case PKV_OK: return "ok";
        case PKV_ERR_INVALID_ARG: return "invalid argument";
        case PKV_ERR_UNSUPPORTED: return "unsupported";
        case PKV_ERR_CUDA: return "CUDA error";
        case PKV_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case PKV_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case PKV_ERR_DEVICE_RANGE: return "device index out of range";
        case PKV_ERR_OUT_OF_BLOCKS: return "out of free blocks";
    }
    return "unknown status";
}

const char* pkv_last_error(void) { return t_last_error.c_str(); }

const char* pkv_version(void) { return "pkv 0.1 sm_100a"; }

pkv_status pkv_slot_mapping(const int32_t* block_tables, int max_blocks_per_seq, const int32_t* query_start_loc,
                            const int32_t* context_lens, int num_reqs, int num_blocks, int64_t* slot_mapping,
                            int num_tokens, pkv_stream_t stream) {
    if (num_reqs < 0 || num_tokens < 0 || max_blocks_per_seq < 0 || num_blocks < 0)
        return fail(PKV_ERR_INVALID_ARG, "negative size");
    if (num_tokens == 0 || num_reqs == 0) return PKV_OK;
    if (!block_tables || !query_start_loc || !context_lens || !slot_mapping)
        return fail(PKV_ERR_INVALID_ARG, "null pointer");
    DeviceError* err = device_error_word();
    if (!err) return fail(PKV_ERR_CUDA, "device error word unavailable");
    ProfileScope prof(PKV_KERNEL_SLOT_MAPPING, (cudaStream_t)stream);
    cudaError_t e = launch_slot_mapping(block_tables, max_blocks_per_seq, query_start_loc, context_lens, num_reqs,
                                        num_blocks, slot_mapping, num_tokens, err, (cudaStream_t)stream);
    return e == cudaSuccess ? PKV_OK : cuda_fail(e, "slot_mapping launch");
}

pkv_status pkv_kv_cache_write(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                              const int64_t* slot_mapping, int num_tokens, int num_blocks, int num_kv_heads,
                              int head_dim, int block_size, pkv_dtype dtype, pkv_stream_t stream) {
    if (num_tokens < 0 || num_blocks < 0 || num_kv_heads <= 0 || head_dim <= 0)
        return fail(PKV_ERR_INVALID_ARG, "bad size");
    if (!dtype_ok(dtype)) return fail(PKV_ERR_INVALID_ARG, "bad dtype");
    if (block_size != kBlockSize) return fail(PKV_ERR_UNSUPPORTED, "block_size %d (only 16)", block_size);
    const int row = head_dim * elem_bytes(dtype);
    if (row % 16 != 0 || row > 1024) return fail(PKV_ERR_UNSUPPORTED, "row of %d bytes", row);
    if (num_tokens == 0) return PKV_OK;
    if (!k_new || !v_new || !k_pool || !v_pool || !slot_mapping) return fail(PKV_ERR_INVALID_ARG, "null pointer");
    if (((uintptr_t)k_new | (uintptr_t)v_new | (uintptr_t)k_pool | (uintptr_t)v_pool) & 15)
        return fail(PKV_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    DeviceError* err = device_error_word();
    if (!err) return fail(PKV_ERR_CUDA, "device error word unavailable");
    ProfileScope prof(PKV_KERNEL_KV_WRITE, (cudaStream_t)stream);
    cudaError_t e = launch_kv_write(k_new, v_new, k_pool, v_pool, slot_mapping, num_tokens, num_blocks, num_kv_heads,
                                    row, err, (cudaStream_t)stream);
    return e == cudaSuccess ? PKV_OK : cuda_fail(e, "kv_cache_write launch");
}

pkv_status pkv_copy_blocks(void* const* k_pools, void* const* v_pools, int num_layers, const int32_t* block_mapping,
                           int num_pairs, int num_blocks, int num_kv_heads, int head_dim, int block_size,
                           pkv_dtype dtype, pkv_stream_t stream) {
    if (num_layers < 0 || num_pairs < 0 || num_blocks < 0 || num_kv_heads <= 0 || head_dim <= 0)
        return fail(PKV_ERR_INVALID_ARG, "bad size");
    if (!dtype_ok(dtype)) return fail(PKV_ERR_INVALID_ARG, "bad dtype");
    if (block_size != kBlockSize) return fail(PKV_ERR_UNSUPPORTED, "block_size %d (only 16)", block_size);
    const long long bb = (long long)num_kv_heads * kBlockSize * head_dim * elem_bytes(dtype);
    if (bb % 16 != 0) return fail(PKV_ERR_UNSUPPORTED, "block of %lld bytes", bb);
    if (num_pairs == 0 || num_layers == 0) return PKV_OK;
    if (!k_pools || !v_pools || !block_mapping) return fail(PKV_ERR_INVALID_ARG, "null pointer");
    for (int l = 0; l < num_layers; ++l) {
        if (!k_pools[l] || !v_pools[l]) return fail(PKV_ERR_INVALID_ARG, "null pool pointer for layer %d", l);
        if (((uintptr_t)k_pools[l] | (uintptr_t)v_pools[l]) & 15)
            return fail(PKV_ERR_INVALID_ARG, "pools must be 16-byte aligned");
    }
    DeviceError* err = device_error_word();
    if (!err) return fail(PKV_ERR_CUDA, "device error word unavailable");
    ProfileScope prof(PKV_KERNEL_COPY_BLOCKS, (cudaStream_t)stream);
    cudaError_t e = launch_copy_blocks(k_pools, v_pools, num_layers, block_mapping, num_pairs, num_blocks, bb, err,
                                       (cudaStream_t)stream);
    return e == cudaSuccess ? PKV_OK : cuda_fail(e, "copy_blocks launch");
}

pkv_status pkv_attention_workspace_size(const int32_t* h_query_start_loc, const int32_t* h_context_lens,
                                        int num_reqs, int num_q_heads, int num_kv_heads, int head_dim,
                                        pkv_dtype dtype, const pkv_plan_options* opts, size_t* bytes) {
    if (!bytes) return fail(PKV_ERR_INVALID_ARG, "null bytes");
    PlanLists& L = thread_lists();
    pkv_plan plan;
    const int sms = (opts && opts->num_sms > 0) ? opts->num_sms : current_sm_count();
    pkv_status s = plan_lists(h_query_start_loc, h_context_lens, num_reqs, num_q_heads, num_kv_heads, head_dim,
                              dtype, opts, sms, &L, &plan);
    if (s != PKV_OK) return s;
    *bytes = (size_t)plan.ws_bytes;
    return PKV_OK;
}

pkv_status pkv_attention_plan_host(const int32_t* h_query_start_loc, const int32_t* h_context_lens, int num_reqs,
                                   int num_q_heads, int num_kv_heads, int head_dim, pkv_dtype dtype,
                                   const pkv_plan_options* opts, void* h_meta, size_t meta_capacity,
                                   pkv_plan* plan) {
    PlanLists& L = thread_lists();
    const int sms = (opts && opts->num_sms > 0) ? opts->num_sms : 148;
    pkv_status s = plan_lists(h_query_start_loc, h_context_lens, num_reqs, num_q_heads, num_kv_heads, head_dim,
                              dtype, opts, sms, &L, plan, static_cast<unsigned char*>(h_meta), h_meta ? meta_capacity : 0);
    if (s != PKV_OK) return s;
    if (h_meta) {
        if (meta_capacity < (size_t)plan->meta_bytes)
            return fail(PKV_ERR_WORKSPACE_TOO_SMALL, "metadata needs %lld bytes", (long long)plan->meta_bytes);
        write_meta(L, *plan, static_cast<unsigned char*>(h_meta));
    }
    return PKV_OK;
}

pkv_status pkv_attention_plan(const int32_t* h_query_start_loc, const int32_t* h_context_lens, int num_reqs,
                              int num_q_heads, int num_kv_heads, int head_dim, pkv_dtype dtype,
                              const pkv_plan_options* opts, void* d_workspace, size_t ws_bytes, pkv_plan* plan,
                              pkv_stream_t stream) {
    PlanLists& L = thread_lists();
    const int sms = (opts && opts->num_sms > 0) ? opts->num_sms : current_sm_count();
    pkv_status s = plan_lists(h_query_start_loc, h_context_lens, num_reqs, num_q_heads, num_kv_heads, head_dim,
                              dtype, opts, sms, &L, plan);
    if (s != PKV_OK) return s;
    if (!d_workspace) return fail(PKV_ERR_INVALID_ARG, "null workspace");
    if (ws_bytes < (size_t)plan->ws_bytes) {
        plan->magic = 0;
        return fail(PKV_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes, plan needs %lld", ws_bytes,
                    (long long)plan->ws_bytes);
    }
    static thread_local std::vector<unsigned char> meta;
    meta.resize((size_t)plan->meta_bytes);
    write_meta(L, *plan, meta.data());
    // Pageable source: the call returns once the bytes are staged, so `meta` may be reused.
    cudaError_t e = cudaMemcpyAsync(d_workspace, meta.data(), meta.size(), cudaMemcpyHostToDevice, (cudaStream_t)stream);
    if (e != cudaSuccess) {
        plan->magic = 0;
        return cuda_fail(e, "plan upload");
    }
    return PKV_OK;
}

pkv_status pkv_attention_plan_async(const int32_t* h_query_start_loc, const int32_t* h_context_lens, int num_reqs,
                                    int num_q_heads, int num_kv_heads, int head_dim, pkv_dtype dtype,
                                    const pkv_plan_options* opts, void* h_meta, size_t meta_capacity,
                                    void* d_workspace, size_t ws_bytes, int32_t* h_desc, int32_t* d_desc,
                                    pkv_plan* plan, pkv_stream_t stream) {
    if ((h_desc == nullptr) != (d_desc == nullptr))
        return fail(PKV_ERR_INVALID_ARG, "h_desc and d_desc must both be given or both be NULL");
    PlanLists& L = thread_lists();
    const int sms = (opts && opts->num_sms > 0) ? opts->num_sms : current_sm_count();
    pkv_status s = plan_lists(h_query_start_loc, h_context_lens, num_reqs, num_q_heads, num_kv_heads, head_dim,
                              dtype, opts, sms, &L, plan, static_cast<unsigned char*>(h_meta), h_meta ? meta_capacity : 0);
    if (s != PKV_OK) return s;
    if (!h_meta || !d_workspace || meta_capacity < (size_t)plan->meta_bytes || ws_bytes < (size_t)plan->ws_bytes) {
        plan->magic = 0;
        return fail(PKV_ERR_WORKSPACE_TOO_SMALL, "work lists need %lld host / %lld device bytes (given %zu / %zu)",
                    (long long)plan->meta_bytes, (long long)plan->ws_bytes, h_meta ? meta_capacity : 0,
                    d_workspace ? ws_bytes : 0);
    }
    write_meta(L, *plan, static_cast<unsigned char*>(h_meta));
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(d_workspace, h_meta, (size_t)plan->meta_bytes, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess && h_desc && num_reqs >= 0) {
        std::memcpy(h_desc, h_query_start_loc, sizeof(int32_t) * ((size_t)num_reqs + 1));
        if (num_reqs > 0) std::memcpy(h_desc + num_reqs + 1, h_context_lens, sizeof(int32_t) * (size_t)num_reqs);
        e = cudaMemcpyAsync(d_desc, h_desc, sizeof(int32_t) * (2 * (size_t)num_reqs + 1), cudaMemcpyHostToDevice, st);
    }
    if (e != cudaSuccess) {
        plan->magic = 0;
        return cuda_fail(e, "plan upload");
    }
    return PKV_OK;
}

pkv_status pkv_paged_attention(void* out, const void* q, const void* k_pool, const void* v_pool,
                               const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                               const int32_t* query_start_loc, int num_blocks, float scale, const pkv_plan* plan,
                               void* d_workspace, size_t ws_bytes, pkv_stream_t stream) {
    if (!plan || plan->magic != PKV_PLAN_MAGIC) return fail(PKV_ERR_INVALID_ARG, "plan missing or not filled");
    if (plan->num_q_tokens == 0) return PKV_OK;
    if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens || !query_start_loc || !d_workspace)
        return fail(PKV_ERR_INVALID_ARG, "null pointer");
    if (ws_bytes < (size_t)plan->ws_bytes)
        return fail(PKV_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes, plan needs %lld", ws_bytes, (long long)plan->ws_bytes);
    if (num_blocks <= 0 || max_blocks_per_seq < plan->max_blocks)
        return fail(PKV_ERR_INVALID_ARG, "num_blocks %d / max_blocks_per_seq %d too small for the plan (%d)", num_blocks,
                    max_blocks_per_seq, plan->max_blocks);
    if (((uintptr_t)out | (uintptr_t)q | (uintptr_t)k_pool | (uintptr_t)v_pool | (uintptr_t)d_workspace) & 15)
        return fail(PKV_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    if (!std::isfinite(scale)) return fail(PKV_ERR_INVALID_ARG, "scale is not finite");
    DeviceError* err = device_error_word();
    if (!err) return fail(PKV_ERR_CUDA, "device error word unavailable");
    const int sms = current_sm_count();
    unsigned char* ws = static_cast<unsigned char*>(d_workspace);
    const float scale_log2 = scale * 1.4426950408889634f;
    cudaStream_t s = (cudaStream_t)stream;
    const int G = plan->num_q_heads / plan->num_kv_heads;
    // Mixed batch: the tcgen05 kernel's persistent CTAs also serve the warp-MMA split-K items
    // (plan->decode_sms of them start on items, the others on tiles; each turns to the other queue
    // once its own is empty), so the HBM-bound items and the tensor-bound tiles share the GPU.
    const bool mixed = plan->decode_sms > 0 && plan->num_tiles > 0 && plan->num_items > 0 && plan->decode_kernel == 2;
    int* work = reinterpret_cast<int*>(ws);  // the header's first 16 bytes: zeroed by the plan upload
    DecodeArgs d{};
    d.q = q; d.out = out; d.k_pool = k_pool; d.v_pool = v_pool; d.block_tables = block_tables;
    d.items = reinterpret_cast<const DecodeItem*>(ws + plan->off_items);
    d.part_o = reinterpret_cast<float*>(ws + plan->off_part_o);
    d.part_ml = reinterpret_cast<float*>(ws + plan->off_part_ml);
    d.err = err; d.work = work; d.num_items = plan->num_items; d.max_blocks_per_seq = max_blocks_per_seq;
    d.num_blocks = num_blocks; d.num_q_heads = plan->num_q_heads; d.num_kv_heads = plan->num_kv_heads;
    d.group = G; d.heads_per_item = plan->heads_per_item;
    d.slots_per_item = plan->heads_per_item * std::max(plan->rows_per_item, 1);
    d.part_stride = plan->part_stride;
    d.scale_log2 = scale_log2;
    d.pdl = true;
    // Streamed once, the split-K kernel's K/V may leave L2 first (measured: c2, c3 and c6 steps 3-4 %
    // faster; the small kernels around it keep their data in L2). Not in the mixed launch, where
    // it measured 0.8 % slower.
    d.evict_first = !mixed && (plan->flags & PKV_PLAN_SINGLE_READ) != 0;
    pkv_status st = PKV_OK;
    if (plan->num_tiles > 0) {
        PrefillArgs a{};
        a.q = q; a.out = out; a.k_pool = k_pool; a.v_pool = v_pool; a.block_tables = block_tables;
        a.context_lens = context_lens; a.query_start_loc = query_start_loc;
        a.tiles = reinterpret_cast<const PrefillTile*>(ws + plan->off_tiles);
        a.err = err; a.work = work; a.decode_ctas = mixed ? plan->decode_sms : 0;
        a.num_tiles = plan->num_tiles; a.max_blocks_per_seq = max_blocks_per_seq;
        a.num_blocks = num_blocks; a.num_q_heads = plan->num_q_heads; a.num_kv_heads = plan->num_kv_heads;
        a.group = G; a.num_q_tokens = plan->num_q_tokens; a.scale_log2 = scale_log2; a.pdl = true;
        DecodeArgs none = d;
        none.num_items = 0;
        ProfileScope prof(PKV_KERNEL_PREFILL_TC, s);
        cudaError_t e = launch_prefill_tc(plan->dtype, a, mixed ? d : none, sms, s);
        if (e != cudaSuccess) st = cuda_fail(e, "prefill tile launch");
    }
    if (st == PKV_OK && plan->num_items > 0 && !mixed) {
        ProfileScope prof(PKV_KERNEL_DECODE, s);
        cudaError_t e = plan->decode_kernel == 2 ? launch_decode_mma(plan->dtype, d, sms, s)
                                                 : launch_decode(plan->dtype, plan->head_dim, d, sms, s);
        if (e != cudaSuccess) st = cuda_fail(e, "decode launch");
    }
    if (st != PKV_OK) return st;
    if (plan->num_merge_rows > 0) {
        MergeArgs m{};
        m.out = out;
        m.rows = reinterpret_cast<const MergeRow*>(ws + plan->off_merge);
        m.part_o = reinterpret_cast<const float*>(ws + plan->off_part_o);
        m.part_ml = reinterpret_cast<const float*>(ws + plan->off_part_ml);
        m.num_rows = plan->num_merge_rows;
        m.num_q_heads = plan->num_q_heads;
        // One warp per (merge row, slot): the stride is the largest merge row, not the largest
        // item (a shared-prefix item packs several requests' rows; each member's merge row is one).
        m.slots_per_entry = std::max(plan->merge_slots, 1);
        m.part_stride = plan->part_stride;
        m.pdl = true;
        ProfileScope prof(PKV_KERNEL_MERGE, s);
        cudaError_t e = launch_merge(plan->dtype, plan->head_dim, m, s);
        if (e != cudaSuccess) return cuda_fail(e, "merge launch");
    }
    return PKV_OK;
}

pkv_status pkv_validate_tables(const int32_t* h_block_tables, const int32_t* h_context_lens, int num_reqs,
                               int max_blocks_per_seq, int num_blocks) {
    if (num_reqs < 0 || max_blocks_per_seq < 0 || num_blocks < 0) return fail(PKV_ERR_INVALID_ARG, "negative size");
    if (num_reqs > 0 && (!h_block_tables || !h_context_lens)) return fail(PKV_ERR_INVALID_ARG, "null pointer");
    for (int r = 0; r < num_reqs; ++r) {
        if (h_context_lens[r] < 0) return fail(PKV_ERR_INVALID_ARG, "request %d: negative context", r);
        const int64_t nb = ceil_div(h_context_lens[r], kBlockSize);
        if (nb > max_blocks_per_seq)
            return fail(PKV_ERR_INVALID_ARG, "request %d: needs %lld blocks, table holds %d", r, (long long)nb,
                        max_blocks_per_seq);
        for (int64_t i = 0; i < nb; ++i) {
            const int32_t b = h_block_tables[(int64_t)r * max_blocks_per_seq + i];
            if (b < 0 || b >= num_blocks)
                return fail(PKV_ERR_INVALID_ARG, "request %d: table entry %lld = %d outside [0, %d)", r, (long long)i, b,
                            num_blocks);
        }
    }
    return PKV_OK;
}

pkv_status pkv_validate_slots(const int64_t* h_slot_mapping, int num_tokens, int num_blocks) {
    if (num_tokens < 0 || num_blocks < 0) return fail(PKV_ERR_INVALID_ARG, "negative size");
    if (num_tokens > 0 && !h_slot_mapping) return fail(PKV_ERR_INVALID_ARG, "null pointer");
    std::vector<int64_t> s;
    s.reserve(num_tokens);
    const int64_t limit = (int64_t)num_blocks * kBlockSize;
    for (int t = 0; t < num_tokens; ++t) {
        const int64_t v = h_slot_mapping[t];
        if (v < 0) continue;
        if (v >= limit) return fail(PKV_ERR_INVALID_ARG, "token %d: slot %lld beyond the pool", t, (long long)v);
        s.push_back(v);
    }
    std::sort(s.begin(), s.end());
    for (size_t i = 1; i < s.size(); ++i)
        if (s[i] == s[i - 1]) return fail(PKV_ERR_INVALID_ARG, "slot %lld used twice", (long long)s[i]);
    return PKV_OK;
}

pkv_status pkv_validate_copy_pairs(const int32_t* h_pairs, int num_pairs, int num_blocks) {
    if (num_pairs < 0 || num_blocks < 0) return fail(PKV_ERR_INVALID_ARG, "negative size");
    if (num_pairs > 0 && !h_pairs) return fail(PKV_ERR_INVALID_ARG, "null pointer");
    std::vector<int32_t> src, dst;
    for (int p = 0; p < num_pairs; ++p) {
        const int32_t a = h_pairs[2 * p], b = h_pairs[2 * p + 1];
        if (a < 0 || a >= num_blocks || b < 0 || b >= num_blocks)
            return fail(PKV_ERR_INVALID_ARG, "pair %d (%d, %d) outside [0, %d)", p, a, b, num_blocks);
        if (a == b) continue;
        src.push_back(a);
        dst.push_back(b);
    }
    std::vector<int32_t> d = dst;
    std::sort(d.begin(), d.end());
    for (size_t i = 1; i < d.size(); ++i)
        if (d[i] == d[i - 1]) return fail(PKV_ERR_INVALID_ARG, "destination block %d repeats", d[i]);
    std::sort(src.begin(), src.end());
    for (int32_t b : d)
        if (std::binary_search(src.begin(), src.end(), b))
            return fail(PKV_ERR_INVALID_ARG, "block %d is both a source and a destination", b);
    return PKV_OK;
}

pkv_status pkv_device_error(int* code, int64_t* detail, pkv_stream_t stream) {
    if (!code || !detail) return fail(PKV_ERR_INVALID_ARG, "null pointer");
    DeviceError* err = device_error_word();
    if (!err) return fail(PKV_ERR_CUDA, "device error word unavailable");
    DeviceError h{};
    cudaError_t e = cudaMemcpyAsync(&h, err, sizeof h, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "device error read");
    *code = h.code;
    *detail = h.code ? h.detail : -1;
    if (h.code) {
        const DeviceError zero{};
        e = cudaMemcpyAsync(err, &zero, sizeof zero, cudaMemcpyHostToDevice, (cudaStream_t)stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
        if (e != cudaSuccess) return cuda_fail(e, "device error clear");
    }
    return PKV_OK;
}

pkv_status pkv_profile_start(int capacity) {
    if (capacity < 1) return fail(PKV_ERR_INVALID_ARG, "capacity < 1");
    Profiler& p = t_prof;
    for (cudaEvent_t e : p.ev) cudaEventDestroy(e);
    p = Profiler{};
    p.ev.resize(2 * (size_t)capacity);
    p.kind.resize((size_t)capacity);
    for (auto& e : p.ev) {
        cudaError_t r = cudaEventCreate(&e);
        if (r != cudaSuccess) {
            p.ev.clear();
            return cuda_fail(r, "profile event create");
        }
    }
    p.on = true;
    return PKV_OK;
}

pkv_status pkv_profile_stop(double* total_ms, int* launches, int* dropped) {
    if (!total_ms || !launches || !dropped) return fail(PKV_ERR_INVALID_ARG, "null output");
    Profiler& p = t_prof;
    if (!p.on) return fail(PKV_ERR_INVALID_ARG, "profiling was not started");
    for (int k = 0; k < PKV_KERNEL_KINDS; ++k) {
        total_ms[k] = 0.0;
        launches[k] = p.launches[k];
    }
    *dropped = p.dropped;
    pkv_status st = PKV_OK;
    for (int i = 0; i < p.used; ++i) {
        cudaError_t r = cudaEventSynchronize(p.ev[2 * i + 1]);
        float ms = 0.f;
        if (r == cudaSuccess) r = cudaEventElapsedTime(&ms, p.ev[2 * i], p.ev[2 * i + 1]);
        if (r != cudaSuccess) {
            st = cuda_fail(r, "profile event read");
            break;
        }
        total_ms[p.kind[i]] += ms;
    }
    for (cudaEvent_t e : p.ev) cudaEventDestroy(e);
    p = Profiler{};
    return st;
}

}  // extern "C"
