// Warp-level split-K paged attention (the per-warp loop of the warp-MMA kernel), shared by the
// split-K kernel (decode_mma.cu) and the tcgen05 tile kernel, whose CTAs also serve split-K items
// in mixed batches (prefill_tc.cu).
//
// What it computes is what decode.cu computes (blog.mckayzhao.com/?p=56, "PagedAttention：操作系统课本里
// 翻出来的灵感": every KV block of a request is found through its block table and read block by
// block; the result equals attention over contiguous storage), for items that pack up to 16
// (query row, query head) slots sharing one KV head: a query group of 8 or 16 heads, or several
// rows of one request (a speculative verify step: 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？,
// "V1 架构：推倒重来的勇气", a request submits k+1 tokens in one {request_id: num_tokens} step).
//
// Why tensor cores here: per 16-token block an item contracts a 16-slot x 128 Q tile with K and
// the 16-slot softmax weights with V -- two small dense products. On CUDA cores that costs about
// a thousand warp instructions per block for 8 slots, so the kernel is bound by instruction issue,
// not by HBM; as m16n8k16 MMAs (fp32 accumulation) it is 32 MMAs and 16 ldmatrix per block and the
// kernel streams K/V at memory speed. The MMAs run per warp: each warp stays an independent
// persistent worker with its own copy ring, as in decode.cu, and needs no tensor memory or
// CTA-wide synchronisation.
//
// Per warp and block: K and V of one (block, KV head) -- 16 rows of 128 elements -- arrive by one
// tensor-map TMA copy each (both 64-column halves through a 3-D view of the pool, 128-byte
// swizzle, so ldmatrix reads are free of bank conflicts; issuing the copies is a large share of a
// warp's time per block, so one copy per operand rather than one per half) into a ring of
// shared-memory stages tracked by mbarriers; the item's q rows come once per item, by plain bulk
// copies into the stage (or, with QREG, straight into registers). S = Q K^T as 16 MMAs (two 8-token n-tiles x 8 k-steps); the online
// softmax runs on the accumulator fragments in the log2 domain (a slot's scores sit in one lane
// quad); P, rounded to the input type, is reused in registers as the A operand of P V (16 MMAs
// over 8-column n-tiles, V fragments by transposing ldmatrix). Masking follows each slot's own
// causal limit; V rows past the item's last visible key are zeroed first (stale slots may hold
// anything). Items that cover part of a row write (unnormalised O, max, sum) partials for the
// log-sum-exp merge in decode.cu. Every wait is bounded, as in decode.cu.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"

namespace pkv {
namespace mma {

constexpr int kSlots = 16;                     // MMA M: (row, head) slots per item
constexpr int kHalf = kBlockSize * 128;        // one 64-column half of a 16-token K or V chunk (bytes)
constexpr int kKV = 4 * kHalf;                 // K half 0, K half 1, V half 0, V half 1
constexpr int kQ = kSlots * 256;               // an item's q rows (256 bytes each)
constexpr int kStage = kKV + kQ;               // 12 KiB, a multiple of the 1 KiB swizzle atom
constexpr int kFifo = 8;                       // items a warp's producer may run ahead (> NSTAGE)

// K or V of one KV block (16 pool rows from row y) in one copy, both 64-column halves, through a
// map made by encode_block_halves; with `hint`, under the L2 cache policy `policy`.
__device__ __forceinline__ void tma_load_block(void* dst, const CUtensorMap* map, int y, uint64_t* bar, bool hint,
                                               uint64_t policy) {
    if (hint)
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(
                smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(y), "r"(0), "r"(smem_u32(bar)), "l"(policy)
            : "memory");
    else
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
                smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(y), "r"(0), "r"(smem_u32(bar))
            : "memory");
}

// Byte offset, inside a 16-row chunk stored as two 64-column halves with the 128-byte swizzle, of
// the 16 bytes holding columns [8 * col8, 8 * col8 + 8) of row r (col8 in 0..15).
__device__ __forceinline__ uint32_t sw_off(int r, int col8) {
    return (uint32_t)((col8 >> 3) * kHalf + r * 128 + (((col8 & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

// d += A (16x16, row-major fragments) * B (16x8, column-major fragments), fp32 accumulation.
template <typename T>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (std::is_same<T, __half>::value) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
}

// Transpose of an 8 x 8 matrix of 16-bit elements held as one fragment (lane l: row l / 4, columns
// 2 (l % 4) and 2 (l % 4) + 1): afterwards lane l holds row l / 4 of the transpose.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// One warp's run over split-K work items. `first` is the warp's first item (none when it is
// >= num_items); every further item is base + a ticket taken from a.work[0], so warps that finish
// early take more items and the planner's longest-first order is served greedily. The producer
// fetches its next ticket when it starts an item, so the atomic's latency hides behind that item's
// blocks. wbase: NSTAGE stages of kStage bytes (1 KiB aligned); bars: NSTAGE mbarriers, initialised
// here (they must be idle); fifo: kFifo ints of shared memory (the items the producer has started,
// in order, for the consumer). On return every copy the warp issued has landed. Returns false when
// a bounded wait expired (recorded in the device error word; the warp's copies then drained).
// QREG (transposed form only): the stages hold K/V alone (kKV bytes each) and the item's q rows go
// from global memory straight into the B fragments -- for the next item as soon as the producer
// starts it, so the load's latency hides behind the blocks still ahead of the consumer.
template <typename T, int NSTAGE, bool T8, bool QREG = false>
__device__ __forceinline__ bool decode_warp(const DecodeArgs& a, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                            unsigned char* wbase, uint64_t* bars, volatile int* fifo, int first,
                                            int base) {
    static_assert(!QREG || T8, "q rows in registers: the transposed form only");
    constexpr int kSt = QREG ? kKV : kStage;   // bytes per stage
    const int lane = threadIdx.x & 31;
    if (lane == 0) {
        for (int s = 0; s < NSTAGE; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    if (first >= a.num_items) return true;
    const unsigned char* qp = static_cast<const unsigned char*>(a.q);
    uint64_t l2_policy = 0;   // evict first: every K/V block is read by one item
    if (a.evict_first) asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(l2_policy));
    const int g = lane >> 2;       // fragment row
    const int c4 = lane & 3;       // fragment column pair
    // QREG: item it's q rows as this lane's B fragments (slot g, words kk * 8 + c4 and + 4; zero
    // past the item's slots).
    auto load_q = [&](const DecodeItem& it, uint32_t (&qf)[8][2]) {
        const int nh = min(a.heads_per_item, a.group - it.head0);
        const bool vq = g < nh * it.num_rows;
        const int jr = vq ? g / nh : 0;
        const uint32_t* qg = reinterpret_cast<const uint32_t*>(
            qp + ((size_t)(it.row + jr) * a.num_q_heads + (size_t)it.kv_head * a.group + it.head0 + (vq ? g - jr * nh : 0)) * 256);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qf[kk][0] = vq ? __ldg(qg + kk * 8 + c4) : 0u;
            qf[kk][1] = vq ? __ldg(qg + kk * 8 + 4 + c4) : 0u;
        }
    };
    [[maybe_unused]] uint32_t qn[8][2];   // QREG: the q fragments of item qn_item, loaded ahead
    [[maybe_unused]] int qn_item = -1;

    // ---------------- producer (lane 0 issues; runs up to NSTAGE blocks ahead) ----------------
    int p_it = first;
    DecodeItem pi = load_item(a.items, p_it);
    int p_blk = pi.blk_begin;
    int p_base = p_blk;
    // Block ids of the producer's item, 32 at a time: p_ids holds those from p_base on (lane l:
    // block p_base + l), p_nxt the next 32, loaded a window ahead so that their latency hides.
    auto ids_at = [&](int from) {
        return (from + lane < pi.blk_end) ? __ldg(a.block_tables + (size_t)pi.req * a.max_blocks_per_seq + from + lane) : 0;
    };
    int p_ids = ids_at(p_blk);
    int p_nxt = ids_at(p_blk + 32);
    int ticket = 0;                      // lane 0: the next item's ticket, fetched ahead
    if (lane == 0) {
        ticket = atomicAdd(&a.work[0], 1);
        fifo[0] = p_it;
    }
    uint32_t pushed = 1;                 // items the producer has started (fifo entries written)
    bool p_done = false;
    uint32_t issued = 0;

    auto issue = [&](int stage) {
        const int id_raw = __shfl_sync(FULL_MASK, p_ids, p_blk - p_base);
        if (lane == 0) {
            int id = id_raw;
            if (id < 0 || id >= a.num_blocks) {
                record_error(a.err, 6 /*PKV_ERR_DEVICE_RANGE*/, (long long)pi.req * a.max_blocks_per_seq + p_blk);
                id = 0;
            }
            unsigned char* st = wbase + stage * kSt;
            const bool first = !QREG && (p_blk == pi.blk_begin);
            const int nh = min(a.heads_per_item, a.group - pi.head0);
            const uint32_t qrow = (uint32_t)(nh * 256);
            const uint32_t qbytes = first ? qrow * (uint32_t)pi.num_rows : 0u;
            mbar_arrive_expect_tx(&bars[stage], (uint32_t)kKV + qbytes);
            const int y = (id * a.num_kv_heads + pi.kv_head) * kBlockSize;  // first pool row of the chunk
            tma_load_block(st, tm_k, y, &bars[stage], a.evict_first, l2_policy);
            tma_load_block(st + 2 * kHalf, tm_v, y, &bars[stage], a.evict_first, l2_policy);
            if (first) {
                for (int j = 0; j < pi.num_rows; ++j) {
                    const size_t qoff =
                        ((size_t)(pi.row + j) * a.num_q_heads + (size_t)pi.kv_head * a.group + pi.head0) * 256;
                    bulk_g2s(st + kKV + j * qrow, qp + qoff, qrow, &bars[stage]);
                }
            }
        }
        ++issued;
        ++p_blk;
        if (p_blk == pi.blk_end) {
            p_it = base + __shfl_sync(FULL_MASK, ticket, 0);
            if (p_it < a.num_items) {
                pi = load_item(a.items, p_it);
                p_blk = pi.blk_begin;
                p_base = p_blk;
                p_ids = ids_at(p_blk);
                p_nxt = ids_at(p_blk + 32);
                if constexpr (QREG) {
                    load_q(pi, qn);
                    qn_item = p_it;
                }
                if (lane == 0) {
                    fifo[pushed % kFifo] = p_it;
                    ticket = atomicAdd(&a.work[0], 1);
                }
                ++pushed;
            } else {
                p_done = true;
            }
        } else if (p_blk - p_base == 32) {
            p_base = p_blk;
            p_ids = p_nxt;
            p_nxt = ids_at(p_blk + 32);
        }
    };

    for (int s = 0; s < NSTAGE && !p_done; ++s) issue(s);

    // ---------------- consumer (the whole warp) ----------------
    int c_it = first;
    uint32_t popped = 0;                 // fifo position of the item being consumed
    DecodeItem ci = load_item(a.items, c_it);
    int c_blk = ci.blk_begin;
    uint32_t consumed = 0;

    const int mi = lane >> 3;      // ldmatrix: which 8x8 matrix this lane addresses
    const int mr = lane & 7;       //           and which of its rows

    if constexpr (T8) {
        // Items of at most 8 (row, head) slots, transposed: S^T = K Q^T (16 tokens x 8 slots, K as the
        // A operand, q rows as the B operand) and O^T = V^T P^T (128 x 8, V as the A operand through
        // transposing ldmatrix, P^T as the B operand moved into place by movmatrix): 16 MMAs per block
        // instead of 32. Lane (g, c4) holds tokens g and g + 8 of slots 2c4 and 2c4 + 1; a slot's
        // reductions over tokens run across the 8 lanes that share its c4.
        uint32_t qb[8][2];         // Q^T as B fragments, one pair per 16-column k-step
        float ot[8][4];            // O^T accumulators, one per 16-row (head_dim) m-tile
        float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;
        int lima = 0, limb = 0, nh = 1, ns = 0;
        const int sa = 2 * c4, sb = 2 * c4 + 1;   // this lane's slots
        bool zeroed = false;                      // V rows of the current stage were zeroed

        while (true) {
            const int stage = consumed % NSTAGE;
            const uint32_t parity = (consumed / NSTAGE) & 1u;
            if (!mbar_wait(&bars[stage], parity)) {
                if (lane == 0) record_error(a.err, 5 /*PKV_ERR_DEVICE_TIMEOUT*/, c_it);
                for (uint32_t k = consumed; k < issued; ++k) (void)mbar_wait(&bars[k % NSTAGE], (k / NSTAGE) & 1u);
                return false;
            }
            unsigned char* st = wbase + stage * kSt;
            const uint32_t kb = smem_u32(st);
            const uint32_t vb = kb + 2 * kHalf;

            if (c_blk == ci.blk_begin) {
                nh = min(a.heads_per_item, a.group - ci.head0);
                ns = nh * ci.num_rows;
                if constexpr (QREG) {
                    if (qn_item == c_it) {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            qb[kk][0] = qn[kk][0];
                            qb[kk][1] = qn[kk][1];
                        }
                    } else {
                        load_q(ci, qb);
                    }
                } else {
                    const uint32_t* qs = reinterpret_cast<const uint32_t*>(st + kKV);
                    const bool vq = g < ns;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        qb[kk][0] = vq ? qs[g * 64 + kk * 8 + c4] : 0u;
                        qb[kk][1] = vq ? qs[g * 64 + kk * 8 + 4 + c4] : 0u;
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) ot[j][0] = ot[j][1] = ot[j][2] = ot[j][3] = 0.f;
                ma = mb = -INFINITY;
                la = lb = 0.f;
                lima = sa < ns ? ci.limit + sa / nh : 0;   // keys visible to slot sa (row sa / nh of the item)
                limb = sb < ns ? ci.limit + sb / nh : 0;
            }

            // ---- S^T = K Q^T, accumulated in two chains (even / odd k-steps) ----
            float s[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t ka[4];
                ldsm_x4(kb + sw_off(((mi & 1) << 3) + mr, 2 * kk + (mi >> 1)), ka[0], ka[1], ka[2], ka[3]);
                mma16816<T>((kk & 1) ? s2 : s, ka, qb[kk][0], qb[kk][1]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) s[e] += s2[e];

            // ---- online softmax per slot (log2 domain), masked by each slot's own limit ----
            const int t0 = c_blk * kBlockSize + g;
            s[0] = t0 < lima ? s[0] * a.scale_log2 : -INFINITY;
            s[1] = t0 < limb ? s[1] * a.scale_log2 : -INFINITY;
            s[2] = t0 + 8 < lima ? s[2] * a.scale_log2 : -INFINITY;
            s[3] = t0 + 8 < limb ? s[3] * a.scale_log2 : -INFINITY;
            float mxa = fmaxf(s[0], s[2]), mxb = fmaxf(s[1], s[3]);
#pragma unroll
            for (int sh = 4; sh < 32; sh <<= 1) {
                mxa = fmaxf(mxa, __shfl_xor_sync(FULL_MASK, mxa, sh));
                mxb = fmaxf(mxb, __shfl_xor_sync(FULL_MASK, mxb, sh));
            }
            const float mna = fmaxf(ma, mxa), mnb = fmaxf(mb, mxb);
            // A slot may see no key of this block: subtracting 0 instead of -inf keeps alpha and p at
            // 0 rather than NaN.
            const float mua = mna == -INFINITY ? 0.f : mna;
            const float mub = mnb == -INFINITY ? 0.f : mnb;
            const float ala = fast_exp2(ma - mua), alb = fast_exp2(mb - mub);
            ma = mna;
            mb = mnb;
            // P^T rounded to T, as two 8 x 8 fragments (tokens 0-7 and 8-15; rows = tokens, columns =
            // slots). The row sums add the weights as rounded; each lane keeps its own part, the 8
            // lanes of a slot are added when the item ends.
            const uint32_t w0 = pack2<T>(fast_exp2(s[0] - mua), fast_exp2(s[1] - mub));
            const uint32_t w1 = pack2<T>(fast_exp2(s[2] - mua), fast_exp2(s[3] - mub));
            const float2 r0 = unpack2<T>(w0), r1 = unpack2<T>(w1);
            la = la * ala + (r0.x + r1.x);
            lb = lb * alb + (r0.y + r1.y);
            if (ala != 1.f || alb != 1.f) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    ot[j][0] *= ala;
                    ot[j][1] *= alb;
                    ot[j][2] *= ala;
                    ot[j][3] *= alb;
                }
            }

            // ---- V rows past the last visible key may hold anything: zero them ----
            const int vis = ci.limit + ci.num_rows - 1 - c_blk * kBlockSize;
            if (vis < kBlockSize) {
                const int first_row = vis > 0 ? vis : 0;
                for (int idx = lane; idx < (kBlockSize - first_row) * 16; idx += 32) {
                    const int r = first_row + (idx >> 4);
                    *reinterpret_cast<uint4*>(st + 2 * kHalf + sw_off(r, idx & 15)) = make_uint4(0u, 0u, 0u, 0u);
                }
                __syncwarp();
                zeroed = true;
            }

            // ---- O^T += V^T P^T: eight 16-row m-tiles of head_dim ----
            const uint32_t pb0 = movmatrix_trans(w0), pb1 = movmatrix_trans(w1);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                uint32_t va[4];
                ldsm_x4_t(vb + sw_off(((mi >> 1) << 3) + mr, 2 * mt + (mi & 1)), va[0], va[1], va[2], va[3]);
                mma16816<T>(ot[mt], va, pb0, pb1);
            }
            __syncwarp();
            ++consumed;

            // Refill this stage with the producer's next block. The warp's reads of the stage are
            // complete (their values are in registers); generic writes to it (zeroed V rows) are
            // ordered before the copy's writes by a proxy fence.
            if (!p_done) {
                if (zeroed) fence_proxy_async_smem();
                issue(stage);
            }
            zeroed = false;

            if (c_blk + 1 == ci.blk_end) {
                // ---- item done: normalised output, or the chunk's partial ----
#pragma unroll
                for (int sh = 4; sh < 32; sh <<= 1) {
                    la += __shfl_xor_sync(FULL_MASK, la, sh);
                    lb += __shfl_xor_sync(FULL_MASK, lb, sh);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int slot = h ? sb : sa;
                    if (slot < ns) {
                        const int jr = slot / nh;
                        const float m = h ? mb : ma, l = h ? lb : la;
                        if (ci.partial < 0) {
                            const float inv = 1.f / l;
                            T* orow = static_cast<T*>(a.out) +
                                      ((size_t)(ci.row + jr) * a.num_q_heads + (size_t)ci.kv_head * a.group + ci.head0 +
                                       (slot - jr * nh)) * 128;
#pragma unroll
                            for (int mt = 0; mt < 8; ++mt) {
                                orow[16 * mt + g] = T(ot[mt][h] * inv);
                                orow[16 * mt + 8 + g] = T(ot[mt][2 + h] * inv);
                            }
                        } else {
                            float* po = a.part_o + ((size_t)ci.partial * a.part_stride + slot) * 128;
#pragma unroll
                            for (int mt = 0; mt < 8; ++mt) {
                                po[16 * mt + g] = ot[mt][h];
                                po[16 * mt + 8 + g] = ot[mt][2 + h];
                            }
                            if (g == 0) {
                                float* pm = a.part_ml + ((size_t)ci.partial * a.part_stride + slot) * 2;
                                pm[0] = m;
                                pm[1] = l;
                            }
                        }
                    }
                }
                // The next item is the producer's next one; none was started: the work is done.
                if (++popped == pushed) break;
                __syncwarp();
                c_it = fifo[popped % kFifo];
                ci = load_item(a.items, c_it);
                c_blk = ci.blk_begin;
            } else {
                ++c_blk;
            }
        }
    } else {
        uint32_t qa[8][4];             // Q as A fragments, one set per 16-column k-step
        float o[16][4];                // O accumulators, one per 8-column n-tile
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        int lim0 = 0, lim1 = 0, nh = 1, ns = 0;
        bool zeroed = false;                      // V rows of the current stage were zeroed

        while (true) {
            const int stage = consumed % NSTAGE;
            const uint32_t parity = (consumed / NSTAGE) & 1u;
            if (!mbar_wait(&bars[stage], parity)) {
                if (lane == 0) record_error(a.err, 5 /*PKV_ERR_DEVICE_TIMEOUT*/, c_it);
                for (uint32_t k = consumed; k < issued; ++k) (void)mbar_wait(&bars[k % NSTAGE], (k / NSTAGE) & 1u);
                return false;
            }
            unsigned char* st = wbase + stage * kSt;
            const uint32_t kb = smem_u32(st);
            const uint32_t vb = kb + 2 * kHalf;

            if (c_blk == ci.blk_begin) {
                nh = min(a.heads_per_item, a.group - ci.head0);
                ns = nh * ci.num_rows;
                const uint32_t* qs = reinterpret_cast<const uint32_t*>(st + kKV);
                const bool v0 = g < ns, v1 = g + 8 < ns;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    qa[kk][0] = v0 ? qs[g * 64 + kk * 8 + c4] : 0u;
                    qa[kk][1] = v1 ? qs[(g + 8) * 64 + kk * 8 + c4] : 0u;
                    qa[kk][2] = v0 ? qs[g * 64 + kk * 8 + 4 + c4] : 0u;
                    qa[kk][3] = v1 ? qs[(g + 8) * 64 + kk * 8 + 4 + c4] : 0u;
                }
#pragma unroll
                for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
                m0 = m1 = -INFINITY;
                l0 = l1 = 0.f;
                lim0 = v0 ? ci.limit + g / nh : 0;         // keys visible to slot g (row g / nh of the item)
                lim1 = v1 ? ci.limit + (g + 8) / nh : 0;
            }

            // ---- S = Q K^T: two 8-token n-tiles, each accumulated in two chains (even / odd k-steps)
            // so that the dependent MMAs per chain are four, not eight ----
            float s[2][4], s2[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
                s2[j][0] = s2[j][1] = s2[j][2] = s2[j][3] = 0.f;
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kb + sw_off(((mi >> 1) << 3) + mr, 2 * kk + (mi & 1)), b0, b1, b2, b3);
                mma16816<T>((kk & 1) ? s2[0] : s[0], qa[kk], b0, b1);
                mma16816<T>((kk & 1) ? s2[1] : s[1], qa[kk], b2, b3);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[j][e] += s2[j][e];

            // ---- online softmax per slot (log2 domain), masked by each slot's own limit ----
            const int t0 = c_blk * kBlockSize + 2 * c4;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int t = t0 + 8 * j;
                s[j][0] = t < lim0 ? s[j][0] * a.scale_log2 : -INFINITY;
                s[j][1] = t + 1 < lim0 ? s[j][1] * a.scale_log2 : -INFINITY;
                s[j][2] = t < lim1 ? s[j][2] * a.scale_log2 : -INFINITY;
                s[j][3] = t + 1 < lim1 ? s[j][3] * a.scale_log2 : -INFINITY;
            }
            float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
            float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
            mx0 = fmaxf(mx0, __shfl_xor_sync(FULL_MASK, mx0, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(FULL_MASK, mx1, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(FULL_MASK, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(FULL_MASK, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            // A slot may see no key of this block (a chunk past an earlier row's limit, a padded slot):
            // subtracting 0 instead of -inf keeps alpha and p at 0 rather than NaN.
            const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
            const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
            const float al0 = fast_exp2(m0 - mu0), al1 = fast_exp2(m1 - mu1);
            m0 = mn0;
            m1 = mn1;
            float p[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                p[j][0] = fast_exp2(s[j][0] - mu0);
                p[j][1] = fast_exp2(s[j][1] - mu0);
                p[j][2] = fast_exp2(s[j][2] - mu1);
                p[j][3] = fast_exp2(s[j][3] - mu1);
            }
            // P as the A operand of P V: rows g / g + 8, token columns 2c, 2c+1 (+8). The row sums
            // add the weights as rounded, so that they match what P V accumulates.
            const uint32_t pa[4] = {pack2<T>(p[0][0], p[0][1]), pack2<T>(p[0][2], p[0][3]), pack2<T>(p[1][0], p[1][1]),
                                    pack2<T>(p[1][2], p[1][3])};
            // Each lane keeps the sum of its own weights; the quad's four partial sums are added once,
            // when the item ends (the rescale factors are the same on all four lanes of a slot).
            const float2 r00 = unpack2<T>(pa[0]), r01 = unpack2<T>(pa[1]), r10 = unpack2<T>(pa[2]), r11 = unpack2<T>(pa[3]);
            l0 = l0 * al0 + ((r00.x + r00.y) + (r10.x + r10.y));
            l1 = l1 * al1 + ((r01.x + r01.y) + (r11.x + r11.y));
            if (al0 != 1.f || al1 != 1.f) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    o[j][0] *= al0;
                    o[j][1] *= al0;
                    o[j][2] *= al1;
                    o[j][3] *= al1;
                }
            }

            // ---- V rows past the last visible key may hold anything: zero them ----
            const int vis = ci.limit + ci.num_rows - 1 - c_blk * kBlockSize;
            if (vis < kBlockSize) {
                const int first = vis > 0 ? vis : 0;
                for (int idx = lane; idx < (kBlockSize - first) * 16; idx += 32) {
                    const int r = first + (idx >> 4);
                    *reinterpret_cast<uint4*>(st + 2 * kHalf + sw_off(r, idx & 15)) = make_uint4(0u, 0u, 0u, 0u);
                }
                __syncwarp();
                zeroed = true;
            }

            // ---- O += P V: sixteen 8-column n-tiles ----
#pragma unroll
            for (int jp = 0; jp < 8; ++jp) {
                uint32_t v0, v1, v2, v3;
                ldsm_x4_t(vb + sw_off(((mi & 1) << 3) + mr, 2 * jp + (mi >> 1)), v0, v1, v2, v3);
                mma16816<T>(o[2 * jp], pa, v0, v1);
                mma16816<T>(o[2 * jp + 1], pa, v2, v3);
            }
            __syncwarp();
            ++consumed;

            // Refill this stage with the producer's next block. The warp's reads of the stage are
            // complete (their values are in registers); generic writes to it (zeroed V rows) are
            // ordered before the copy's writes by a proxy fence.
            if (!p_done) {
                if (zeroed) fence_proxy_async_smem();
                issue(stage);
            }
            zeroed = false;

            if (c_blk + 1 == ci.blk_end) {
                // ---- item done: normalised output, or the chunk's partial ----
                l0 += __shfl_xor_sync(FULL_MASK, l0, 1);
                l1 += __shfl_xor_sync(FULL_MASK, l1, 1);
                l0 += __shfl_xor_sync(FULL_MASK, l0, 2);
                l1 += __shfl_xor_sync(FULL_MASK, l1, 2);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int slot = g + 8 * h;
                    if (slot < ns) {
                        const int jr = slot / nh;
                        const float m = h ? m1 : m0, l = h ? l1 : l0;
                        if (ci.partial < 0) {
                            const float inv = 1.f / l;
                            T* orow = static_cast<T*>(a.out) +
                                      ((size_t)(ci.row + jr) * a.num_q_heads + (size_t)ci.kv_head * a.group + ci.head0 +
                                       (slot - jr * nh)) * 128;
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                *reinterpret_cast<uint32_t*>(orow + 8 * j + 2 * c4) =
                                    pack2<T>(o[j][2 * h] * inv, o[j][2 * h + 1] * inv);
                        } else {
                            float* po = a.part_o + ((size_t)ci.partial * a.part_stride + slot) * 128;
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                *reinterpret_cast<float2*>(po + 8 * j + 2 * c4) = make_float2(o[j][2 * h], o[j][2 * h + 1]);
                            if (c4 == 0) {
                                float* pm = a.part_ml + ((size_t)ci.partial * a.part_stride + slot) * 2;
                                pm[0] = m;
                                pm[1] = l;
                            }
                        }
                    }
                }
                // The next item is the producer's next one; none was started: the work is done.
                if (++popped == pushed) break;
                __syncwarp();
                c_it = fifo[popped % kFifo];
                ci = load_item(a.items, c_it);
                c_blk = ci.blk_begin;
            } else {
                ++c_blk;
            }
        }
    }
    return true;
}

}  // namespace mma
}  // namespace pkv
