// CUDA-core paged attention: split-K ("flash-decoding") over KV blocks with GQA packing, plus the
// log-sum-exp merge of chunk partials.
//
// What it computes follows blog.mckayzhao.com/?p=56, "PagedAttention：操作系统课本里翻出来的灵感":
// each KV block of a request is found through its block table and K and V are read block by block;
// the result equals attention over contiguous storage. Rows of any length are served: decode rows,
// and the rows of multi-token requests that the tcgen05 path does not take -- a speculative verify
// step, where a request submits its k draft tokens plus one (一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？,
// "V1 架构：推倒重来的勇气": the step is a {request_id: num_tokens} dictionary), or rows of fp32 /
// other shapes -- each row with its causal limit.
//
// Design (B200): every warp is an independent persistent worker. It walks a static round-robin
// share of the planner's work items (consecutive rows of a request x up to 8 query heads of a KV
// head -- at most 8 (row, head) slots that share every K/V block -- and a block range) and streams
// each (block, KV head) K and V chunk -- a contiguous 16*D run in the pool -- with one
// cp.async.bulk (TMA engine, no tensor map) into a private ring of shared-memory stages,
// completion tracked by an mbarrier per stage. The ring runs ahead across item boundaries, so
// the copy engine is never idle between items. Each lane owns one 16-byte column chunk of a K/V
// row: QK partial dots are fp32 FMAs on registers, reduced across the row's lanes with a
// butterfly reduce-scatter of warp shuffles; the online softmax is per query head in fp32 (log2
// domain, ex2.approx); P*V accumulates in fp32 registers. Items covering part of a row write
// (unnormalised output, max, sum) partials; merge_kernel combines them by log-sum-exp.
#include <cstdlib>
#include <type_traits>

#include "common.cuh"

namespace pkv {
namespace {

constexpr int log2i(int x) { return x <= 1 ? 0 : 1 + log2i(x / 2); }
constexpr int round16(int x) { return (x + 15) / 16 * 16; }

template <typename T, int D, int GP, int NSTAGE>
struct Dec {
    static constexpr int EB = sizeof(T);
    static constexpr int ROW = D * EB;                 // bytes of one K/V row
    static constexpr int CPR = ROW / 16;               // 16-byte chunks per row = lanes per row
    static constexpr int LOG_CPR = log2i(CPR);
    static constexpr int TPP = 32 / CPR;               // rows (tokens) handled per warp pass
    static constexpr int EPC = 16 / EB;                // elements per chunk
    static constexpr int E2 = EPC / 2;                 // element pairs per chunk
    static constexpr int PASSES = kBlockSize / TPP;    // passes per 16-token block
    static constexpr int LOG_PASSES = log2i(PASSES);
    static constexpr int NV = GP * PASSES;             // partial dots per lane per block
    static constexpr int LOG_NV = log2i(NV);
    static constexpr int SPLIT = LOG_CPR < LOG_NV ? LOG_CPR : LOG_NV;  // reduce-scatter rounds
    static constexpr int NOWN = NV >> SPLIT;           // full dots owned per lane afterwards
    static constexpr int BLK = kBlockSize * ROW;       // bytes of one (block, head) K or V chunk
    static constexpr int QB = GP * ROW;                // bytes of an item's query rows
    static constexpr int STAGE = 2 * BLK + QB;
    static constexpr int STAGES = NSTAGE;
    static constexpr int P_FLOATS = GP * TPP * PASSES; // softmax weights of one block
    static constexpr int SCR = round16(P_FLOATS * 4 + GP * 4 + GP * 8);
    static constexpr int WARP_SMEM = STAGES * STAGE + SCR + round16(STAGES * 8);
    static_assert(CPR >= 8 && CPR <= 32, "K/V rows of 128..512 bytes");
    static_assert(GP <= CPR, "query group larger than the lanes of a row");
    static_assert(PASSES % 4 == 0, "weights are read four at a time");
};

constexpr int kDecodeWarps = 2;  // independent warps per CTA

// Default ring depth: three stages for small groups (pure streaming), two for large groups
// (more resident warps matter more there, the kernel being issue-bound).
template <int GP>
constexpr int default_stages() { return GP >= 4 ? 2 : 3; }

template <typename T, int D, int GP, int NSTAGE>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_kernel(const DecodeArgs a) {
    using C = Dec<T, D, GP, NSTAGE>;
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    unsigned char* wbase = smem + warp * C::WARP_SMEM;
    float* p_s = reinterpret_cast<float*>(wbase + C::STAGES * C::STAGE);
    float* alpha_s = p_s + C::P_FLOATS;
    float* ml_s = alpha_s + GP;
    uint64_t* bars = reinterpret_cast<uint64_t*>(wbase + C::STAGES * C::STAGE + C::SCR);

    if (lane == 0) {
        for (int s = 0; s < C::STAGES; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    griddep_wait();

    const int W = gridDim.x * kDecodeWarps;
    const int gw = blockIdx.x * kDecodeWarps + warp;
    if (gw >= a.num_items) return;

    const int sub = lane >> C::LOG_CPR;       // token slot inside a pass
    const int chunk = lane & (C::CPR - 1);    // 16-byte column chunk of a row
    const size_t head_stride = (size_t)C::BLK;
    const unsigned char* kp = static_cast<const unsigned char*>(a.k_pool);
    const unsigned char* vp = static_cast<const unsigned char*>(a.v_pool);
    const unsigned char* qp = static_cast<const unsigned char*>(a.q);

    // ---------------- producer (runs up to STAGES blocks ahead of the consumer) ----------------
    int p_it = gw;
    DecodeItem pi = load_item(a.items, p_it);
    int p_blk = pi.blk_begin;
    int p_base = p_blk;
    int p_ids = (p_blk + lane < pi.blk_end) ? __ldg(a.block_tables + (size_t)pi.req * a.max_blocks_per_seq + p_blk + lane) : 0;
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
            unsigned char* st = wbase + stage * C::STAGE;
            const bool first = (p_blk == pi.blk_begin);
            const int nh = min(a.heads_per_item, a.group - pi.head0);
            const uint32_t qrow = (uint32_t)(nh * C::ROW);  // one row's heads, contiguous in q
            const uint32_t qbytes = first ? qrow * (uint32_t)pi.num_rows : 0u;
            mbar_arrive_expect_tx(&bars[stage], 2u * C::BLK + qbytes);
            const size_t off = ((size_t)id * a.num_kv_heads + pi.kv_head) * head_stride;
            bulk_g2s(st, kp + off, C::BLK, &bars[stage]);
            bulk_g2s(st + C::BLK, vp + off, C::BLK, &bars[stage]);
            if (first) {
                // The item's (row, head) slots land contiguously: slot j * nh + h at (j * nh + h) * ROW.
                for (int j = 0; j < pi.num_rows; ++j) {
                    const size_t qoff =
                        ((size_t)(pi.row + j) * a.num_q_heads + (size_t)pi.kv_head * a.group + pi.head0) * C::ROW;
                    bulk_g2s(st + 2 * C::BLK + j * qrow, qp + qoff, qrow, &bars[stage]);
                }
            }
        }
        ++issued;
        // advance to the next (item, block)
        ++p_blk;
        if (p_blk == pi.blk_end) {
            p_it += W;
            if (p_it < a.num_items) {
                pi = load_item(a.items, p_it);
                p_blk = pi.blk_begin;
                p_base = p_blk;
                p_ids = (p_blk + lane < pi.blk_end)
                            ? __ldg(a.block_tables + (size_t)pi.req * a.max_blocks_per_seq + p_blk + lane) : 0;
            } else {
                p_done = true;
            }
        } else if (p_blk - p_base == 32) {
            p_base = p_blk;
            p_ids = (p_blk + lane < pi.blk_end)
                        ? __ldg(a.block_tables + (size_t)pi.req * a.max_blocks_per_seq + p_blk + lane) : 0;
        }
    };

    for (int s = 0; s < C::STAGES && !p_done; ++s) issue(s);

    // ---------------- consumer ----------------
    int c_it = gw;
    DecodeItem ci = load_item(a.items, c_it);
    int c_blk = ci.blk_begin;
    uint32_t consumed = 0;

    // Dots are indexed x = head * PASSES + pass. The butterfly reduce-scatter halves the index range
    // each round, the lane keeping the half selected by its own lane bit. Storing slot s as logical
    // index s ^ M (M = the lane's kept bits) puts the kept half always in the low slots, so a round
    // is one shuffle and one add per value. M is applied by loading q heads in permuted order and by
    // permuting which token each pass reads.
    int M = 0;
#pragma unroll
    for (int r = 0; r < C::SPLIT; ++r)
        if (lane & (C::CPR >> (r + 1))) M |= C::NV >> (r + 1);
    const int g_own = M / C::PASSES;           // head whose scores this lane owns after the rounds
    const int i_own0 = M % C::PASSES;          // first owned pass
    const int gm = M / C::PASSES;              // head-slot permutation
    const int im = M % C::PASSES;              // pass permutation

    float2 q2[GP][C::E2];                      // q (scaled, log2 domain), slots permuted by gm
    float2 acc2[GP][C::E2];                    // output accumulator, logical slot order
    float m_own = -INFINITY, l_own = 0.f;
    int own_limit = 0;                         // keys visible to the slot this lane owns

    while (true) {
        const int stage = consumed % C::STAGES;
        const uint32_t parity = (consumed / C::STAGES) & 1u;
        if (!mbar_wait(&bars[stage], parity)) {
            if (lane == 0) record_error(a.err, 5 /*PKV_ERR_DEVICE_TIMEOUT*/, c_it);
            // Drain the copies still in flight (bounded) before leaving.
            for (uint32_t k = consumed; k < issued; ++k)
                (void)mbar_wait(&bars[k % C::STAGES], (k / C::STAGES) & 1u);
            return;
        }
        const unsigned char* st = wbase + stage * C::STAGE;
        const unsigned char* Ks = st;
        const unsigned char* Vs = st + C::BLK;
        const int nh = min(a.heads_per_item, a.group - ci.head0);
        const int ns = nh * ci.num_rows;          // (row, head) slots of the item

        if (c_blk == ci.blk_begin) {
            own_limit = ci.limit + (g_own < ns ? g_own / nh : 0);
#pragma unroll
            for (int gs = 0; gs < GP; ++gs) {
                const int g = gs ^ gm;
                if (g < ns) {
                    float f[C::EPC];
                    Chunk<T>::unpack(lds128(st + 2 * C::BLK + g * C::ROW + chunk * 16), f);
#pragma unroll
                    for (int e = 0; e < C::E2; ++e) q2[gs][e] = make_float2(f[2 * e] * a.scale_log2, f[2 * e + 1] * a.scale_log2);
                } else {
#pragma unroll
                    for (int e = 0; e < C::E2; ++e) q2[gs][e] = make_float2(0.f, 0.f);
                }
#pragma unroll
                for (int e = 0; e < C::E2; ++e) acc2[gs][e] = make_float2(0.f, 0.f);
            }
            m_own = -INFINITY;
            l_own = 0.f;
        }
        // Keys of this block visible to the item's last row (V rows past it are zeroed) and to the
        // slot this lane owns (its scores past it are masked).
        const int valid = min(kBlockSize, ci.limit + ci.num_rows - 1 - c_blk * kBlockSize);
        const int valid_own = own_limit - c_blk * kBlockSize;

        // ---- QK: partial dots of this lane's chunk for every (head slot, pass slot) ----
        float dots[C::NV];
#pragma unroll
        for (int is = 0; is < C::PASSES; ++is) {
            float k[C::EPC];
            Chunk<T>::unpack(lds128(Ks + ((is ^ im) * C::TPP + sub) * C::ROW + chunk * 16), k);
#pragma unroll
            for (int gs = 0; gs < GP; ++gs) {
                float2 d2 = __fmul2_rn(q2[gs][0], make_float2(k[0], k[1]));
#pragma unroll
                for (int e = 1; e < C::E2; ++e) d2 = __ffma2_rn(q2[gs][e], make_float2(k[2 * e], k[2 * e + 1]), d2);
                dots[gs * C::PASSES + is] = d2.x + d2.y;
            }
        }
        // ---- reduce-scatter across the CPR lanes of a row (kept half always in the low slots) ----
#pragma unroll
        for (int r = 0; r < C::LOG_CPR; ++r) {
            const int o = C::CPR >> (r + 1);
            if (r < C::LOG_NV) {
                const int h = C::NV >> (r + 1);
#pragma unroll
                for (int k = 0; k < h; ++k) dots[k] += __shfl_xor_sync(FULL_MASK, dots[k + h], o);
            } else {
                dots[0] += __shfl_xor_sync(FULL_MASK, dots[0], o);
            }
        }
        // ---- online softmax for head g_own over this block's tokens ----
        float mb = -INFINITY;
#pragma unroll
        for (int k = 0; k < C::NOWN; ++k) {
            const int t = (i_own0 + k) * C::TPP + sub;
            if (t >= valid_own) dots[k] = -INFINITY;
            mb = fmaxf(mb, dots[k]);
        }
#pragma unroll
        for (int r = 0; r < C::SPLIT; ++r)
            if (C::LOG_NV - 1 - r < C::LOG_PASSES) mb = fmaxf(mb, __shfl_xor_sync(FULL_MASK, mb, C::CPR >> (r + 1)));
#pragma unroll
        for (int o = C::CPR; o < 32; o <<= 1) mb = fmaxf(mb, __shfl_xor_sync(FULL_MASK, mb, o));
        const float m_new = fmaxf(m_own, mb);
        // A slot can see no key of a chunk that starts past its row's limit (rows of one item have
        // different limits): with m_new = -inf, subtract 0 so that alpha and p come out 0, not NaN.
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = fast_exp2(m_own - m_use);
        float ps = 0.f;
        float* prow = p_s + (g_own * C::TPP + sub) * C::PASSES;
#pragma unroll
        for (int k = 0; k < C::NOWN; ++k) {
            const float p = fast_exp2(dots[k] - m_use);
            ps += p;
            prow[i_own0 + k] = p;
        }
#pragma unroll
        for (int r = 0; r < C::SPLIT; ++r)
            if (C::LOG_NV - 1 - r < C::LOG_PASSES) ps += __shfl_xor_sync(FULL_MASK, ps, C::CPR >> (r + 1));
#pragma unroll
        for (int o = C::CPR; o < 32; o <<= 1) ps += __shfl_xor_sync(FULL_MASK, ps, o);
        l_own = l_own * alpha + ps;
        m_own = m_new;
        alpha_s[g_own] = alpha;
        __syncwarp();

        // ---- P*V (logical head order) ----
        bool rescale = false;
#pragma unroll
        for (int g = 0; g < GP; ++g) rescale |= alpha_s[g] != 1.f;
        if (rescale) {  // warp-uniform: every lane reads the same alphas
#pragma unroll
            for (int g = 0; g < GP; ++g) {
                const float al = alpha_s[g];
#pragma unroll
                for (int e = 0; e < C::E2; ++e) acc2[g][e] = __fmul2_rn(acc2[g][e], make_float2(al, al));
            }
        }
#pragma unroll
        for (int i4 = 0; i4 < C::PASSES; i4 += 4) {
            float4 pw[GP];
#pragma unroll
            for (int g = 0; g < GP; ++g)
                pw[g] = *reinterpret_cast<const float4*>(p_s + (g * C::TPP + sub) * C::PASSES + i4);
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                const int t = (i4 + ii) * C::TPP + sub;
                float v[C::EPC];
                Chunk<T>::unpack(lds128(Vs + t * C::ROW + chunk * 16), v);
                if (t >= valid) {
#pragma unroll
                    for (int e = 0; e < C::EPC; ++e) v[e] = 0.f;  // slots past the context may hold anything
                }
#pragma unroll
                for (int g = 0; g < GP; ++g) {
                    const float p = ii == 0 ? pw[g].x : ii == 1 ? pw[g].y : ii == 2 ? pw[g].z : pw[g].w;
                    const float2 p2 = make_float2(p, p);
#pragma unroll
                    for (int e = 0; e < C::E2; ++e) acc2[g][e] = __ffma2_rn(p2, make_float2(v[2 * e], v[2 * e + 1]), acc2[g][e]);
                }
            }
        }
        __syncwarp();
        ++consumed;

        // Refill this stage with the producer's next block.
        if (!p_done) {
            fence_proxy_async_smem();
            issue(stage);
        }

        if (c_blk + 1 == ci.blk_end) {
            // ---- item done: combine token slots, then write the output or the partial ----
#pragma unroll
            for (int o = C::CPR; o < 32; o <<= 1)
#pragma unroll
                for (int g = 0; g < GP; ++g)
#pragma unroll
                    for (int e = 0; e < C::E2; ++e) {
                        acc2[g][e].x += __shfl_xor_sync(FULL_MASK, acc2[g][e].x, o);
                        acc2[g][e].y += __shfl_xor_sync(FULL_MASK, acc2[g][e].y, o);
                    }
            ml_s[2 * g_own] = m_own;
            ml_s[2 * g_own + 1] = l_own;
            __syncwarp();
            if (sub == 0) {
#pragma unroll
                for (int g = 0; g < GP; ++g) {
                    if (g < ns) {
                        const int jr = g / nh;
                        const size_t qh = (size_t)(ci.row + jr) * a.num_q_heads + (size_t)ci.kv_head * a.group +
                                          ci.head0 + (g - jr * nh);
                        if (ci.partial < 0) {
                            const float inv = 1.f / ml_s[2 * g + 1];
                            float o[C::EPC];
#pragma unroll
                            for (int e = 0; e < C::E2; ++e) {
                                o[2 * e] = acc2[g][e].x * inv;
                                o[2 * e + 1] = acc2[g][e].y * inv;
                            }
                            *reinterpret_cast<uint4*>(static_cast<unsigned char*>(a.out) + qh * C::ROW + chunk * 16) =
                                Chunk<T>::pack(o);
                        } else {
                            float* po = a.part_o + ((size_t)ci.partial * a.part_stride + g) * D + chunk * C::EPC;
#pragma unroll
                            for (int e = 0; e < C::E2; e += 2)
                                *reinterpret_cast<float4*>(po + 2 * e) =
                                    make_float4(acc2[g][e].x, acc2[g][e].y, acc2[g][e + 1].x, acc2[g][e + 1].y);
                            if (chunk == 0) {
                                float* pm = a.part_ml + ((size_t)ci.partial * a.part_stride + g) * 2;
                                pm[0] = ml_s[2 * g];
                                pm[1] = ml_s[2 * g + 1];
                            }
                        }
                    }
                }
            }
            __syncwarp();
            c_it += W;
            if (c_it >= a.num_items) break;
            ci = load_item(a.items, c_it);
            c_blk = ci.blk_begin;
        } else {
            ++c_blk;
        }
    }
}

// One warp per (merge row, slot): out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i over the row's
// partials -- its own chunks and, for a request sharing its leading blocks with others, the shared
// items' chunks. A chunk that saw no key of a slot has m = -inf and weight 0.
// The kernel is a chain of dependent memory latencies, so it keeps that chain short: once the merge
// row is read, the (m, l) pairs (one partial per lane) and the output columns of the first kPre
// partials (each lane its D/32 columns) are loaded together; the weights then reach every lane by
// shuffles. Further partials, if any, are read kPre at a time.
template <int PER>
struct MergeVec;
template <>
struct MergeVec<4> {
    using type = float4;
    __device__ static void fma(float w, const float4& v, float* o) {
        o[0] = fmaf(w, v.x, o[0]); o[1] = fmaf(w, v.y, o[1]); o[2] = fmaf(w, v.z, o[2]); o[3] = fmaf(w, v.w, o[3]);
    }
};
template <>
struct MergeVec<2> {
    using type = float2;
    __device__ static void fma(float w, const float2& v, float* o) {
        o[0] = fmaf(w, v.x, o[0]); o[1] = fmaf(w, v.y, o[1]);
    }
};

template <typename T, int D>
__global__ void __launch_bounds__(128) merge_kernel(const MergeArgs a) {
    constexpr int PER = D / 32;
    constexpr int kPre = 4;
    using V = MergeVec<PER>;
    using VT = typename V::type;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int entry = gw / a.slots_per_entry;
    const int g = gw % a.slots_per_entry;
    griddep_wait();
    if (entry >= a.num_rows) return;
    const MergeRow mr = a.rows[entry];
    if (g >= mr.num_slots) return;
    const int total = mr.count + (mr.extra_first >= 0 ? mr.extra_count : 0);
    auto slot_of = [&](int i) -> size_t {
        return i < mr.count ? (size_t)(mr.first_partial + i) * a.part_stride + g
                            : (size_t)(mr.extra_first + i - mr.count) * a.part_stride + mr.extra_slot + g;
    };
    auto o_at = [&](int i) { return *reinterpret_cast<const VT*>(a.part_o + slot_of(i) * D + lane * PER); };
    const float2* ml = reinterpret_cast<const float2*>(a.part_ml);
    // Issued together: this lane's (m, l) and the first partials' output columns.
    const float2 mine = lane < total ? ml[slot_of(lane)] : make_float2(-INFINITY, 0.f);
    VT pre[kPre];
#pragma unroll
    for (int u = 0; u < kPre; ++u)
        if (u < total) pre[u] = o_at(u);
    // Row maximum over all partials (lanes hold the first 32; more are folded in by a loop).
    float M = mine.x;
    for (int i = lane + 32; i < total; i += 32) M = fmaxf(M, ml[slot_of(i)].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL_MASK, M, o));
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    float L = 0.f;
    for (int base = 0; base < total; base += 32) {
        const int n = min(32, total - base);
        float w = 0.f;
        if (lane < n) {
            const float2 v = base == 0 ? mine : ml[slot_of(base + lane)];
            w = fast_exp2(v.x - M);
            L = fmaf(w, v.y, L);
        }
        int j = 0;
        if (base == 0) {
#pragma unroll
            for (int u = 0; u < kPre; ++u)
                if (u < n) V::fma(__shfl_sync(FULL_MASK, w, u), pre[u], acc);
            j = min(n, kPre);
        }
        for (; j < n; j += kPre) {
            VT v[kPre];
#pragma unroll
            for (int u = 0; u < kPre; ++u)
                if (j + u < n) v[u] = o_at(base + j + u);
#pragma unroll
            for (int u = 0; u < kPre; ++u)
                if (j + u < n) V::fma(__shfl_sync(FULL_MASK, w, j + u), v[u], acc);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(FULL_MASK, L, o);
    const float inv = 1.f / L;
    const int jr = g / mr.heads_per_row;
    T* out = static_cast<T*>(a.out) +
             ((size_t)(mr.row + jr) * a.num_q_heads + mr.q_head0 + (g - jr * mr.heads_per_row)) * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        if constexpr (sizeof(T) == 4) out[e] = acc[e] * inv;
        else if constexpr (std::is_same<T, __half>::value) out[e] = __float2half_rn(acc[e] * inv);
        else out[e] = __float2bfloat16_rn(acc[e] * inv);
    }
}

template <typename T, int D, int GP, int NSTAGE>
cudaError_t launch_decode_t(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    using C = Dec<T, D, GP, NSTAGE>;
    const int smem = kDecodeWarps * C::WARP_SMEM;
    // The shared-memory attribute and the occupancy are per device; cache both per instantiation.
    static int per_sm_cache[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int per_sm = (dev >= 0 && dev < 64) ? per_sm_cache[dev] : 0;
    if (per_sm == 0) {
        e = cudaFuncSetAttribute(decode_kernel<T, D, GP, NSTAGE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<T, D, GP, NSTAGE>, kDecodeWarps * 32, smem);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) per_sm = 1;
        if (dev >= 0 && dev < 64) per_sm_cache[dev] = per_sm;
    }
    const int need = (a.num_items + kDecodeWarps - 1) / kDecodeWarps;
    int grid = num_sms * per_sm;
    if (grid > need) grid = need;
    if (grid < 1) return cudaSuccess;
    return launch_k(a.pdl, decode_kernel<T, D, GP, NSTAGE>, dim3(grid), dim3(kDecodeWarps * 32), smem, s, a);
}

// Ring depth: the default per group size, or PKV_DECODE_STAGES (2..4) as a tuning override.
inline int stage_override() {
    static const int v = [] {
        const char* e = getenv("PKV_DECODE_STAGES");
        const int x = e ? atoi(e) : 0;
        return (x >= 2 && x <= 4) ? x : 0;
    }();
    return v;
}

template <typename T, int D, int GP>
cudaError_t launch_decode_s(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    switch (stage_override() ? stage_override() : default_stages<GP>()) {
        case 2: return launch_decode_t<T, D, GP, 2>(a, num_sms, s);
        case 4: return launch_decode_t<T, D, GP, 4>(a, num_sms, s);
        default: return launch_decode_t<T, D, GP, 3>(a, num_sms, s);
    }
}

template <typename T, int D>
cudaError_t launch_decode_g(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    const int g = a.slots_per_item;
    if (g <= 1) return launch_decode_s<T, D, 1>(a, num_sms, s);
    if (g <= 2) return launch_decode_s<T, D, 2>(a, num_sms, s);
    if (g <= 4) return launch_decode_s<T, D, 4>(a, num_sms, s);
    return launch_decode_s<T, D, 8>(a, num_sms, s);
}

template <typename T>
cudaError_t launch_decode_d(int head_dim, const DecodeArgs& a, int num_sms, cudaStream_t s) {
    if (head_dim == 64) return launch_decode_g<T, 64>(a, num_sms, s);
    return launch_decode_g<T, 128>(a, num_sms, s);
}

template <typename T>
cudaError_t launch_merge_d(int head_dim, const MergeArgs& a, cudaStream_t s) {
    const long long warps = (long long)a.num_rows * a.slots_per_entry;
    const int grid = (int)((warps * 32 + 127) / 128);
    if (grid < 1) return cudaSuccess;
    if (head_dim == 64) return launch_k(a.pdl, merge_kernel<T, 64>, dim3(grid), dim3(128), 0, s, a);
    return launch_k(a.pdl, merge_kernel<T, 128>, dim3(grid), dim3(128), 0, s, a);
}

}  // namespace

cudaError_t launch_decode(int dtype, int head_dim, const DecodeArgs& a, int num_sms, cudaStream_t s) {
    if (a.num_items <= 0) return cudaSuccess;
    switch (dtype) {
        case 0: return launch_decode_d<float>(head_dim, a, num_sms, s);
        case 1: return launch_decode_d<__half>(head_dim, a, num_sms, s);
        default: return launch_decode_d<__nv_bfloat16>(head_dim, a, num_sms, s);
    }
}

cudaError_t launch_merge(int dtype, int head_dim, const MergeArgs& a, cudaStream_t s) {
    if (a.num_rows <= 0) return cudaSuccess;
    switch (dtype) {
        case 0: return launch_merge_d<float>(head_dim, a, s);
        case 1: return launch_merge_d<__half>(head_dim, a, s);
        default: return launch_merge_d<__nv_bfloat16>(head_dim, a, s);
    }
}

}  // namespace pkv
