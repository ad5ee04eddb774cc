// Chunked-prefill attention tiles on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes: for a request with n > 1 query rows at prior context P (blog.mckayzhao.com/?p=56,
// "进阶特性：让推理再快一点" -- chunked prefill; "V1 架构：推倒重来的勇气" -- one mixed batch), row j
// attends keys 0 .. P+j of the request's cache, read block by block through its block table
// ("PagedAttention：操作系统课本里翻出来的灵感"). Here QK^T and PV are dense contractions, so they run
// on tcgen05 with fp32 accumulation in tensor memory; softmax stays in fp32 on the CUDA cores and
// P is rounded to the input type for the PV product.
//
// CTA: two 128-row MMA tiles (A, B), each (128/G) consecutive query rows x the G query heads of one
// KV head (GQA packing), sharing one stream of 128-key K/V tiles (8 blocks), so every K/V byte
// fetched from L2 serves 256 rows. Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: one thread per row
//   warp  8    TMA producer: both Q tiles once (3-D tensor map, SWIZZLE_128B), then per key tile
//              8 blocks x 2 column halves of K and of V (2-D tensor map over the pool rows),
//              double-buffered, K and V released separately
//   warp  9    MMA issuer (one thread): S_X = Q_X K^T into TMEM; after softmax X has written
//              P_X (16-bit, over the first 64 columns of S_X), O_X += P_X V with A read from TMEM.
//              The two tiles ping-pong: one tile's softmax overlaps the other tile's MMAs.
//   warps 10-11 idle; they complete the third warpgroup, whose registers move to the softmax
//              warpgroups (setmaxnreg).
// The CTAs are persistent (one per SM): they take tiles, longest first, from a ticket counter. In a
// mixed batch they also serve the split-K decode items (the warp-MMA loop of decode_mma.cuh over
// buffers carved from the tile stages: all twelve warps for items of at most 8 (row, head) slots,
// warps 0-7 for larger items), so the HBM-bound decode rows and the tensor-bound tiles share the
// GPU in one launch.
// A softmax thread reads its row's whole key tile from TMEM in one round trip, then works on it
// in two halves of 64 columns and signals each half's P separately. O accumulates in TMEM across
// key tiles. A row's
// exponentials use a reference maximum that is raised only when a half's maximum exceeds it by
// 2^8; O is then rescaled in TMEM (exact: softmax is shift invariant, and p stays <= 2^8). The
// half's maximum is only taken when the weights' sum against the current reference shows that a
// raise may be due.
// Blocks past the context are fetched at an out-of-range coordinate (TMA fills zeros); V rows past
// the context inside the last block are zeroed before PV (stale slots may hold anything).
// Every wait is bounded; on expiry the CTA records PKV_ERR_DEVICE_TIMEOUT, drains its own copies
// and MMAs (bounded), frees its tensor memory and stops taking work. No TMA multicast.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "decode_mma.cuh"
#include "tma_host.h"

namespace pkv {
namespace {

constexpr int kThreads = 384;
// Registers per thread after the split (setmaxnreg): the third warpgroup gives up registers so the
// two softmax warpgroups may grow. The launch holds kThreads x 168 registers (the most 384 threads
// get: three warps share each SM sub-partition's 16384); the split needs exactly as many,
// 2 x 128 x 216 + 128 x 72 = 64512 = 384 x 168, so the growing warpgroups never wait for more than
// the shrinking one releases. ptxas fits both regions without spilling at these counts.
constexpr int kSoftmaxRegs = 216;
constexpr int kOtherRegs = 72;
// Rounds of split-K items of at most 8 (row, head) slots run on all twelve warps, each at 168.
constexpr int kItemRegs = 168;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs == kThreads * 168 && kItemRegs == 168,
              "register split: every split must add up to the launch's registers");
constexpr int kHalf = 128 * 128;        // 128 rows x 64 elements x 2 bytes
constexpr int kTile = 2 * kHalf;        // 128 x 128 x 2 bytes
constexpr int OFF_Q = 0;                // Q_A, Q_B
constexpr int OFF_K = OFF_Q + 2 * kTile;    // 2 stages
constexpr int OFF_V = OFF_K + 2 * kTile;    // 2 stages
constexpr int OFF_BAR = OFF_V + 2 * kTile;
// barrier slots (8 bytes each); per-tile barriers are indexed by tile 0 (A) / 1 (B)
enum {
    B_Q = 0, B_F0 = 1, B_E0 = 3, B_SF0 = 5, B_PF0 = 7, B_OF0 = 9, B_DRAIN = 11, B_PH0 = 12, B_OH0 = 14,
    NUM_BARS = 16
};
constexpr int OFF_TMEM = OFF_BAR + 2 * NUM_BARS * 8; // tcgen05.alloc result (after two barrier sets)
constexpr int OFF_BSET = OFF_TMEM + 12;              // the current tile's barrier set (thread 0 writes it)
constexpr int OFF_ABORT = OFF_TMEM + 4;
constexpr int OFF_CTRL = OFF_ABORT + 4;              // the CTA's next step (thread 0 writes it)
// Rounds of split-K items take kDecodeStages stages per warp from the tile buffers, with their own
// mbarriers and item rings after the tile barriers. An SM serving items is bound by its warps'
// instruction issue, not by bytes in flight (4 warps stream half what 8 do; a third stage per warp
// adds nothing), so items of at most 8 (row, head) slots -- the transposed form -- run on all 12
// warps with K/V-only stages (12 x 2 x 8 KiB = 192 KiB) and q rows in registers; items of up to 16
// slots on warps 0-7 with q staged beside K/V (8 x 2 x 12 KiB).
constexpr int kDecodeStages = 2;
template <int DEC> struct ItemRound {
    static constexpr bool kQreg = DEC == 2;
    static constexpr int kWarps = DEC == 2 ? 12 : 8;
    static constexpr int kStageBytes = DEC == 2 ? mma::kKV : mma::kStage;
    static_assert(kWarps * kDecodeStages * kStageBytes <= OFF_BAR, "split-K stages overlap the tile barriers");
};
constexpr int kMaxItemWarps = 12;
constexpr int OFF_DBAR = OFF_TMEM + 16;
constexpr int OFF_FIFO = OFF_DBAR + kMaxItemWarps * kDecodeStages * 8;
constexpr int SMEM_USED = OFF_FIFO + kMaxItemWarps * mma::kFifo * 4;
constexpr int SMEM_BYTES = SMEM_USED + 1024;         // slack to align the base to 1024 bytes
static_assert(OFF_DBAR % 8 == 0, "mbarrier alignment");
constexpr uint32_t kTmemCols = 512;                  // S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512)
// A row's exponentials use a reference max that is only raised when the tile max exceeds it by
// more than this (log2 units); the result is exact (softmax is shift invariant) and p <= 2^8.
constexpr float kRescaleThreshold = 8.f;
// A half key tile whose weights (against the current reference) sum to at most this has none
// above 2^kRescaleThreshold, even counting the fp16 rounding of the summed weights.
constexpr float kRescaleBound = 255.f;
// Of each 32 exponentials of an unmasked key tile, 2 * POLY are computed by exp2_poly2 on the FMA
// pipe (the kernel's template parameter). Measured slower at every share tried (MUFU is not what
// bounds the softmax: ex2 runs at 16 per clock per SM and the softmax keeps it about half busy), so
// kernels are built with none.
constexpr int kPolyPairs = 0;

// ---- tcgen05 / TMA primitives ---------------------------------------------------------------
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// tcgen05.mma kind::f16 with each shared-memory descriptor given as its low and high 32-bit words;
// the _ts form reads the A operand (M x K, K-major, two 16-bit elements per 32-bit column) from TMEM.
__device__ __forceinline__ void tc_mma_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi, uint32_t idesc,
                                          bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 ad, bd;\n\tsetp.ne.b32 p, %5, 0;\n\t"
        "mov.b64 ad, {%1, %3};\n\tmov.b64 bd, {%2, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %4, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"((uint32_t)acc)
        : "memory");
}
__device__ __forceinline__ void tc_mma_ts_lo(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t hi,
                                             uint32_t idesc, bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 bd;\n\tsetp.ne.b32 p, %5, 0;\n\t"
        "mov.b64 bd, {%2, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %4, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(idesc), "r"((uint32_t)acc)
        : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns from registers (thread i writes TMEM lane base + i).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive fp32 columns: thread i of the warp receives TMEM lane (base lane + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 32 lanes x 128 consecutive fp32 columns in one round trip, complete on return (the wait is part
// of the same asm statement, so no use of the destination registers can come before it).
__device__ __forceinline__ void tmem_ld128_sync(uint32_t taddr, float* v) {
    uint32_t r[128];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%128];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%129];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95}, [%130];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%131];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
        : "r"(taddr), "r"(taddr + 32), "r"(taddr + 64), "r"(taddr + 96)
        : "memory");
#pragma unroll
    for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
}

// High word of every shared-memory descriptor here: SBO 1024 bytes (bits 32-45), descriptor
// version 1 (bit 46), 128-byte swizzling (bits 61-63 = 2).
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
// Instruction descriptor of kind::f16 with fp32 accumulation, M = N = 128.
__host__ __device__ constexpr uint32_t idesc_f16(uint32_t ab_format, uint32_t b_mn_major) {
    return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (b_mn_major << 16) | ((128u >> 3) << 17) |
           ((128u >> 4) << 24);
}

// Bounded wait that also gives up when another role has aborted the CTA.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag, DeviceError* err,
                                              int where) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > WAIT_BUDGET_CYCLES) {
            *abort_flag = 1;
            record_error(err, 5 /*PKV_ERR_DEVICE_TIMEOUT*/, where);
            return false;
        }
    }
    return true;
}

// CTA-wide barrier 0 that the warps may reach at different instructions (the two register-split
// branches each end with one).
__device__ __forceinline__ void cta_sync() { asm volatile("barrier.sync 0;" ::: "memory"); }

// Warp-uniform "all succeeded" for the lanes of one warp.
__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(FULL_MASK, v); }

// What a pair of softmax weights adds to the row sum. PV uses the weights rounded to T; for fp16
// the sum takes them as rounded too, so that the normalisation matches the numerator exactly (an
// fp16 output of magnitude 4..8 has a rounding step of ~2e-3, which leaves no room for the
// mismatch on rows dominated by one key). For bf16 the unrounded weights are summed: the
// mismatch (at most 2^-9 relative) stays far inside bf16's own output rounding, and the unpack
// costs about 5 % of the kernel.
template <typename T>
__device__ __forceinline__ float2 row_sum_term(float2 p, uint32_t packed) {
    if constexpr (std::is_same<T, __half>::value) return unpack2<T>(packed);
    else return p;
}

// What every role needs to know about one tile (request, KV head, 2 x 128 packed rows).
struct TileCtx {
    int req, kvh, tok0, q0, n, ctx, prior, G, tt, nkt, nblk_ctx, rows_total;
    int nkt_a, nkt_b;  // key tiles each MMA tile (A, B) needs: keys visible to its last valid row
    // Key tiles of MMA tile x (a select, so that no per-tile array lands in local memory).
    __device__ __forceinline__ int nkt_of(int x) const { return x ? nkt_b : nkt_a; }
    bool has_b, sane;
};

__device__ __forceinline__ TileCtx tile_ctx(const PrefillArgs& a, int t) {
    TileCtx c;
    const PrefillTile pt = a.tiles[t];
    c.req = pt.req;
    c.kvh = pt.kv_head;
    c.tok0 = pt.tok0;
    c.q0 = a.query_start_loc[c.req];
    c.n = a.query_start_loc[c.req + 1] - c.q0;
    c.ctx = a.context_lens[c.req];
    c.prior = c.ctx - c.n;
    c.G = a.group;
    c.tt = 128 / c.G;
    c.has_b = c.tok0 + c.tt < c.n;
    c.nkt_a = (min(c.ctx, c.prior + min(c.n, c.tok0 + c.tt)) + 127) / 128;
    c.nkt_b = c.has_b ? (min(c.ctx, c.prior + min(c.n, c.tok0 + 2 * c.tt)) + 127) / 128 : 0;
    c.nkt = max(c.nkt_a, c.nkt_b);
    c.nblk_ctx = (c.ctx + kBlockSize - 1) / kBlockSize;
    c.rows_total = a.num_blocks * a.num_kv_heads * kBlockSize;
    c.sane = c.nkt >= 1 && c.n > 1 && c.tok0 < c.n;
    return c;
}

// Arms the tile barriers for a new tile (thread 0; they are idle: the previous tile waited for
// every phase it started).
__device__ __forceinline__ void init_tile_barriers(uint64_t* bars) {
    mbar_init(&bars[B_Q], 1);
    for (int s = 0; s < 2; ++s) {
        mbar_init(&bars[B_F0 + s], 1);
        mbar_init(&bars[B_E0 + s], 1);
        mbar_init(&bars[B_SF0 + s], 1);
        mbar_init(&bars[B_PF0 + s], 128);
        mbar_init(&bars[B_OF0 + s], 1);
        mbar_init(&bars[B_PH0 + s], 128);
        mbar_init(&bars[B_OH0 + s], 1);
    }
    mbar_init(&bars[B_DRAIN], 1);
    fence_mbar_init();
}

// ---- TMA producer (warp 8) ----
// Loads go in groups, one barrier wait and one transaction barrier per key tile: the Q tiles with
// K(0) on B_Q, then group kt = V(kt) and K(kt+1) on B_F(kt & 1), the two operands the MMA issuer
// consumes in its iteration kt (PV(kt), QK^T(kt+1)). V(kt) goes to V stage kt & 1, K(kt+1) to K
// stage (kt+1) & 1, so group kt reuses the stages of group kt-2, which the issuer frees with one
// commit on B_E(kt & 1) at the end of its iteration kt-2; for group 1 that is the commit after
// the prologue's QK^T(0), which frees K(0)'s stage. Lane l < 16 serves one block of a group:
// l < 8 block l of V(kt), l >= 8 block l-8 of K(kt+1); each lane reads its own block-table entry
// a group ahead.
__device__ __forceinline__ void tile_producer(const PrefillArgs& a, const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                              const CUtensorMap* tm_v, unsigned char* smem, uint64_t* bars,
                                              volatile int* abort_flag, const TileCtx& tile, int lane) {
    const int j = lane & 7;
    // Table entry of block j of key tile t: -2 past the context (never read), -3 past the table's
    // width (device lengths larger than the planned ones: a range error below).
    auto block_id = [&](int t) -> int {
        const int b = t * 8 + j;
        return b >= tile.nblk_ctx ? -2
               : b < a.max_blocks_per_seq ? __ldg(a.block_tables + (size_t)tile.req * a.max_blocks_per_seq + b) : -3;
    };
    // Pool row of that block's K/V for this KV head; the row past the pool (zero fill) past the
    // context or on a range error.
    auto block_row = [&](int id, int t) -> int {
        if (id == -2) return tile.rows_total;
        if (id < 0 || id >= a.num_blocks) {
            record_error(a.err, 6 /*PKV_ERR_DEVICE_RANGE*/, (long long)tile.req * a.max_blocks_per_seq + t * 8 + j);
            return tile.rows_total;
        }
        return (id * a.num_kv_heads + tile.kvh) * kBlockSize;
    };
    const bool v_lane = lane < 8, k_lane = lane >= 8 && lane < 16;
    const int id0 = k_lane ? block_id(0) : 0;
    if (lane == 0) {
        mbar_arrive_expect_tx(&bars[B_Q], (tile.has_b ? 2 * kTile : kTile) + kTile);
        for (int x = 0; x < (tile.has_b ? 2 : 1); ++x) {
            const int z = tile.q0 + tile.tok0 + x * tile.tt;
            tma_load_3d(smem + OFF_Q + x * kTile, tm_q, 0, tile.kvh * tile.G, z, &bars[B_Q]);
            tma_load_3d(smem + OFF_Q + x * kTile + kHalf, tm_q, 64, tile.kvh * tile.G, z, &bars[B_Q]);
        }
    }
    __syncwarp();
    if (k_lane) {
        const int y = block_row(id0, 0);
        tma_load_2d(smem + OFF_K + j * 2048, tm_k, 0, y, &bars[B_Q]);
        tma_load_2d(smem + OFF_K + kHalf + j * 2048, tm_k, 64, y, &bars[B_Q]);
    }
    int id_next = v_lane ? block_id(0) : k_lane && 1 < tile.nkt ? block_id(1) : -2;
    int last = -1;  // the last group issued
    bool ok = true;
    for (int kt = 0; kt < tile.nkt && ok; ++kt) {
        const int g = kt & 1;
        const bool has_k = kt + 1 < tile.nkt;
        const int id = id_next;
        if (has_k) id_next = v_lane ? block_id(kt + 1) : k_lane && kt + 2 < tile.nkt ? block_id(kt + 2) : -2;
        if (kt >= 1) ok = warp_all(wait_or_abort(&bars[B_E0 + g], ((kt - 2 + g) >> 1) & 1, abort_flag, a.err, 100));
        if (!ok) break;
        if (lane == 0) mbar_arrive_expect_tx(&bars[B_F0 + g], has_k ? 2 * kTile : kTile);
        __syncwarp();
        if (v_lane) {
            unsigned char* vs = smem + OFF_V + g * kTile;
            const int y = block_row(id, kt);
            tma_load_2d(vs + j * 2048, tm_v, 0, y, &bars[B_F0 + g]);
            tma_load_2d(vs + kHalf + j * 2048, tm_v, 64, y, &bars[B_F0 + g]);
        } else if (k_lane && has_k) {
            unsigned char* ks = smem + OFF_K + (g ^ 1) * kTile;
            const int y = block_row(id, kt + 1);
            tma_load_2d(ks + j * 2048, tm_k, 0, y, &bars[B_F0 + g]);
            tma_load_2d(ks + kHalf + j * 2048, tm_k, 64, y, &bars[B_F0 + g]);
        }
        last = kt;
        __syncwarp();
    }
    if (!ok && lane == 0) {
        // Drain: wait (bounded) for the last group issued on each barrier, and for Q with K(0).
        for (int g = 0; g < 2; ++g) {
            const int jl = last - ((last - g) & 1);
            if (last >= 0 && jl >= 0) (void)mbar_wait(&bars[B_F0 + g], (jl >> 1) & 1);
        }
        (void)mbar_wait(&bars[B_Q], 0);
    }
}

// ---- MMA issuer (warp 9, one thread) ----
template <typename T>
__device__ __forceinline__ void tile_mma(const PrefillArgs& a, unsigned char* smem, uint64_t* bars,
                                         volatile int* abort_flag, uint32_t tmem, const TileCtx& tile, int lane) {
    if (lane == 0) {
        const uint32_t fmt = std::is_same<T, __half>::value ? 0u : 1u;
        const uint32_t id_qk = idesc_f16(fmt, 0);
        const uint32_t id_pv = idesc_f16(fmt, 1);
        // This thread shares its SM sub-partition with two busy softmax warps, so each of its
        // instructions waits for an issue slot while the tensor pipe may run dry. The shared-memory
        // descriptors are therefore a precomputed low word plus a constant per MMA (the high word,
        // SBO 1024 with 128-byte swizzling, is the same for all).
        const uint32_t base = smem_u32(smem) >> 4;
        const uint32_t lo_q = base + (OFF_Q >> 4) + (1u << 16);                       // K-major, LBO 16 B
        const uint32_t lo_k = base + (OFF_K >> 4) + (1u << 16);
        const uint32_t lo_v = base + (OFF_V >> 4) + ((uint32_t)(kHalf >> 4) << 16);   // MN-major, LBO one half
        auto issue_qk = [&](int x, int kt) {
            const uint32_t qa = lo_q + (uint32_t)x * (kTile >> 4), kb = lo_k + (uint32_t)(kt & 1) * (kTile >> 4);
            const uint32_t d = tmem + x * 128;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t off = (uint32_t)(((k >> 2) * kHalf + (k & 3) * 32) >> 4);
                tc_mma_lo(d, qa + off, kb + off, kDescHi, id_qk, k > 0);
            }
            tc_commit(&bars[B_SF0 + x]);
        };
        // PV of one half (64 keys) of key tile kt. P_X(kt) sits as packed 16-bit pairs in the first
        // 64 columns of S_X; each K step of 16 keys is 8 columns.
        auto issue_pv = [&](int x, int kt, int h) {
            const uint32_t vb = lo_v + (uint32_t)(kt & 1) * (kTile >> 4);
            const uint32_t d = tmem + 256 + x * 128, pa = tmem + x * 128;
#pragma unroll
            for (int k = 4 * h; k < 4 * h + 4; ++k)
                tc_mma_ts_lo(d, pa + k * 8, vb + (uint32_t)(k * (2048 >> 4)), kDescHi, id_pv, kt > 0 || k > 0);
            tc_commit(&bars[(h ? B_OF0 : B_OH0) + x]);
        };
        // Each barrier wait of this thread leaves the tensor pipe idle for its latency, so an
        // iteration waits three times: P_A, the group's loads (once), P_B; and commits once.
        bool ok = wait_or_abort(&bars[B_Q], 0, abort_flag, a.err, 200);   // Q tiles and K(0)
        if (ok) {
            tc_fence_after();
            issue_qk(0, 0);
            if (tile.has_b) issue_qk(1, 0);
            tc_commit(&bars[B_E0 + 1]);   // K(0)'s stage, for group 1
        }
        for (int kt = 0; kt < tile.nkt && ok; ++kt) {
            const int g = kt & 1;
            bool f_ready = false;
            for (int x = 0; x < 2 && ok; ++x) {
                if (kt < tile.nkt_of(x)) {
                    ok = wait_or_abort(&bars[B_PH0 + x], kt & 1, abort_flag, a.err, 210 + x);
                    if (ok && !f_ready) ok = f_ready = wait_or_abort(&bars[B_F0 + g], (kt >> 1) & 1, abort_flag, a.err, 204);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(x, kt, 0);
                    ok = wait_or_abort(&bars[B_PF0 + x], kt & 1, abort_flag, a.err, 202 + x);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(x, kt, 1);
                }
                // QK^T(kt+1) of tile x follows its PV(kt) (kt + 1 < nkt_x implies kt < nkt_x), so
                // group kt (which holds K(kt+1)) has been waited for.
                if (kt + 1 < tile.nkt_of(x)) issue_qk(x, kt + 1);
            }
            if (!ok) break;
            tc_commit(&bars[B_E0 + g]);
        }
        if (ok) {
            // Every commit of this tile has arrived before the barriers are armed for the next one:
            // the last phase of each stage-free barrier (B_E0 takes iterations 0, 2, ...; B_E1 the
            // prologue and iterations 1, 3, ...) and of each tile's O.
            const int n_e[2] = {(tile.nkt + 1) / 2, 1 + tile.nkt / 2};
            for (int g = 0; g < 2 && ok; ++g) {
                ok = wait_or_abort(&bars[B_E0 + g], (n_e[g] - 1) & 1, abort_flag, a.err, 207);
                if (ok && tile.nkt_of(g) > 0)
                    ok = wait_or_abort(&bars[B_OF0 + g], (tile.nkt_of(g) - 1) & 1, abort_flag, a.err, 209);
                if (ok && tile.nkt_of(g) > 0)
                    ok = wait_or_abort(&bars[B_OH0 + g], (tile.nkt_of(g) - 1) & 1, abort_flag, a.err, 212);
            }
        } else {
            tc_commit(&bars[B_DRAIN]);
            (void)mbar_wait(&bars[B_DRAIN], 0);
        }
    }
}

// ---- softmax (warps 0-7: one thread per row of tile A or B) ----
template <typename T, int POLY>
__device__ __forceinline__ void tile_softmax(const PrefillArgs& a, unsigned char* smem, uint64_t* bars,
                                             volatile int* abort_flag, uint32_t tmem, const TileCtx& tile, int warp,
                                             int lane) {
    const int x = warp >> 2;                 // tile
    const int row = (warp & 3) * 32 + lane;
    const int t_local = row / tile.G, g = row % tile.G;
    const int j = tile.tok0 + x * tile.tt + t_local;
    const bool row_valid = j < tile.n;
    const int limit = row_valid ? tile.prior + j + 1 : tile.prior + 1;  // keys visible: [0, limit)
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t ts = tl + x * 128, to = tl + 256 + x * 128;
    // Keys below this bound are visible to every row of the tile: no masking needed there.
    const int all_visible = tile.prior + tile.tok0 + x * tile.tt + 1;
    const int my_nkt = tile.nkt_of(x);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // O in TMEM times f, row by row (warp-collective; rows whose factor is 1 are rewritten unchanged).
    auto scale_o = [&](float f) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(to + c * 32, o);
            tmem_wait_ld();
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o[i] * f);
            tmem_st32(to + c * 32, w);
        }
    };
    // P of the first half of a key tile (keys 0..63, columns 0..31) is signalled on B_PH, the rest
    // on B_PF, so that the PV of the first half runs while the second half's exponentials are taken.
    auto signal = [&](int bar) {
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[bar + x]);
    };
    for (int kt = 0; kt < my_nkt && ok; ++kt) {
        ok = warp_all(wait_or_abort(&bars[B_SF0 + x], kt & 1, abort_flag, a.err, 300));
        if (!ok) break;
        tc_fence_after();
        const bool full = kt * 128 + 128 <= all_visible;   // no masking anywhere in this key tile
        float alpha = 1.f;
        float2 ps2 = make_float2(0.f, 0.f);
        if (full && a.scale_log2 >= 0.f) {
            // S in one TMEM round trip; then per half of 64 keys, P against the row's reference m
            // (raised first, when needed, as below). P of keys 64*h.. goes to columns 32*h.. (over S
            // already read) and is signalled per half. A raise rescales what O holds against the old
            // reference: PV(kt-1) before the first half (none when kt = 0), the first half's PV
            // before the second.
            const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
            float sa[128];
            tmem_ld128_sync(ts, sa);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float* sv = sa + 64 * h;
                uint32_t pk[32];
                float2 hs;
                // P of the half against the row's current reference m. Its sum bounds every weight,
                // so a sum within kRescaleBound shows that no key of the half exceeds m by more than
                // the threshold and m stays: the half's maximum is not needed. Otherwise (rare after the
                // first key tiles; always while m is -inf, whose sum is infinite) the half takes the
                // maximum, raises m as before and computes P again. The weights are the same as
                // with the maximum taken first.
                auto weights = [&]() {
                    const float2 nm2 = make_float2(-m, -m);
                    hs = make_float2(0.f, 0.f);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float2 e = __ffma2_rn(make_float2(sv[2 * i], sv[2 * i + 1]), sc2, nm2);
                        const float2 p = (i & 15) < POLY ? exp2_poly2(e) : make_float2(fast_exp2(e.x), fast_exp2(e.y));
                        pk[i] = pack2<T>(p.x, p.y);
                        hs = __fadd2_rn(hs, row_sum_term<T>(p, pk[i]));
                    }
                };
                weights();
                if (__any_sync(FULL_MASK, !(hs.x + hs.y <= kRescaleBound))) {
                    float hm = -INFINITY;
#pragma unroll
                    for (int i = 0; i < 64; ++i) hm = fmaxf(hm, sv[i]);
                    hm *= a.scale_log2;
                    const bool raise = hm > m + kRescaleThreshold;
                    const float f = raise ? fast_exp2(m - hm) : 1.f;  // 0 while m is -inf
                    if (raise) {
                        ps2 = make_float2(ps2.x * f, ps2.y * f);
                        alpha *= f;
                        m = hm;
                    }
                    // The TMEM accesses are warp-collective: the whole warp takes this branch when
                    // any of its rows raised, each lane scaling its own row by its own factor.
                    if ((kt >= 1 || h == 1) && __any_sync(FULL_MASK, raise)) {
                        ok = warp_all(h == 0 ? wait_or_abort(&bars[B_OF0 + x], (kt - 1) & 1, abort_flag, a.err, 301)
                                             : wait_or_abort(&bars[B_OH0 + x], kt & 1, abort_flag, a.err, 304));
                        if (!ok) break;
                        tc_fence_after();
                        scale_o(f);
                    }
                    weights();
                }
                ps2 = __fadd2_rn(ps2, hs);
                tmem_st32(ts + h * 32, pk);
                signal(h ? B_PF0 : B_PH0);
            }
            if (!ok) break;
        } else {
            // S in one TMEM round trip; the row maximum of scale * s over the visible keys first.
            float sa[128];
            tmem_ld128_sync(ts, sa);
            const int key0 = kt * 128;
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 128; ++i)
                mx = fmaxf(mx, (full || key0 + i < limit) ? sa[i] * a.scale_log2 : -INFINITY);
            if (mx > m + kRescaleThreshold) {
                alpha = fast_exp2(m - mx);  // 0 on the first tile
                m = mx;
            }
            // O against the old reference (PV(kt-1) complete) is rescaled before any P is signalled.
            if (kt >= 1 && __any_sync(FULL_MASK, alpha != 1.f)) {
                ok = warp_all(wait_or_abort(&bars[B_OF0 + x], (kt - 1) & 1, abort_flag, a.err, 301));
                if (!ok) break;
                tc_fence_after();
                scale_o(alpha);
            }
            // V rows past the context (only possible in the CTA's final key tile) are zeroed by the
            // tile whose PV of that key tile is issued first: A when it reaches it, else B.
            if (kt == tile.nkt - 1 && (kt + 1) * 128 > tile.ctx && x == (tile.nkt_a == tile.nkt ? 0 : 1)) {
                ok = warp_all(wait_or_abort(&bars[B_F0 + (kt & 1)], (kt >> 1) & 1, abort_flag, a.err, 302));
                if (!ok) break;
                unsigned char* vs = smem + OFF_V + (kt & 1) * kTile;
                const int r0 = tile.ctx - kt * 128;  // first V row past the context
                const int chunks = (128 - r0) * 16;  // 16-byte chunks over both halves
                for (int c = (warp & 3) * 32 + lane; c < chunks; c += 128) {
                    const int r = r0 + (c >> 4), h = (c >> 3) & 1, k = c & 7;
                    *reinterpret_cast<uint4*>(vs + h * kHalf + r * 128 + k * 16) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            // p = 2^(s*scale - m), rounded to T, written over S (already in registers) as the A
            // operand of PV, 32 keys at a time into columns 16c..
            const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(-m, -m);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float* sv = sa + 32 * c;
                uint32_t pk[16];
                const int kc = key0 + c * 32;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 e = __ffma2_rn(make_float2(sv[2 * i], sv[2 * i + 1]), sc2, nm2);
                    const float p0 = (full || kc + 2 * i < limit) ? fast_exp2(e.x) : 0.f;
                    const float p1 = (full || kc + 2 * i + 1 < limit) ? fast_exp2(e.y) : 0.f;
                    pk[i] = pack2<T>(p0, p1);
                    ps2 = __fadd2_rn(ps2, row_sum_term<T>(make_float2(p0, p1), pk[i]));
                }
                tmem_st16(ts + c * 16, pk);
                if (c & 1) signal(c == 1 ? B_PH0 : B_PF0);
            }
        }
        const float ps = ps2.x + ps2.y;
        l = l * alpha + ps;
    }
    if (ok) ok = warp_all(wait_or_abort(&bars[B_OF0 + x], (my_nkt - 1) & 1, abort_flag, a.err, 303));
    if (ok) {
        tc_fence_after();
        const float inv = 1.f / l;
        unsigned char* dst = static_cast<unsigned char*>(a.out) +
                             ((size_t)(tile.q0 + (row_valid ? j : 0)) * a.num_q_heads + (size_t)tile.kvh * tile.G + g) * 256;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(to + c * 32, o);
            tmem_wait_ld();
            if (row_valid) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float v[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = o[q * 8 + e] * inv;
                    *reinterpret_cast<uint4*>(dst + c * 64 + q * 16) = Chunk<T>::pack(v);
                }
            }
        }
    }
}

// Control word written by thread 0 before each step of the CTA: a tile index, or one of these.
constexpr int kJobExit = -1;    // the CTA is done
constexpr int kJobDecode = -2;  // a round of split-K items
constexpr int kJobNone = -3;    // nothing in this step
constexpr int kJobTilesDone = -4;  // no tile is left

// A round of split-K items: this warp takes tickets until none is left.
template <typename T, int DEC>
__device__ __forceinline__ void item_round(const DecodeArgs& d, const CUtensorMap* tm_kb, const CUtensorMap* tm_vb,
                                           unsigned char* smem, volatile int* abort_flag, int warp, int lane) {
    using R = ItemRound<DEC>;
    int first = 0;
    if (lane == 0) first = atomicAdd(&d.work[0], 1);
    first = __shfl_sync(FULL_MASK, first, 0);
    uint64_t* dbars = reinterpret_cast<uint64_t*>(smem + OFF_DBAR) + warp * kDecodeStages;
    volatile int* fifo = reinterpret_cast<volatile int*>(smem + OFF_FIFO) + warp * mma::kFifo;
    if (!mma::decode_warp<T, kDecodeStages, DEC == 2, R::kQreg>(d, tm_kb, tm_vb, smem + warp * kDecodeStages * R::kStageBytes,
                                                                 dbars, fifo, first, 0) &&
        lane == 0)
        *abort_flag = 1;
    fence_proxy_async_smem();   // its generic writes (zeroed V rows) before later TMA writes
}

// Persistent CTAs (one per SM) over the batch's tcgen05 tiles and, in a mixed batch, its split-K
// work items: tiles come from a ticket counter (a.work[2], longest first), items from the split-K
// counter (d.work[0]). A CTA b < a.decode_ctas first serves items until none is left; every CTA
// then serves tiles until none is left, then items again if any remain. So the HBM-bound items and
// the tensor-bound tiles run side by side, and whichever queue empties first hands its CTAs to the
// other. In a round of items, warps run the warp-MMA loop over two stages each, carved from the
// tile buffers: all twelve for items of at most 8 (row, head) slots (every warp at kItemRegs
// registers for the round), warps 0-7 otherwise (the third warpgroup waits). The last CTA to finish
// (a.work[3] counts them) resets the counters for the next launch.
template <typename T, int POLY, int DEC>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const PrefillArgs a, const DecodeArgs d, const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_kb, const __grid_constant__ CUtensorMap tm_vb) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
    volatile int* ctrl = reinterpret_cast<volatile int*>(smem + OFF_CTRL);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    griddep_wait();

    if (threadIdx.x == 0) *abort_flag = 0;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem + OFF_TMEM)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM);
    // Items of at most 8 slots run on all twelve warps at the launch's register count, so their
    // rounds come before and after the register split; items of up to 16 slots need more registers
    // and run on the softmax warps inside it.
    constexpr bool kAllWarps = ItemRound<DEC>::kWarps > 8;
    [[maybe_unused]] auto items_left = [&]() {
        return d.num_items > 0 && *reinterpret_cast<volatile int*>(&d.work[0]) < d.num_items && !*abort_flag;
    };
    // One step of items, between the two CTA barriers of a step (below): thread 0 decides whether
    // there are items to serve (in the first round only on the CTAs that start on items), then the
    // item warps serve them until none is left.
    [[maybe_unused]] auto item_step = [&](bool first_round) {
        if (threadIdx.x == 0)
            *ctrl = ((!first_round || (int)blockIdx.x < a.decode_ctas) && items_left()) ? kJobDecode : kJobNone;
        cta_sync();                                   // (1)
        if (*ctrl == kJobDecode && warp < ItemRound<DEC>::kWarps)
            item_round<T, DEC>(d, &tm_kb, &tm_vb, smem, abort_flag, warp, lane);
        tc_fence_before();
        cta_sync();                                   // (2)
    };
    // The end of the CTA: TMEM back, and the last CTA resets the counters for the next launch.
    auto finish = [&]() {
        if (threadIdx.x < 32) {   // warp 0; the TMEM address is read again rather than kept live
            tc_fence_after();
            const uint32_t t = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM);
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(t), "r"(kTmemCols) : "memory");
        }
        if (threadIdx.x == 0) {
            __threadfence();
            if (atomicAdd(&a.work[3], 1) == (int)gridDim.x - 1) {
                atomicExch(&a.work[2], 0);
                atomicExch(&a.work[3], 0);
                if (d.num_items > 0) atomicExch(&d.work[0], 0);
            }
        }
    };
    // (a) CTAs that start on items: a round of them first.
    if constexpr (kAllWarps) item_step(true);
    // Register split: the third warpgroup (producer, MMA issuer, two idle warps) shrinks to
    // kOtherRegs, the softmax warpgroups grow to kSoftmaxRegs. Each warpgroup runs in its own branch;
    // every step is bracketed by two CTA barriers: (1) thread 0 has written the step into *ctrl,
    // (2) the step is done.
    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
        while (true) {
            cta_sync();                                   // (1)
            const int job = *ctrl;
            if (job == kJobExit) break;
            if (job >= 0) {
                const TileCtx tile = tile_ctx(a, job);
                uint64_t* tb = bars + *reinterpret_cast<volatile int*>(smem + OFF_BSET) * NUM_BARS;
                if (tile.sane) {
                    if (warp == 8) tile_producer(a, &tm_q, &tm_k, &tm_v, smem, tb, abort_flag, tile, lane);
                    else if (warp == 9) tile_mma<T>(a, smem, tb, abort_flag, tmem, tile, lane);
                }
            }
            tc_fence_before();
            cta_sync();                                   // (2)
            if (kAllWarps && job == kJobTilesDone) break;
        }
        if constexpr (kAllWarps) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kItemRegs));
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        if constexpr (DEC != 0 && !kAllWarps) item_step(true);
        // (b) tiles, longest first, while any is left.
        int bset_seq = 1;   // thread 0: the barrier set of the last tile (tiles alternate between two)
        while (true) {
            if (threadIdx.x == 0) {
                int t = kJobTilesDone;
                if (!*abort_flag && *reinterpret_cast<volatile int*>(&a.work[2]) < a.num_tiles) {
                    t = atomicAdd(&a.work[2], 1);
                    if (t < a.num_tiles) {
                        // Tiles alternate between two barrier sets, so a tile's barriers are armed
                        // again only two tiles later. (With one set armed for every tile, batches
                        // whose CTAs take several tiles met bounded-wait timeouts under some
                        // schedules; the cause was not found.)
                        bset_seq ^= 1;
                        *reinterpret_cast<volatile int*>(smem + OFF_BSET) = bset_seq;
                        init_tile_barriers(bars + bset_seq * NUM_BARS);
                    }
                    else t = kJobTilesDone;
                }
                *ctrl = t;
            }
            cta_sync();                                   // (1)
            const int job = *ctrl;
            if (job >= 0) {
                tc_fence_after();
                const TileCtx tile = tile_ctx(a, job);
                uint64_t* tb = bars + *reinterpret_cast<volatile int*>(smem + OFF_BSET) * NUM_BARS;
                if (tile.sane && (warp < 4 || tile.has_b)) tile_softmax<T, POLY>(a, smem, tb, abort_flag, tmem, tile, warp, lane);
            }
            tc_fence_before();
            cta_sync();                                   // (2)
            if (job < 0) break;
        }
        if constexpr (kAllWarps) {
            asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kItemRegs));
        } else {
            // (c) the items still left once the tiles are gone; then the third warpgroup leaves.
            if constexpr (DEC != 0) item_step(false);
            if (threadIdx.x == 0) *ctrl = kJobExit;
            cta_sync();                                   // (1)
            finish();
        }
    }
    if constexpr (kAllWarps) {
        // (c) the items still left once the tiles are gone, on all twelve warps again.
        item_step(false);
        finish();
    }
}

template <typename T, int POLY, int DEC>
cudaError_t launch_t(const PrefillArgs& a, const DecodeArgs& d, int num_sms, cudaStream_t s) {
    const CUtensorMapDataType dt =
        std::is_same<T, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int G = a.group;
    CUtensorMap mq, mk, mv;
    const cuuint64_t qdims[3] = {128, (cuuint64_t)a.num_q_heads, (cuuint64_t)a.num_q_tokens};
    const cuuint64_t qstr[2] = {128 * 2, (cuuint64_t)a.num_q_heads * 128 * 2};
    const cuuint32_t qbox[3] = {64, (cuuint32_t)G, (cuuint32_t)(128 / G)};
    const long long rows = (long long)a.num_blocks * a.num_kv_heads * kBlockSize;
    const cuuint64_t kdims[2] = {128, (cuuint64_t)rows};
    const cuuint64_t kstr[1] = {128 * 2};
    const cuuint32_t kbox[2] = {64, (cuuint32_t)kBlockSize};
    // The tiles read the pool rows through a 64-column x 16-row box (8 blocks per key tile, two
    // halves each); the split-K items through the block-halves view (one copy per block).
    CUtensorMap mkb, mvb;
    if (!encode_tiled(&mq, dt, 3, a.q, qdims, qstr, qbox) || !encode_tiled(&mk, dt, 2, a.k_pool, kdims, kstr, kbox) ||
        !encode_tiled(&mv, dt, 2, a.v_pool, kdims, kstr, kbox) || !encode_block_halves(&mkb, dt, a.k_pool, rows) ||
        !encode_block_halves(&mvb, dt, a.v_pool, rows))
        return cudaErrorInvalidValue;
    static int configured[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(prefill_tc_kernel<T, POLY, DEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = 1;
    }
    // One persistent CTA per SM (fewer when the batch has fewer tiles and no split-K items).
    int grid = num_sms;
    if (d.num_items <= 0 && a.num_tiles < grid) grid = a.num_tiles;
    return launch_k(a.pdl, prefill_tc_kernel<T, POLY, DEC>, dim3(grid), dim3(kThreads), SMEM_BYTES, s, a, d, mq, mk,
                    mv, mkb, mvb);
}

// Batches with tcgen05 tiles only run an instantiation without the split-K rounds (fewer registers
// live in the softmax warps); mixed batches one whose rounds take the item form of the batch's
// items (the transposed form for items of at most 8 (row, head) slots).
template <typename T>
cudaError_t launch_m(const PrefillArgs& a, const DecodeArgs& d, int num_sms, cudaStream_t s) {
    if (d.num_items <= 0) return launch_t<T, kPolyPairs, 0>(a, d, num_sms, s);
    return d.slots_per_item <= 8 ? launch_t<T, kPolyPairs, 2>(a, d, num_sms, s)
                                 : launch_t<T, kPolyPairs, 1>(a, d, num_sms, s);
}

}  // namespace

bool prefill_tc_supported(int dtype, int head_dim, int group) {
    return (dtype == 1 || dtype == 2) && head_dim == 128 && group >= 1 && group <= 16 && (128 % group) == 0;
}

cudaError_t launch_prefill_tc(int dtype, const PrefillArgs& a, const DecodeArgs& d, int num_sms, cudaStream_t s) {
    if (a.num_tiles <= 0 && d.num_items <= 0) return cudaSuccess;
    if (!a.work || (d.num_items > 0 && !d.work)) return cudaErrorInvalidValue;
    if ((long long)a.num_blocks * a.num_kv_heads * kBlockSize >= (1LL << 31) - 1) return cudaErrorInvalidValue;
    if (((uintptr_t)a.q | (uintptr_t)a.k_pool | (uintptr_t)a.v_pool) & 15) return cudaErrorInvalidValue;
    return dtype == 1 ? launch_m<__half>(a, d, num_sms, s) : launch_m<__nv_bfloat16>(a, d, num_sms, s);
}

}  // namespace pkv
