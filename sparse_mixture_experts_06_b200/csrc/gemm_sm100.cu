// Grouped expert GEMMs on the 5th-generation tensor cores (sm_100a).
//
//   up   (SwiGLU expert, first half; "Mixtral of Experts" §2.1, Method:
//         SwiGLU expert):  for every permuted row r of expert e,
//         a = W1_e x_r, b = W3_e x_r (fp32 in tensor memory),
//         h_r = SiLU(a) * b rounded to bf16.
//   down (second half, the gate weighting and the scatter-back of §2.1
//         display 3): obuf_r = topk_w[perm[r]] * (W2_e h_r), fp32, parked;
//         the last of a token's slot rows to arrive (per 128 output
//         columns) adds the parked rows in slot order into y[t] (bf16).
//
// Both are one persistent, warp-specialised kernel (320 threads per CTA):
//   warp 0      TMA producer: 2-D tiled bulk copies (128-byte swizzle) of the
//               A tile (token rows x 64 k) and the B tile (weight rows x 64 k)
//               into a shared-memory ring of stages, signalled on mbarriers;
//   warp 1      MMA issuer: one thread issues tcgen05.mma (bf16 x bf16 ->
//               fp32, K = 16) into a tensor-memory (TMEM) accumulator and
//               releases ring stages with tcgen05.commit;
//   warps 2-9   epilogue: tcgen05.ld of the accumulator (two warps per
//               quadrant of 32 TMEM lanes, splitting the tile's columns),
//               fused SiLU(a)*b or gate scaling, and the stores.
// Tile shapes (template variants; the host picks one per launch):
//   single CTA   128 (or 32) rows x 256 columns, M = 128 N = 256 MMAs; two
//                TMEM accumulators, so a tile's epilogue overlaps the next
//                tile's main loop;
//   CTA pair     256 rows x 512 columns (default) or 256 x 256: cta_group::2
//                M = 256 MMAs issued by the even CTA, each CTA holding 128
//                rows of A and half of each MMA's B.  The 512-column tile
//                issues two N = 256 MMAs per k step on the same A and fills
//                all of TMEM (one accumulator buffer).
//
// Up tiles: B = 128 rows of W1_e stacked on the same 128 rows of W3_e, so
// one N = 256 MMA produces a (columns 0-127) and b (128-255) for 128
// hidden units.  Down tiles: B = 256 rows of W2_e per MMA.
//
// In a pair, the last row block of an expert that holds at most 128 rows
// runs as an M = 128 pair MMA (each CTA loads 64 rows of A), so pairs pad
// an expert to a multiple of 128 rows, not 256.  In a pair up tile each
// CTA's part of B is 64 rows of W1 followed by the same 64 rows of W3, so
// that a and b of one hidden unit sit in the same TMEM lane for both MMA
// shapes.
//
// Tiles are enumerated per expert from the device-side offsets (no host
// round trip): expert e owns ceil(M_e / tile rows) row blocks x n_tiles column
// blocks.  The row blocks are taken in groups of G; inside a group the row
// block is the fastest index, so the P tiles that run at the same time cover
// ~G row blocks x P / G column blocks and share both operands through L2.
// G = sqrt(P x tile columns / tile rows) makes the bytes of those distinct
// A rows and B columns least (G x A-tile + P / G x B-tile, with the A and B
// tiles' bytes in proportion to their rows); an expert of at most G row
// blocks is one group (every expert at T = 4096 on Mixtral shapes; at
// T = 16384 with skewed routing the hottest expert has 45).  The down
// projection numbers its short pair tiles after all others.  Tiles are
// handed out dynamically: the producer (the even CTA's, for pairs) takes
// the next tile number from a global counter and passes it to the other
// roles (and to the odd CTA) through a small shared-memory ring, so short
// and full tiles balance across the persistent CTAs.  Weight-streaming
// launches (32-row tiles) run in even waves and start their first weight
// loads before the dependency wait (see below).  Ragged row blocks read the
// next expert's rows (or the zero fill past the end) and simply do not
// store them; ragged column blocks are masked the same way.
//
// Every mbarrier wait is bounded (4 s of globaltimer): on expiry the waiting
// role raises MOE_DEVERR_PIPELINE_TIMEOUT, sets a block-wide abort flag that
// releases the other roles, and the block frees its TMEM and returns.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = 128;            // tile rows (permuted tokens)
constexpr int BK = 64;             // k per stage: 64 bf16 = one 128-byte swizzle row
constexpr int UMMA_K = 16;         // k per tcgen05.mma (kind::f16)
constexpr int A_TILE = BM * BK * 2;            // 16 KiB: 128 rows x 64 k
constexpr int kEpiWarps = 8;                  // two per TMEM lane quadrant
constexpr int NUM_THREADS = 64 + 32 * kEpiWarps;
constexpr int TMEM_COLS = 512;                 // 2 accumulators x 256 fp32 columns
constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // default bound of a pipeline wait
constexpr unsigned long long kDrainLimitNs = 1000000000ull;  // bound of the exit drain of issued MMAs
constexpr unsigned long long kQuiesceNs = 100000ull;         // after an abort: copies in flight land


enum Mode { kUp = 0, kDown = 1 };

struct KParams {
    const int32_t* offsets;  // [E+1]
    int E;
    int n_out;               // f (up) or d (down): valid output columns
    int Kdim;                // d (up) or f (down)
    int n_tiles;             // column tiles per expert
    int b_rows_per_expert;   // f (up) or d (down): expert stride in the 2-D weight view
    __nv_bfloat16* h;        // up output [rows, f]
    const int32_t* perm;     // down: assignment of each permuted row
    const int32_t* inv;      // down: permuted row of each assignment [T*k]
    const float* topk_w;     // down: gate weights [T*k]
    float* obuf;             // down: parked gate-scaled rows [rows, d] (fp32)
    unsigned int* arrivals;  // down: [T, ceil(d / 128)] slot arrival counters, zero at launch
    __nv_bfloat16* y;        // down: layer output [T, d]
    const __nv_bfloat16* residual;  // down: added to y after the slot sum, or null
    int k;                   // experts per token
    int rows;                // T*k
    unsigned int* err;       // device error word (MOE_DEVERR_*)
    int row_mode;            // rows of each expert to cover: kAllRows, kFullPairBlocks or kPairRemainders
    int* tile_counter;       // next tile to hand out; zero at launch (the row gather zeroes it)
    unsigned long long wait_limit_ns;  // bound of every pipeline wait
    int stall_test;          // failure-detection test: the epilogue waits on a barrier nothing completes
    int m_group;             // row blocks per group of the tile order (>= 1)
};

// Row ranges: all rows of each expert; only its whole 256-row blocks; or
// only the rows after them.  A layer can run the pair kernel on the blocks
// and the single-CTA kernel (128-row tiles, less padding) on the rest.
enum RowMode { kAllRows = 0, kFullPairBlocks = 1, kPairRemainders = 2 };

// ---------------------------------------------------------------------------
// PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait with cluster-scope acquire: for barriers completed by the other
// CTA of a pair, whose shared-memory writes must be visible after the wait.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor for a K-major tile written by TMA with
// 128-byte swizzle: rows of 128 bytes, 8-row core groups 1024 bytes apart
// (stride byte offset), leading byte offset unused (1), version 1 (bit 46),
// layout SWIZZLE_128B (2 in bits 61-63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
          "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
          "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Epilogue helpers

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// SiLU(a) * b with the logistic sigma(a) = (1 + tanh(a / 2)) / 2 (an exact
// identity) on the hardware tanh approximation: one special-function op per
// output instead of an exponential and a reciprocal, which bound the
// epilogue's throughput.  The approximation's absolute error (about 2^-11)
// gives |error of SiLU(a)| <= |a| * 2^-12, below the bf16 rounding of h for
// a >= 0 and about that of one bf16 ulp of a * b elsewhere.
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float silu_mul(float a, float b) {
    const float sig = fmaf(0.5f, tanh_approx(0.5f * a), 0.5f);
    return a * sig * b;
}

// ---------------------------------------------------------------------------
// Pair (cta_group::2) helpers

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared::cluster address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// Bulk tensor load of this CTA's half of a pair tile; completion is counted
// on the mbarrier of the pair's even CTA (the address with the peer bit cleared).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar & 0xFEFFFFFFu)
        : "memory");
}

// A_USE: how the MMA treats the tensor core's collector buffer for A.
// 0: A read from shared memory (no reuse); 1 (fill): read from shared
// memory and kept in the collector; 2 (lastuse): taken from the collector,
// which the previous MMA filled with the same A, and released.  The two
// MMAs of a 256 x 512 pair tile share each A block, so the second one
// reads no A from shared memory.
template <int A_USE = 0>
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    if constexpr (A_USE == 1) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16.collector::a::fill [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
            "l"(a), "l"(b), "r"(idesc), "r"(acc));
    } else if constexpr (A_USE == 2) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16.collector::a::lastuse [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
            "l"(a), "l"(b), "r"(idesc), "r"(acc));
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
            "l"(a), "l"(b), "r"(idesc), "r"(acc));
    }
}

// Arrive-one on the mbarrier at the same offset in both CTAs of the pair when
// the pair's previously issued MMAs complete.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"((uint16_t)0x3)
        : "memory");
}

// Arrive-one on this CTA's own mbarrier when the pair MMAs this thread issued
// complete.
__device__ __forceinline__ void umma_commit_pair_own(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Bulk tensor store of a 32-row box from this CTA's shared memory (async
// proxy); completion is tracked per thread with bulk groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Epilogue staging: each of the 8 epilogue warps owns a 4 KiB buffer
// holding one 32-row x 128-byte output box in the 128-byte swizzled layout
// the store's tensor map expects: 16-byte chunk j of row r sits at
// r * 128 + ((j ^ (r & 7)) << 4), which also makes the 32 lanes'
// shared-memory writes conflict-free.
constexpr int kOutBoxBytes = 32 * 128;
// Whole 32-row boxes go out through shared memory and bulk tensor stores.
// (false: every lane stores its row's 128-byte line directly; measured on
// B200 slower: prefill +81 us, skewed +348 us per layer.)
constexpr bool kStagedStores = true;
constexpr int kOutBytes = kEpiWarps * kOutBoxBytes;

// ---------------------------------------------------------------------------
// Per-variant constants.  BN = accumulator columns of a tile (the MMA's N):
// 256 or 128.  CG = 1: one CTA per 128-row tile, the whole BN-row B tile in
// its own shared memory.  CG = 2: a CTA pair per 256-row tile; each CTA
// holds its 128 rows of A and its BN/2-row half of B; the even CTA issues
// M = 256 MMAs that read both CTAs' shared memory and write both CTAs' TMEM.
// A short pair tile (an expert's last block, at most 128 rows) loads 64 rows
// of A per CTA and issues M = 128 MMAs; each CTA's 64 x BN accumulator then
// occupies TMEM lanes 0-63 for columns 0 .. BN/2-1 and lanes 64-127 for
// columns BN/2 .. BN-1, both at column offsets 0 .. BN/2-1 (the 2x2
// datapath layout of the 2-SM M = 128 shape).
// NH (pairs only): MMAs of N = BN per tile along N.  NH = 2 makes a 256 x 2BN
// tile: both MMAs of a k step share the A tile, so each CTA loads A once per
// 2 BN columns (a quarter fewer bytes per MMA than NH = 1), and each CTA's
// B stage holds NH parts of BN/2 rows, part h feeding MMA h.  The two
// accumulators then fill all 512 TMEM columns, so there is one accumulator
// buffer and the epilogue of a tile is not overlapped with the next tile's
// MMAs (NH = 1 keeps two buffers and overlaps them).
// The stage ring fills 192 KiB of shared memory.
//
// Instruction descriptor (kind::f16): D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 in
// bits 17-22, M >> 4 in bits 24-28.

template <int CG, int BN, int RB, int NH = 1>
struct Cfg {
    // RB (single CTA only): token rows loaded per tile, 128 or 32.  With 32
    // the TMA fills only the first 32 rows of the 128-row A buffer; the MMA
    // still computes 128 rows, and rows 32..127 (stale shared memory) give
    // accumulator rows that are never stored: row i of the product depends
    // on row i of A alone.  For decode, where experts hold a few rows each.
    static_assert(CG == 1 || RB == 128, "pairs load 128 rows per CTA");
    static_assert(NH == 1 || CG == 2, "two MMAs per tile along N: pairs only");
    static constexpr int kTileRows = (CG == 1) ? RB : 256;   // rows of one tile (pair)
    static constexpr int kABytes = ((CG == 1) ? RB : 128) * BK * 2;  // A bytes loaded per stage
    static constexpr int kBRows = (CG == 1) ? BN : NH * BN / 2;   // B rows held by one CTA
    static constexpr int kBHalf = (BN / 2) * BK * 2;         // bytes of BN/2 rows of B (one part, pairs)
    static constexpr int kBBytes = kBRows * BK * 2;
    static constexpr int kNAcc = (NH == 1) ? 2 : 1;          // accumulator buffers in TMEM
    static constexpr int kTileN = NH * BN;                   // accumulator columns of a tile
    static constexpr int kStageBytes = A_TILE + kBBytes;     // per CTA (A buffer always 128 rows)
    static constexpr int kStages = (196608 / kStageBytes) > 8 ? 8 : (196608 / kStageBytes);
    static constexpr int kSmem = 1024 + kStages * kStageBytes + kOutBytes + 1024;
    static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                       ((uint32_t)((128 * CG) >> 4) << 24);
    // short pair tiles: M = 128 across the pair, 64 rows of A per CTA
    static constexpr int kAShortBytes = 64 * BK * 2;
    static constexpr uint32_t kIdescShort = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                            ((uint32_t)(128 >> 4) << 24);
};

// A pair tile whose rows [start, end) number at most 128 runs as M = 128.
__device__ __forceinline__ bool short_pair_tile(int start, int end) { return end - start <= 128; }

// Tiles of expert e cover rows [s_beg[e], s_end[e]) in blocks of rows_per_tile.
__device__ __forceinline__ int count_tiles_rows(const int* s_beg, const int* s_end, int E, int n_tiles,
                                                int rows_per_tile) {
    int total = 0;
    for (int e = 0; e < E; ++e) total += ((s_end[e] - s_beg[e] + rows_per_tile - 1) / rows_per_tile) * n_tiles;
    return total;
}

// An expert's last row block is short when it holds at most 128 rows (pair
// tiles: an M = 128 MMA).
__device__ __forceinline__ bool short_last_block(int rows, int mt, int rows_per_tile) {
    return mt > 0 && rows - (mt - 1) * rows_per_tile <= 128;
}

// Tile number -> (expert, row block, column block): experts in order; inside
// an expert, groups of G row blocks (the last one may be shorter); inside a
// group, column block major and row block fastest.  With short_last (the
// down projection's pair tiles) the short last row blocks are taken out of
// that order and numbered after all other tiles, expert by expert, so the
// shorter tiles come last and even out the CTA pairs' finishing times.
__device__ __forceinline__ void decode_tile_rows(int tile, const int* s_beg, const int* s_end, int E, int n_tiles,
                                                 int rows_per_tile, int G, bool short_last, int& e, int& m_blk,
                                                 int& n_blk) {
    int base = 0;
    for (e = 0; e < E; ++e) {
        const int rows = s_end[e] - s_beg[e];
        int mt = (rows + rows_per_tile - 1) / rows_per_tile;
        if (short_last && short_last_block(rows, mt, rows_per_tile)) --mt;
        const int tiles = mt * n_tiles;
        if (tile < base + tiles) {
            const int local = tile - base;
            const int g = local / (G * n_tiles);
            const int g0 = g * G;
            const int gs = min(G, mt - g0);  // row blocks of this group
            const int r = local - g0 * n_tiles;
            n_blk = r / gs;
            m_blk = g0 + (r - n_blk * gs);
            return;
        }
        base += tiles;
    }
    if (short_last) {
        for (e = 0; e < E; ++e) {
            const int rows = s_end[e] - s_beg[e];
            const int mt = (rows + rows_per_tile - 1) / rows_per_tile;
            if (!short_last_block(rows, mt, rows_per_tile)) continue;
            if (tile < base + n_tiles) {
                m_blk = mt - 1;
                n_blk = tile - base;
                return;
            }
            base += n_tiles;
        }
    }
    e = E - 1; m_blk = 0; n_blk = 0;  // not reached for tile < total
}

// Bounded wait that, on timeout, also raises the peer CTA's abort flag
// (pairs).  The hot path is a bare try_wait spin; the abort flag and the
// clock are consulted only every 1024 tries, so a phase that completes
// while the waiter spins is seen within one try (a timer read costs
// hundreds of cycles, which would delay the next MMA issue).
template <bool kClusterScope = false>
__device__ __forceinline__ bool wait_bounded_pair(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                  unsigned int* err, uint32_t peer_abort_addr,
                                                  unsigned long long limit_ns) {
    unsigned long long t0 = 0;
    for (uint32_t i = 1;; ++i) {
        if (kClusterScope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
        if ((i & 1023u) == 0) {
            if (*abort_flag) return false;
            const unsigned long long now = globaltimer();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > limit_ns) {
                *abort_flag = 1;
                if (peer_abort_addr) st_cluster_u32(peer_abort_addr, 1u);
                atomicOr(err, 1u);
                return false;
            }
        }
    }
}

// Exit-path wait for work this thread has already issued (the MMAs, which
// need nothing more from any other role to complete): bounded by
// kDrainLimitNs and blind to the abort flag; on expiry it raises the error
// flag and gives up.
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, unsigned int* err) {
    unsigned long long t0 = 0;
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 1023u) == 0) {
            const unsigned long long now = globaltimer();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > kDrainLimitNs) {
                atomicOr(err, 1u);
                return false;
            }
        }
    }
}

// After an abort, bulk copies a producer issued may still be landing in
// shared memory, and some complete on barrier phases that will never finish
// (the other CTA of the pair stopped issuing first), so they cannot be
// waited for one by one: the producer waits kQuiesceNs, many times the
// latency of a copy, before the CTA frees its resources.
__device__ __forceinline__ void quiesce_copies() {
    const unsigned long long t0 = globaltimer();
    while (globaltimer() - t0 < kQuiesceNs) __nanosleep(1000);
}

// Tile-number ring between the producer that takes tiles from the global
// counter and the roles that follow it.  Readers of a slot: the MMA thread
// and the kEpiWarps epilogue warps of the CTA, and for pairs also the odd
// CTA's producer and its epilogue warps (they read the copy the even CTA's
// producer writes into the odd CTA's ring).  The slot's empty barrier lives
// in the even CTA.  A tile number of -1 ends the loops.
constexpr int kSchedSlots = 4;
template <int CG>
struct Sched {
    static constexpr uint32_t kReaders = (CG == 1) ? 1u + kEpiWarps : 2u * (1u + kEpiWarps);
};

// ---------------------------------------------------------------------------
// The combine, fused into the down-projection's epilogue (§2.1 display 3:
// y[t] = sum_j w[t, j] * SwiGLU_{idx[t, j]}(x[t]); Method: the expert results
// are scattered back to the token order).
//
// Every permuted row r (assignment q = perm[r] = t*k + j) first parks its
// gate-scaled fp32 row in obuf[r] with the tile's bulk stores, and the warp
// releases the accumulator.  Then, per group of 128 output columns, each
// lane adds one to the counter of (its token, the group); the arrival that
// brings the counter to the token's number of routed slots is the last one.
// Every other slot parked its row before it counted (bulk-store completion,
// proxy fence, release fence, atomic), so the last arrival reads the k rows
// back, adds them in slot order j = 0, 1, ... (then the residual, if any),
// rounds once to bf16 and stores y[t].  The sum is the same whichever tile
// finishes last, nothing waits on another CTA, and all of it overlaps the
// next tile's main loop.  Counters start at zero (the permutation kernels
// clear them before the GEMMs run).

__device__ __forceinline__ float4 ldcg_f4(const float* a) { return __ldcg(reinterpret_cast<const float4*>(a)); }

// Drops a 128-byte L2 line without writing it back (its contents become
// undefined): a parked row is dead once the last arrival has read it, so a
// line still in L2 then never reaches DRAM.
__device__ __forceinline__ void discard_l2_line(const void* a) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(a) : "memory");
}

// a = v for the first routed slot, a += v after it (slot order)
__device__ __forceinline__ void add_slot(float4& a, const float4& v, bool& first) {
    if (first) {
        a = v;
        first = false;
    } else {
        a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
    }
}

// Rows `m` (a warp-uniform lane mask) are last arrivals of the 128-column
// group that starts at output column c0; lane l sums columns c0 + 4l .. +3
// of each such row's token (t, and the token's slot rows rr0 / rr1 for
// j = 0 / 1, are held by the row's lane).  Eight rows at a time, all their
// loads issued before the sums.
__device__ __forceinline__ void combine_group(unsigned m, int t, int rr0, int rr1, int c0, const KParams& p,
                                           int lane) {
    constexpr int B = 8;
    const int d = p.n_out;
    const unsigned nrows = (unsigned)p.rows;
    const int c = c0 + 4 * lane;
    const bool colok = c < d;  // d is a multiple of 8: four columns are all in or all out
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    while (m) {
        int src[B], tb[B], r0[B], r1[B];
#pragma unroll
        for (int b = 0; b < B; ++b) {
            src[b] = m ? __ffs(m) - 1 : -1;
            m = m ? (m & (m - 1)) : 0u;
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const int s = src[b] < 0 ? 0 : src[b];
            tb[b] = __shfl_sync(0xffffffffu, t, s);
            r0[b] = __shfl_sync(0xffffffffu, rr0, s);
            r1[b] = __shfl_sync(0xffffffffu, rr1, s);
        }
        float4 v0[B], v1[B];
        uint2 rs[B];
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const bool live = src[b] >= 0 && colok;
            v0[b] = (live && (unsigned)r0[b] < nrows) ? ldcg_f4(p.obuf + (size_t)r0[b] * d + c) : zero;
            v1[b] = (live && (unsigned)r1[b] < nrows) ? ldcg_f4(p.obuf + (size_t)r1[b] * d + c) : zero;
            rs[b] = (live && p.residual)
                        ? __ldg(reinterpret_cast<const uint2*>(p.residual + (size_t)tb[b] * d + c))
                        : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
            if (src[b] < 0 || !colok) continue;
            float4 a = zero;
            bool first = true;
            if ((unsigned)r0[b] < nrows) add_slot(a, v0[b], first);
            if ((unsigned)r1[b] < nrows) add_slot(a, v1[b], first);
            for (int j = 2; j < p.k; ++j) {  // slots beyond the first two (general top-k)
                const int r = __ldg(p.inv + (size_t)tb[b] * p.k + j);
                if ((unsigned)r < nrows) add_slot(a, ldcg_f4(p.obuf + (size_t)r * d + c), first);
            }
            if (p.residual) {
                a.x = __uint_as_float(rs[b].x << 16) + a.x;
                a.y = __uint_as_float(rs[b].x & 0xFFFF0000u) + a.y;
                a.z = __uint_as_float(rs[b].y << 16) + a.z;
                a.w = __uint_as_float(rs[b].y & 0xFFFF0000u) + a.w;
            }
            uint2 out;
            out.x = pack_bf16x2(a.x, a.y);
            out.y = pack_bf16x2(a.z, a.w);
            *reinterpret_cast<uint2*>(p.y + (size_t)tb[b] * d + c) = out;
        }
        // the parked rows of slots 0 and 1 are dead: lanes 0-3 and 4-7 drop
        // their 128-byte lines (whole lines of the row only: d % 32 == 0),
        // after every lane's loads of them have returned
        __syncwarp();
        if ((d & 31) == 0 && lane < 8) {
            const int line = lane & 3;
            const int col = c0 + 32 * line;
#pragma unroll
            for (int b = 0; b < B; ++b) {
                const int r = lane < 4 ? r0[b] : r1[b];
                if (src[b] >= 0 && col < d && (unsigned)r < nrows) discard_l2_line(p.obuf + (size_t)r * d + col);
            }
        }
    }
}

template <int MODE, int CG, int BN, int RB, int NH>
__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
                    const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                    const __grid_constant__ CUtensorMap tmOut, const KParams p) {
    using C = Cfg<CG, BN, RB, NH>;
    // pair up tiles interleave 64 rows of W1 and of W3 per CTA (N = 256)
    static_assert(!(CG == 2 && MODE == kUp) || BN == 256, "pair up-projection tiles are 256 columns wide");
    constexpr int STG = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STG * A_TILE;
    uint8_t* sOut = sB + STG * C::kBBytes;  // 1024-aligned: stage sizes are multiples of 1 KiB
    uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + kOutBytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + STG;
    uint64_t* tfull = bars + 2 * STG;
    uint64_t* tempty = bars + 2 * STG + 2;
    uint64_t* sfull = bars + 2 * STG + 4;                 // [kSchedSlots] tile number published
    uint64_t* sempty = sfull + kSchedSlots;               // [kSchedSlots] all readers done (even CTA)
    uint64_t* mma_done = sempty + kSchedSlots;            // the MMA issuer's exit drain
    uint64_t* stall_bar = mma_done + 1;                   // failure-detection test: never completed
    volatile int* stile = reinterpret_cast<volatile int*>(stall_bar + 1);  // [kSchedSlots]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stall_bar + 1) + kSchedSlots;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_beg = reinterpret_cast<int*>(tmem_slot + 2);  // [E] first row of expert e's range
    int* s_end = s_beg + kMaxExperts;                   // [E] end of expert e's range

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = (CG == 2) ? cluster_rank() : 0u;
    const bool leader = rank == 0;
    const uint32_t peer_abort = (CG == 2) ? map_to_rank(smem_u32((const void*)abort_flag), rank ^ 1u) : 0u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STG; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), kEpiWarps * CG);  // one arrival per epilogue warp of the tile
        }
        for (int q = 0; q < kSchedSlots; ++q) {
            mbar_init(smem_u32(&sfull[q]), 1);
            mbar_init(smem_u32(&sempty[q]), Sched<CG>::kReaders);
        }
        mbar_init(smem_u32(mma_done), 1);
        mbar_init(smem_u32(stall_bar), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        if constexpr (CG == 1) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                         "r"(TMEM_COLS) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                         "r"(TMEM_COLS) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        }
    }
    // The set-up above overlaps the previous kernel's tail.  The A rows, the
    // tile counter and (for the down projection) the arrival counters are
    // written by the kernel launched just before this one, so they are read
    // only after pdl_wait().  Weight-streaming launches (kEarlyB) read the
    // offsets before it: they come from the kernel that built the
    // permutation (the permutation kernels, or the router of a small
    // layer), launched at least two launches earlier, and the previous
    // kernel let this one start only after its own wait, i.e. after that
    // kernel had completed and its writes were visible.  Their producer then issues the weight loads of
    // its first tile's first stages (the weights are inputs no kernel of the
    // layer writes) before it waits, so the HBM stream starts while the
    // previous kernel finishes.
    constexpr bool kEarlyB = (CG == 1 && RB == 32);
    const bool early_producer = kEarlyB && warp == 0 && lane == 0;
    if constexpr (!kEarlyB) {
        pdl_wait();
        pdl_trigger();
    }
    if (threadIdx.x < p.E) {
        const int o0 = p.offsets[threadIdx.x], o1 = p.offsets[threadIdx.x + 1];
        const int split = o0 + ((o1 - o0) / 256) * 256;  // end of the whole 256-row blocks
        s_beg[threadIdx.x] = (p.row_mode == kPairRemainders) ? split : o0;
        s_end[threadIdx.x] = (p.row_mode == kFullPairBlocks) ? split : o1;
    }
    tc_fence_before();
    if constexpr (CG == 2) cluster_sync_all(); else __syncthreads();
    tc_fence_after();
    if (kEarlyB && !early_producer) {
        pdl_wait();
        pdl_trigger();
    }
    const uint32_t tmem_base = *tmem_slot;

    const int total = count_tiles_rows(s_beg, s_end, p.E, p.n_tiles, C::kTileRows);
    // the down projection's short pair tiles last (the up projection keeps
    // them next to the full tiles that share their weight slices in L2)
    constexpr bool kShortLast = (MODE == kDown && CG == 2);
    // Weight-streaming tiles (32 token rows: HBM-bound) in even waves: with
    // w = ceil(total / grid) waves, only ceil(total / w) CTAs take tiles, so
    // no last wave of a few tiles streams alone while the others idle (at
    // decode 896 tiles run as 7 waves of 128, not 6 of 148 and one of 8).
    // The other CTAs take no tile and leave.
    int active = (int)gridDim.x / CG;
    if constexpr (CG == 1 && RB == 32) {
        const int waves = (total + active - 1) / active;
        if (waves > 0) active = (total + waves - 1) / waves;
    }
    const bool takes_tiles = (int)blockIdx.x / CG < active;
    const int kblocks = (p.Kdim + BK - 1) / BK;
    // a reader of tile-ring slot i: wait for the number, read it, release the slot
    const uint32_t sempty_leader0 = (CG == 2) ? map_to_rank(smem_u32(&sempty[0]), 0) : smem_u32(&sempty[0]);
    auto read_tile = [&](uint32_t i, bool& ok) -> int {
        const uint32_t q = i % kSchedSlots, ph = (i / kSchedSlots) & 1u;
        if (!wait_bounded_pair<CG == 2>(smem_u32(&sfull[q]), ph, abort_flag, p.err, peer_abort, p.wait_limit_ns)) {
            ok = false;
            return -1;
        }
        return stile[q];
    };
    auto release_tile = [&](uint32_t i) {
        const uint32_t q = i % kSchedSlots;
        if constexpr (CG == 2) mbar_arrive_cluster(sempty_leader0 + q * (uint32_t)sizeof(uint64_t));
        else mbar_arrive(smem_u32(&sempty[q]));
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer (both CTAs)
            uint32_t it = 0;
            bool ok = true;
            // The next tile's number is taken while the last STG stages of the
            // current tile are issued, so the atomic's latency is hidden.
            // (the odd CTA of a pair reads the even one's; a CTA beyond the
            // active ones publishes the end at once).  Weight-streaming
            // launches take tile blockIdx.x first, without the counter (it is
            // cleared by the previous kernel), and the counter's numbers
            // after the first wave.
            const int counter_base = kEarlyB ? active : 0;
            int next = leader ? (takes_tiles ? (kEarlyB ? (int)blockIdx.x : atomicAdd(p.tile_counter, 1)) : total) : -1;
            int pre = 0;  // stages of the first tile whose weight loads were issued before the wait
            if constexpr (kEarlyB) {
                if (next < total) {
                    int e, mb, nb;
                    decode_tile_rows(next, s_beg, s_end, p.E, p.n_tiles, C::kTileRows, p.m_group, kShortLast, e, mb, nb);
                    const int rowB0 = e * p.b_rows_per_expert + nb * (MODE == kUp ? BN / 2 : BN);
                    const int rowB1 = (MODE == kUp) ? rowB0 : rowB0 + BN / 2;
                    pre = kblocks < STG ? kblocks : STG;
                    for (int kb = 0; kb < pre; ++kb) {  // fresh stages: nothing to wait for
                        const uint32_t fb = smem_u32(&full[kb]);
                        mbar_arrive_expect_tx(fb, C::kABytes + C::kBBytes);
                        tma_load_2d(smem_u32(sB + kb * C::kBBytes), &tmB0, fb, kb * BK, rowB0);
                        tma_load_2d(smem_u32(sB + kb * C::kBBytes + C::kBHalf), &tmB1, fb, kb * BK, rowB1);
                    }
                }
                pdl_wait();
                pdl_trigger();
            }
            for (uint32_t ti = 0; ok; ++ti) {
                int tile;
                if (leader) {
                    // publish the tile taken (to both CTAs of a pair)
                    const uint32_t q = ti % kSchedSlots, ph = (ti / kSchedSlots) & 1u;
                    if (!wait_bounded_pair<CG == 2>(smem_u32(&sempty[q]), ph ^ 1u, abort_flag, p.err, peer_abort, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tile = next < total ? next : -1;
                    stile[q] = tile;
                    if constexpr (CG == 2) {
                        st_cluster_u32(map_to_rank(smem_u32((const void*)&stile[q]), 1), (uint32_t)tile);
                        mbar_arrive_cluster(map_to_rank(smem_u32(&sfull[q]), 1));
                    }
                    mbar_arrive(smem_u32(&sfull[q]));
                } else {
                    tile = read_tile(ti, ok);
                    if (!ok) break;
                    release_tile(ti);
                }
                if (tile < 0) break;
                int e, mb, nb;
                decode_tile_rows(tile, s_beg, s_end, p.E, p.n_tiles, C::kTileRows, p.m_group, kShortLast, e, mb, nb);
                const int start = s_beg[e] + mb * C::kTileRows;
                const bool shrt = (CG == 2) && short_pair_tile(start, min(s_end[e], start + C::kTileRows));
                const int rowA = start + (int)rank * (shrt ? 64 : 128);
                int rowB0, rowB1;
                if constexpr (CG == 1) {
                    rowB0 = e * p.b_rows_per_expert + nb * (MODE == kUp ? BN / 2 : BN);
                    rowB1 = (MODE == kUp) ? rowB0 : rowB0 + BN / 2;
                } else if constexpr (MODE == kUp) {
                    // part h: this CTA's 64 hidden units of MMA h, W1 rows then
                    // the same W3 rows (rowB0 + h * BN / 2 for part h)
                    rowB0 = e * p.b_rows_per_expert + nb * (NH * BN / 2) + (int)rank * (BN / 4);
                    rowB1 = rowB0;
                } else {
                    // part h: rows rowB0 + h * BN of W2
                    rowB0 = e * p.b_rows_per_expert + nb * (NH * BN) + (int)rank * (BN / 2);
                    rowB1 = rowB0;
                }
                const int kb_next = kblocks > STG ? kblocks - STG : 0;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    if (leader && kb == kb_next) next = counter_base + atomicAdd(p.tile_counter, 1);
                    const uint32_t s = it % STG;
                    const uint32_t ph = (it / STG) & 1u;
                    if constexpr (kEarlyB) {
                        if (ti == 0 && kb < pre) {  // weights already on their way: the A rows only
                            tma_load_2d(smem_u32(sA + s * A_TILE), &tmA, smem_u32(&full[s]), kb * BK, rowA);
                            continue;
                        }
                    }
                    if (!wait_bounded_pair(smem_u32(&empty[s]), ph ^ 1u, abort_flag, p.err, peer_abort, p.wait_limit_ns)) { ok = false; break; }
                    const uint32_t fb = smem_u32(&full[s]);
                    if constexpr (CG == 1) {
                        mbar_arrive_expect_tx(fb, C::kABytes + C::kBBytes);
                        tma_load_2d(smem_u32(sA + s * A_TILE), &tmA, fb, kb * BK, rowA);
                        tma_load_2d(smem_u32(sB + s * C::kBBytes), &tmB0, fb, kb * BK, rowB0);
                        tma_load_2d(smem_u32(sB + s * C::kBBytes + C::kBHalf), &tmB1, fb, kb * BK, rowB1);
                    } else {
                        // both CTAs' bytes are counted on the even CTA's barrier
                        if (leader) mbar_arrive_expect_tx(fb, 2 * ((shrt ? C::kAShortBytes : A_TILE) + C::kBBytes));
                        tma_load_2d_pair(smem_u32(sA + s * A_TILE), shrt ? &tmAs : &tmA, fb, kb * BK, rowA);
#pragma unroll
                        for (int h = 0; h < NH; ++h) {
                            const uint32_t part = smem_u32(sB + s * C::kBBytes + h * C::kBHalf);
                            if constexpr (MODE == kUp) {
                                tma_load_2d_pair(part, &tmB0, fb, kb * BK, rowB0 + h * (BN / 2));
                                tma_load_2d_pair(part + C::kBHalf / 2, &tmB1, fb, kb * BK, rowB1 + h * (BN / 2));
                            } else {
                                tma_load_2d_pair(part, &tmB0, fb, kb * BK, rowB0 + h * BN);
                            }
                        }
                    }
                }
            }
            // Drain: wait until the MMAs have released the last min(it, STG)
            // issued stages (use j of a stage completes phase j / STG of its
            // empty barrier), so no arrival from the pair's commits is still
            // on its way when the CTA exits.
            bool drained = ok;
            if (ok) {
                const uint32_t first = it > (uint32_t)STG ? it - (uint32_t)STG : 0u;
                for (uint32_t j = first; j < it; ++j) {
                    if (!wait_bounded_pair(smem_u32(&empty[j % STG]), (j / STG) & 1u, abort_flag, p.err, peer_abort,
                                           p.wait_limit_ns)) {
                        drained = false;
                        break;
                    }
                }
            }
            if (!drained) quiesce_copies();
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issuer (even CTA)
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (;; ++tcount) {
                const int tile = read_tile(tcount, ok);
                if (!ok) break;
                release_tile(tcount);
                if (tile < 0) break;
                const uint32_t acc = tcount % C::kNAcc;
                const uint32_t use = tcount / C::kNAcc;
                if (!wait_bounded_pair(smem_u32(&tempty[acc]), (use & 1u) ^ 1u, abort_flag, p.err, peer_abort, p.wait_limit_ns)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * C::kTileN;
                uint32_t idesc = C::kIdesc;
                if constexpr (CG == 2) {
                    int e, mb, nb;
                    decode_tile_rows(tile, s_beg, s_end, p.E, p.n_tiles, C::kTileRows, p.m_group, kShortLast, e, mb, nb);
                    const int start = s_beg[e] + mb * C::kTileRows;
                    if (short_pair_tile(start, min(s_end[e], start + C::kTileRows))) idesc = C::kIdescShort;
                }
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t s = it % STG;
                    const uint32_t ph = (it / STG) & 1u;
                    if (!wait_bounded_pair(smem_u32(&full[s]), ph, abort_flag, p.err, peer_abort, p.wait_limit_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = sw128_desc(smem_u32(sA + s * A_TILE));
                    const uint64_t bdesc = sw128_desc(smem_u32(sB + s * C::kBBytes));
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        // advance 16 bf16 = 32 bytes along K inside the swizzle row
                        if constexpr (CG == 1) {
                            umma_bf16(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), C::kIdesc,
                                      (kb | kk) != 0 ? 1u : 0u);
                        } else {
                            // part h of B (kBHalf bytes = kBHalf >> 4 descriptor units)
                            const uint64_t ak = adesc + (uint64_t)(kk * 2);
                            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
                            if constexpr (NH == 2) {
                                umma_bf16_pair<1>(d_tmem, ak, bdesc + (uint64_t)(kk * 2), idesc, accum);
                                umma_bf16_pair<2>(d_tmem + BN, ak, bdesc + (uint64_t)((C::kBHalf >> 4) + kk * 2),
                                                  idesc, accum);
                            } else {
                                umma_bf16_pair(d_tmem, ak, bdesc + (uint64_t)(kk * 2), idesc, accum);
                            }
                        }
                    }
                    if constexpr (CG == 1) umma_commit(smem_u32(&empty[s])); else umma_commit_pair(smem_u32(&empty[s]));
                }
                if (ok) {
                    if constexpr (CG == 1) umma_commit(smem_u32(&tfull[acc])); else umma_commit_pair(smem_u32(&tfull[acc]));
                }
            }
            // Exit drain: every MMA issued here has completed before the block
            // frees its tensor memory and its peer's shared memory goes away
            // (after an abort some were never waited for).
            if (it > 0) {
                if constexpr (CG == 1) umma_commit(smem_u32(mma_done)); else umma_commit_pair_own(smem_u32(mma_done));
                wait_drain(smem_u32(mma_done), 0u, p.err);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue (both CTAs)
        // Two warps per TMEM lane quadrant (warp % 4 selects the lanes a warp
        // may read).  Up: of the tile's 64-hidden-unit segments (over all MMA
        // parts) warp sub = 0 takes the even ones and sub = 1 the odd ones.
        // Down: the quadrant's columns in groups of 128 (four 32-column
        // boxes; the unit of the combine's arrival counters), sub = 0 taking
        // the first half of the groups and sub = 1 the rest.
        const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
        const int sub = (warp - 2) >> 2;
        const uint32_t t_lane = tmem_base + ((uint32_t)(quad * 32) << 16);
        const uint32_t tempty_leader0 = (CG == 2) ? map_to_rank(smem_u32(&tempty[0]), 0) : 0u;
        const uint32_t buf = smem_u32(sOut) + (uint32_t)(warp - 2) * kOutBoxBytes;
        const unsigned nrows = (unsigned)p.rows;
        const int ngrp = (p.n_out + kCombineCols - 1) / kCombineCols;  // down: arrival counters per token
        uint32_t tcount = 0;
        for (;; ++tcount) {
            bool got = true;
            const int tile = read_tile(tcount, got);  // every lane waits and reads
            __syncwarp();
            if (!__all_sync(0xffffffffu, got)) break;
            if (lane == 0) release_tile(tcount);
            if (tile < 0) break;
            int e, mb, nb;
            decode_tile_rows(tile, s_beg, s_end, p.E, p.n_tiles, C::kTileRows, p.m_group, kShortLast, e, mb, nb);
            const uint32_t acc = tcount % C::kNAcc;
            const uint32_t use = tcount / C::kNAcc;
            const int start = s_beg[e] + mb * C::kTileRows;
            const int tile_end = min(s_end[e], start + C::kTileRows);
            // Rows and accumulator columns of this warp's TMEM lanes.  Full
            // tiles: 32 rows, all BN columns.  Short pair tiles: lanes 0-63
            // hold the CTA's 64 rows for columns 0 .. BN/2-1 and lanes 64-127
            // the same rows for BN/2 .. BN-1, so quads 0-1 take the first
            // half of the columns and quads 2-3 the second.
            const bool shrt = (CG == 2) && short_pair_tile(start, tile_end);
            const int colhalf = shrt ? (quad >> 1) : 0;
            const int row = start + (shrt ? (int)rank * 64 + (quad & 1) * 32 : (int)rank * 128 + quad * 32) + lane;
            const bool valid = row < tile_end;
            // rows of this warp: whole box stored by TMA when all 32 are the
            // expert's own; a box straddling the end of the expert's block
            // uses per-row stores (a full-box store would overwrite the next
            // expert's rows)
            const int wrow0 = row - lane;
            const bool box_ok = kStagedStores && wrow0 + 32 <= tile_end;
            // down: the row's assignment, its gate weight, and its token's
            // slot rows, loaded while the tile's MMAs run
            int tok = 0, rr0 = -1, rr1 = -1, nvalid = 0;
            bool row_ok = false;
            float wgt = 0.f;
            if constexpr (MODE == kDown) {
                if (valid) {
                    const int q = __ldg(p.perm + row);
                    if ((unsigned)q < nrows) {
                        row_ok = true;
                        wgt = __ldg(p.topk_w + q);
                        tok = q / p.k;
                        const int32_t* iv = p.inv + (size_t)tok * p.k;
                        rr0 = __ldg(iv);
                        rr1 = p.k > 1 ? __ldg(iv + 1) : -1;
                        nvalid = ((unsigned)rr0 < nrows ? 1 : 0) + ((unsigned)rr1 < nrows ? 1 : 0);
                        for (int j = 2; j < p.k; ++j) nvalid += (unsigned)__ldg(iv + j) < nrows ? 1 : 0;
                    }
                }
            }
            // every lane waits; the decision to stop is warp-uniform so the
            // .sync.aligned TMEM loads below always run on a converged warp
            // (the failure-detection test waits on a barrier that nothing completes)
            const bool okw = p.stall_test
                                 ? wait_bounded_pair(smem_u32(stall_bar), 0u, abort_flag, p.err, peer_abort, p.wait_limit_ns)
                                 : wait_bounded_pair(smem_u32(&tfull[acc]), use & 1u, abort_flag, p.err, peer_abort,
                                                     p.wait_limit_ns);
            if (!__all_sync(0xffffffffu, okw)) break;
            tc_fence_after();
            // down: 128-column groups of this warp, [g_lo, g_hi) of the quadrant's
            // G = NH * gpp groups (gpp per MMA part; part h of a tile covers
            // output columns nb * NH * BN + h * BN ..)
            const int ncol = shrt ? BN / 2 : BN;  // columns of each MMA part held by the quadrant
            const int cbase = colhalf * (BN / 2);
            const int gpp = ncol / kCombineCols;
            const int G = NH * gpp;
            const int g_lo = sub ? (G + 1) / 2 : 0, g_hi = sub ? G : (G + 1) / 2;
            (void)g_lo;
            (void)g_hi;
            bool released = false;  // this warp's TMEM arrival for the tile done
            if constexpr (MODE == kUp) {
                // The tile's output units (64-hidden-unit segments over all MMA
                // parts, part-major); this warp takes units sub, sub + 2, ...,
                // each as two 32-unit halves ("items", at most 4).  64-unit
                // segments: hidden units c64 .. c64+63 of the tile have a at TMEM
                // columns acol .. acol+63 and b at acol+bdelta ...
                //   single CTA: a = columns 0 .. BN/2-1, b = BN/2 .. BN-1;
                //   pair, full: [a 64 | b 64] per CTA half of B, two halves;
                //   pair, short: one half per lane group, at columns 0-127.
                // The TMEM loads of item i+1 are issued before item i's math, and
                // the warp releases the accumulator after its last item's loads
                // have landed, before that item's math and stores.
                const int nseg = (CG == 1) ? BN / 128 : (shrt ? 1 : 2);
                const int n_items = 2 * ((NH * nseg - sub + 1) / 2);
                const int bdelta = (CG == 1) ? BN / 2 : 64;
                __nv_bfloat16* hrow = p.h + (size_t)row * p.n_out;
                auto item_cols = [&](int it, uint32_t& ta, int& hcol) {
                    const int u = sub + 2 * (it >> 1);
                    const int h = u / nseg, seg = u - h * nseg, half = it & 1;
                    const int c64 = (shrt ? colhalf : seg) * 64;  // hidden offset in MMA part h
                    const int acol = (CG == 1) ? seg * 64 : (shrt ? 0 : seg * 128);
                    ta = t_lane + acc * C::kTileN + h * BN + acol + half * 32;
                    hcol = nb * (NH * BN / 2) + h * (BN / 2) + c64 + half * 32;  // first hidden unit
                };
                constexpr int kMaxItems = (NH == 2) ? 4 : 2;
                uint32_t ra[2][32], rb[32];
                if (n_items > 0) {
                    uint32_t ta;
                    int hc;
                    item_cols(0, ta, hc);
                    tmem_ld32(ta, ra[0]);
                    tmem_ld32(ta + bdelta, rb);
                }
#pragma unroll
                for (int it = 0; it < kMaxItems; ++it) {
                    if (it >= n_items) break;  // warp-uniform
                    uint32_t ta;
                    int hc;
                    item_cols(it, ta, hc);
                    tmem_wait_ld();
                    if (it + 1 < n_items) {
                        uint32_t tn;
                        int hn;
                        item_cols(it + 1, tn, hn);
                        tmem_ld32(tn, ra[(it + 1) & 1]);
                    } else {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if constexpr (CG == 1) mbar_arrive(smem_u32(&tempty[acc]));
                            else mbar_arrive_cluster(tempty_leader0 + acc * (uint32_t)sizeof(uint64_t));
                        }
                        released = true;
                    }
                    const uint32_t* a = ra[it & 1];
                    const uint32_t* b = rb;
                    uint4 pk[4];
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        pk[g].x = pack_bf16x2(silu_mul(__uint_as_float(a[g * 8 + 0]), __uint_as_float(b[g * 8 + 0])),
                                              silu_mul(__uint_as_float(a[g * 8 + 1]), __uint_as_float(b[g * 8 + 1])));
                        pk[g].y = pack_bf16x2(silu_mul(__uint_as_float(a[g * 8 + 2]), __uint_as_float(b[g * 8 + 2])),
                                              silu_mul(__uint_as_float(a[g * 8 + 3]), __uint_as_float(b[g * 8 + 3])));
                        pk[g].z = pack_bf16x2(silu_mul(__uint_as_float(a[g * 8 + 4]), __uint_as_float(b[g * 8 + 4])),
                                              silu_mul(__uint_as_float(a[g * 8 + 5]), __uint_as_float(b[g * 8 + 5])));
                        pk[g].w = pack_bf16x2(silu_mul(__uint_as_float(a[g * 8 + 6]), __uint_as_float(b[g * 8 + 6])),
                                              silu_mul(__uint_as_float(a[g * 8 + 7]), __uint_as_float(b[g * 8 + 7])));
                    }
                    if (it + 1 < n_items) {  // b of the next item, now that this one's b is consumed
                        uint32_t tn;
                        int hn;
                        item_cols(it + 1, tn, hn);
                        tmem_ld32(tn + bdelta, rb);
                    }
                    const int half = it & 1;
                    if (box_ok) {
                        if (half == 0) {
                            // the buffer's previous store has read it (waited for
                            // only now, so the wait overlaps the loads and the math)
                            if (lane == 0) bulk_wait_read_all();
                            __syncwarp();
                        }
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            st_shared_v4(buf + lane * 128 + ((((half * 4 + g) ^ (lane & 7))) << 4), pk[g]);
                        if (half == 1) {
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                // a box wholly past the last column is not stored; the
                                // (empty) group keeps one group per staged box
                                const int c64 = hc - 32;
                                if (c64 < p.n_out) tma_store_2d(&tmOut, buf, c64, wrow0);
                                bulk_commit();
                            }
                        }
                    } else if (valid) {
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            if (hc + g * 8 < p.n_out) *reinterpret_cast<uint4*>(hrow + hc + g * 8) = pk[g];
                    }
                }
            } else {
                // park: the gate-scaled fp32 rows of this warp's groups in obuf
                float* orow = p.obuf + (size_t)row * p.n_out;
#pragma unroll 1
                for (int g = g_lo; g < g_hi; ++g) {
                    const int h = g / gpp;
                    const uint32_t tacc = t_lane + acc * C::kTileN + h * BN;
                    const int ob = nb * (NH * BN) + h * BN + cbase;  // output column of TMEM column 0 of part h
#pragma unroll 1
                    for (int u = 0; u < kCombineCols / 32; ++u) {
                        const int cc = (g - h * gpp) * kCombineCols + u * 32;  // TMEM column within part h
                        const int col = ob + cc;
                        uint32_t o[32];
                        tmem_ld32(tacc + cc, o);
                        tmem_wait_ld();
                        uint4 v[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            v[i].x = __float_as_uint(wgt * __uint_as_float(o[i * 4 + 0]));
                            v[i].y = __float_as_uint(wgt * __uint_as_float(o[i * 4 + 1]));
                            v[i].z = __float_as_uint(wgt * __uint_as_float(o[i * 4 + 2]));
                            v[i].w = __float_as_uint(wgt * __uint_as_float(o[i * 4 + 3]));
                        }
                        if (box_ok) {
                            // the buffer's previous store has read it (waited for only
                            // now, so the wait overlaps the load and the scaling)
                            if (lane == 0) bulk_wait_read_all();
                            __syncwarp();
#pragma unroll
                            for (int i = 0; i < 8; ++i) st_shared_v4(buf + lane * 128 + ((i ^ (lane & 7)) << 4), v[i]);
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                if (col < p.n_out) tma_store_2d(&tmOut, buf, col, wrow0);
                                bulk_commit();
                            }
                        } else if (valid) {
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                if (col + i * 4 < p.n_out) *reinterpret_cast<uint4*>(orow + col + i * 4) = v[i];
                        }
                    }
                }
            }
            if (!released) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (CG == 1) mbar_arrive(smem_u32(&tempty[acc]));
                    else mbar_arrive_cluster(tempty_leader0 + acc * (uint32_t)sizeof(uint64_t));
                }
            }
            if constexpr (MODE == kDown) {
                // Count the parked groups (release: the park stores are complete
                // and ordered before the counts), then let the last arrivals sum.
                if (lane == 0) {
                    bulk_wait_all();
                    fence_proxy_async_global();
                }
                __syncwarp();
                __threadfence();
                unsigned last = 0;
                if (row_ok) {
                    for (int g = g_lo; g < g_hi; ++g) {
                        const int h = g / gpp;
                        const int col = nb * (NH * BN) + h * BN + cbase + (g - h * gpp) * kCombineCols;
                        if (col >= p.n_out) continue;
                        const bool is_last =
                            p.k == 1 || atomicAdd(p.arrivals + (size_t)tok * ngrp + col / kCombineCols, 1u) == (unsigned)(nvalid - 1);
                        if (is_last) last |= 1u << (g - g_lo);
                    }
                }
                if (__any_sync(0xffffffffu, last != 0)) {
                    __threadfence();  // acquire: the other slots' parked rows
                    for (int g = g_lo; g < g_hi; ++g) {
                        const unsigned m = __ballot_sync(0xffffffffu, (last >> (g - g_lo)) & 1u);
                        if (!m) continue;
                        const int h = g / gpp;
                        const int col = nb * (NH * BN) + h * BN + cbase + (g - h * gpp) * kCombineCols;
                        combine_group(m, tok, rr0, rr1, col, p, lane);
                    }
                }
            }
        }
        if (lane == 0) bulk_wait_all();  // stores complete before the CTA's shared memory goes away
        __syncwarp();
    }

    tc_fence_before();
    if constexpr (CG == 2) cluster_sync_all(); else __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (CG == 1)
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
    }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps through the driver entry point (no libcuda link).

// Process-wide settings of the test and measurement hooks (moe.h:
// moe_set_gemm_variant, moe_set_wait_test); 0 = automatic / default.
std::atomic<int> g_force_cg{0};         // 1 single-CTA tiles, 2 CTA pairs, 3 hybrid
std::atomic<int> g_force_up_bn{0};      // 128 or 256: single-CTA up-projection tile width
std::atomic<int> g_force_rows{0};       // 32 or 128: token rows of a single-CTA tile
std::atomic<int> g_force_pair_cols{0};  // 256 or 512: columns of a pair tile
std::atomic<unsigned long long> g_wait_limit_ns{kWaitLimitNs};
std::atomic<int> g_stall_test{0};

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
const char* g_init_err = nullptr;
std::once_flag g_once;

void init_encode() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
        g_init_err = "cuTensorMapEncodeTiled is not available from the CUDA driver";
        return;
    }
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

// 2-D row-major [rows, cols] map (bf16 or fp32) with a (box_cols x box_rows)
// box and 128-byte swizzle; box_cols * element size must be 128 bytes.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
              bool fp32 = false) {
    std::call_once(g_once, init_encode);
    if (!g_encode) return false;
    const uint32_t esz = fp32 ? 4 : 2;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * esz};
    cuuint32_t box[2] = {128 / esz, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                          const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Co-resident persistent grid: CTAs (CG = 1) or CTA pairs (CG = 2) that
// fit on the device at once, capped by an upper bound on the tile count.
// Tensor maps of one GEMM: A with 128-, 32- and 64-row boxes (full tiles,
// decode tiles, short pair tiles); B as single-CTA tiles read it (W1 / W3
// halves of BN/2 rows, or W2 in 128-row boxes) and as pair tiles read it
// (64-row W1 / W3 boxes; W2 unchanged); the output in 32-row boxes.
struct GemmMaps {
    CUtensorMap A, A32, A64, B0, B1, B0p, B1p, Out;
};

// Tensor maps of recent calls.  A map is a pure function of its pointer,
// shape and box, so a call whose pointers and sizes equal an earlier one's
// reuses that call's maps (a serving loop or a layer stack repeats them)
// instead of encoding 5-8 maps per GEMM on the host.
struct MapKey {
    int mode, bn;
    const void* p[4];
    int rows, d, f, E;
    bool operator==(const MapKey& o) const {
        return mode == o.mode && bn == o.bn && p[0] == o.p[0] && p[1] == o.p[1] && p[2] == o.p[2] &&
               p[3] == o.p[3] && rows == o.rows && d == o.d && f == o.f && E == o.E;
    }
};
constexpr int kMapCacheSlots = 16;
struct MapCache {
    std::mutex mu;
    MapKey key[kMapCacheSlots];
    GemmMaps maps[kMapCacheSlots];
    int used = 0, next = 0;
} g_map_cache;

bool map_cache_get(const MapKey& k, GemmMaps* out) {
    std::lock_guard<std::mutex> lock(g_map_cache.mu);
    for (int i = 0; i < g_map_cache.used; ++i)
        if (g_map_cache.key[i] == k) {
            *out = g_map_cache.maps[i];
            return true;
        }
    return false;
}

void map_cache_put(const MapKey& k, const GemmMaps& m) {
    std::lock_guard<std::mutex> lock(g_map_cache.mu);
    const int i = g_map_cache.next;
    g_map_cache.key[i] = k;
    g_map_cache.maps[i] = m;
    g_map_cache.next = (i + 1) % kMapCacheSlots;
    if (g_map_cache.used < kMapCacheSlots) ++g_map_cache.used;
}

template <int MODE, int CG, int BN, int RB, int NH = 1>
cudaError_t launch_gemm(const GroupedGemmArgs& a, const CUtensorMap& mA, const CUtensorMap& mAs,
                        const CUtensorMap& mB0, const CUtensorMap& mB1, const CUtensorMap& mOut, const KParams& p0,
                        cudaStream_t s) {
    using C = Cfg<CG, BN, RB, NH>;
    KParams p = p0;
    p.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
    p.stall_test = g_stall_test.load(std::memory_order_relaxed);
    static std::atomic<int> units_cache[64];  // per device and variant; any thread may fill it (same value)
    int dev = 0;
    cudaGetDevice(&dev);
    int units = (dev < 64) ? units_cache[dev].load(std::memory_order_relaxed) : 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    if (CG == 2) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.numAttrs = 1;
    }
    if (!units) {
        cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<MODE, CG, BN, RB, NH>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return e;
        units = a.num_sms / CG;
        if (CG == 2) {
            int clusters = 0;
            cfg.gridDim = dim3(2 * units);
            if (cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_kernel<MODE, CG, BN, RB, NH>, &cfg) == cudaSuccess &&
                clusters > 0 && clusters < units)
                units = clusters;
            cudaGetLastError();  // an unsupported query is not an error for the launch
        }
        if (dev < 64) units_cache[dev].store(units, std::memory_order_relaxed);
    }
    const long long ub = (long long)p.n_tiles * ((a.rows + C::kTileRows - 1) / C::kTileRows + a.E);
    const int grid_units = (int)(ub < units ? ub : units);
    if (grid_units <= 0) return cudaSuccess;
    // row blocks per group of the tile order: sqrt(units x tile columns / tile rows)
    p.m_group = std::max(1, (int)std::lround(std::sqrt((double)grid_units * C::kTileN / C::kTileRows)));
    cfg.gridDim = dim3(grid_units * CG);
    set_pdl(attr[cfg.numAttrs++]);  // after the occupancy query, which takes the cluster attribute only
    return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<MODE, CG, BN, RB, NH>, mA, mAs, mB0, mB1, mOut, p);
}

// Variant choice: 1 = single-CTA tiles, 2 = CTA-pair tiles, 3 = hybrid.
// Measured on B200 with Mixtral shapes (d = 4096, f = 14336, E = 8):
//  * pairs need a third fewer bytes per MMA from L2 than single-CTA tiles,
//    and 256 x 512 pair tiles (two MMAs sharing each A tile, see NH) a
//    quarter fewer again.  Prefill (T = 4096, ~1000 rows per expert), both
//    GEMMs: single up + 256 x 256 pair down 2.50-2.54 ms per layer, pairs
//    256 x 256 for both 2.50 ms, pairs 256 x 512 for both 2.38-2.42 ms;
//    skewed (T = 16384): 10.2, 10.1 and 9.3 ms;
//  * the hybrid (pairs on whole 256-row blocks, then a single-CTA launch on
//    the remaining rows) was slower: the second launch has only 1-2 row
//    tiles per weight tile and streams every expert's weights again;
//  * decode (a few rows per expert): single-CTA tiles of 32 token rows.
// Pairs are used once experts average 512 rows; moe_set_gemm_variant forces
// a variant (all exact; the tests run each).
int choose_cta_group(const GroupedGemmArgs& a, int mode) {
    const int forced = g_force_cg.load(std::memory_order_relaxed);
    if (forced) return forced;
    (void)mode;
    return a.rows >= 512 * a.E ? 2 : 1;
}

}  // namespace

const char* gemm_init_error() {
    std::call_once(g_once, init_encode);
    return g_init_err;
}

int set_gemm_variant(int cta_group, int up_bn, int token_rows, int pair_cols) {
    if (cta_group < 0 || cta_group > 3 || (up_bn && up_bn != 128 && up_bn != 256) ||
        (token_rows && token_rows != 32 && token_rows != 128) ||
        (pair_cols && pair_cols != 256 && pair_cols != 512))
        return -1;
    g_force_cg.store(cta_group);
    g_force_up_bn.store(up_bn);
    g_force_rows.store(token_rows);
    g_force_pair_cols.store(pair_cols);
    return 0;
}

void set_wait_test(unsigned long long wait_limit_ns, int stall) {
    g_wait_limit_ns.store(wait_limit_ns ? wait_limit_ns : kWaitLimitNs);
    g_stall_test.store(stall ? 1 : 0);
}

namespace {

// N width of the up-projection tiles: 256 (128 hidden units of W1 and of
// W3).  128-wide tiles (64 + 64) exist for finer load balance, but measured
// on B200 at decode (T = 32) they were slower (0.336 vs 0.323 ms): twice the
// tiles cost more per-tile work than the shorter last wave saves.
// moe_set_gemm_variant can select them (exact; the tests run both widths).
int choose_up_bn(const GroupedGemmArgs&) {
    const int forced = g_force_up_bn.load(std::memory_order_relaxed);
    return forced ? forced : 256;
}

// Token rows per single-CTA tile: 32 when experts average at most 16 rows
// (decode), so tiles do not stream 128 mostly unused A rows from L2 for every
// weight tile; 128 otherwise (or as moe_set_gemm_variant forces).
int choose_rb(const GroupedGemmArgs& a) {
    const int forced = g_force_rows.load(std::memory_order_relaxed);
    if (forced) return forced;
    return a.rows <= 16 * a.E ? 32 : 128;
}

// Pair tiles of 256 x 512 (two N = 256 MMAs sharing each A tile; default)
// or 256 x 256 (two TMEM accumulator buffers, epilogue overlapped).
bool choose_wide(const GroupedGemmArgs&) {
    const int forced = g_force_pair_cols.load(std::memory_order_relaxed);
    return forced ? forced == 512 : true;
}

template <int MODE, int BN>
cudaError_t launch_variant(const GroupedGemmArgs& a, const GemmMaps& m, const KParams& p, cudaStream_t s) {
    // pairs: 256-column tiles only (the up-projection's interleaved B halves)
    const int cg = (MODE == kUp && BN != 256) ? 1 : choose_cta_group(a, MODE);
    if constexpr (MODE == kDown || BN == 256) {
        if (cg == 2 && choose_wide(a)) {
            // 256 x 512 pair tiles: twice the columns per tile
            KParams pw = p;
            const int cols = (MODE == kUp) ? BN : 2 * BN;  // output columns of a wide tile
            pw.n_tiles = (p.n_out + cols - 1) / cols;
            return launch_gemm<MODE, 2, BN, 128, 2>(a, m.A, m.A64, m.B0p, m.B1p, m.Out, pw, s);
        }
        if (cg == 2) return launch_gemm<MODE, 2, BN, 128>(a, m.A, m.A64, m.B0p, m.B1p, m.Out, p, s);
        if (cg == 3) {  // hybrid: pairs on whole 256-row blocks, then single CTAs on the rest (same stream)
            KParams pf = p, pr = p;
            pf.row_mode = kFullPairBlocks;
            pr.row_mode = kPairRemainders;
            pr.tile_counter = p.tile_counter + 1;  // the second launch has its own counter
            cudaError_t e = launch_gemm<MODE, 2, BN, 128>(a, m.A, m.A64, m.B0p, m.B1p, m.Out, pf, s);
            if (e != cudaSuccess) return e;
            return launch_gemm<MODE, 1, BN, 128>(a, m.A, m.A, m.B0, m.B1, m.Out, pr, s);
        }
    }
    return choose_rb(a) == 32 ? launch_gemm<MODE, 1, BN, 32>(a, m.A32, m.A32, m.B0, m.B1, m.Out, p, s)
                              : launch_gemm<MODE, 1, BN, 128>(a, m.A, m.A, m.B0, m.B1, m.Out, p, s);
}

}  // namespace

cudaError_t launch_up_swiglu(const GroupedGemmArgs& a, const __nv_bfloat16* x_perm,
                             const __nv_bfloat16* W1, const __nv_bfloat16* W3, __nv_bfloat16* h,
                             cudaStream_t s) {
    // pairs and the hybrid use 256-column tiles whatever the forced width
    const int bn = choose_cta_group(a, kUp) == 1 ? choose_up_bn(a) : 256;
    GemmMaps m;
    const MapKey key{kUp, bn, {x_perm, W1, W3, h}, a.rows, a.d, a.f, a.E};
    if (!map_cache_get(key, &m)) {
        if (!make_map(&m.A, x_perm, (uint64_t)a.rows, (uint64_t)a.d, BM) ||
            !make_map(&m.A32, x_perm, (uint64_t)a.rows, (uint64_t)a.d, 32) ||
            !make_map(&m.A64, x_perm, (uint64_t)a.rows, (uint64_t)a.d, 64) ||
            !make_map(&m.B0, W1, (uint64_t)a.E * a.f, (uint64_t)a.d, bn / 2) ||
            !make_map(&m.B1, W3, (uint64_t)a.E * a.f, (uint64_t)a.d, bn / 2) ||
            !make_map(&m.B0p, W1, (uint64_t)a.E * a.f, (uint64_t)a.d, 64) ||
            !make_map(&m.B1p, W3, (uint64_t)a.E * a.f, (uint64_t)a.d, 64) ||
            !make_map(&m.Out, h, (uint64_t)a.rows, (uint64_t)a.f, 32))
            return cudaErrorInvalidValue;
        map_cache_put(key, m);
    }
    KParams p{};
    p.offsets = a.offsets; p.E = a.E; p.n_out = a.f; p.Kdim = a.d;
    p.n_tiles = (a.f + bn / 2 - 1) / (bn / 2); p.b_rows_per_expert = a.f; p.h = h; p.rows = a.rows;
    p.err = a.err;
    p.tile_counter = a.tile_counters + 0;
    return bn == 128 ? launch_variant<kUp, 128>(a, m, p, s) : launch_variant<kUp, 256>(a, m, p, s);
}

cudaError_t launch_down_combine(const GroupedGemmArgs& a, const DownCombineArgs& c, cudaStream_t s) {
    GemmMaps m;
    const MapKey key{kDown, 256, {c.h, c.W2, c.obuf, nullptr}, a.rows, a.d, a.f, a.E};
    if (!map_cache_get(key, &m)) {
        if (!make_map(&m.A, c.h, (uint64_t)a.rows, (uint64_t)a.f, BM) ||
            !make_map(&m.A32, c.h, (uint64_t)a.rows, (uint64_t)a.f, 32) ||
            !make_map(&m.A64, c.h, (uint64_t)a.rows, (uint64_t)a.f, 64) ||
            !make_map(&m.B0, c.W2, (uint64_t)a.E * a.d, (uint64_t)a.f, 128) ||
            !make_map(&m.Out, c.obuf, (uint64_t)a.rows, (uint64_t)a.d, 32, true))
            return cudaErrorInvalidValue;
        m.B1 = m.B0;
        m.B0p = m.B0;
        m.B1p = m.B0;
        map_cache_put(key, m);
    }
    KParams p{};
    p.offsets = a.offsets; p.E = a.E; p.n_out = a.d; p.Kdim = a.f;
    p.n_tiles = (a.d + 255) / 256; p.b_rows_per_expert = a.d;
    p.perm = c.perm; p.inv = c.inv; p.topk_w = c.topk_w; p.obuf = c.obuf;
    p.arrivals = c.arrivals; p.y = c.y; p.residual = c.residual; p.k = c.k;
    p.rows = a.rows;
    p.err = a.err;
    p.tile_counter = a.tile_counters + 2;
    return launch_variant<kDown, 256>(a, m, p, s);
}

}  // namespace moe
