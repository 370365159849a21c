// Grouped expert GEMMs on the 5th-generation tensor cores (sm_100a).
//
//   up   (SwiGLU expert, first half; "Mixtral of Experts" §2.1, Method:
//         SwiGLU expert):  for every permuted row r of expert e,
//         a = W1_e x_r, b = W3_e x_r (fp32 in tensor memory),
//         h_r = SiLU(a) * b rounded to bf16.
//   down (second half and the gate weighting of §2.1 display 3):
//         obuf_r = topk_w[perm[r]] * (W2_e h_r), fp32.
//
// Both are one persistent, warp-specialised kernel over output tiles of
// 128 permuted rows:
//   warp 0      TMA producer: 2-D tiled bulk copies (128-byte swizzle) of the
//               A tile (128 rows x 64 k) and the B tile (256 rows x 64 k)
//               into a 4-stage shared-memory ring, signalled on mbarriers;
//   warp 1      MMA issuer: one thread issues tcgen05.mma (bf16 x bf16 ->
//               fp32, M = 128, N = 256, K = 16) into a tensor-memory (TMEM)
//               accumulator and releases ring stages with tcgen05.commit;
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (each warp owns the
//               32 TMEM lanes = tile rows of its quadrant), fused SiLU(a)*b
//               or gate scaling, and the stores.
// TMEM holds two 256-column accumulators, so the epilogue of one tile
// overlaps the main loop of the next.
//
// Up tiles: B = 128 rows of W1_e stacked on the same 128 rows of W3_e, so
// one N = 256 MMA produces a (columns 0-127) and b (128-255) for 128
// hidden units.  Down tiles: B = 256 rows of W2_e.
//
// Tiles are enumerated per expert from the device-side offsets (no host
// round trip): expert e owns ceil(M_e / 128) row blocks x n_tiles column
// blocks, numbered with the row block fastest so that the CTAs running at
// the same time share weight tiles through L2.  Ragged row blocks read the
// next expert's rows (or the zero fill past the end) and simply do not
// store them; ragged column blocks are masked the same way.
//
// Every mbarrier wait is bounded (4 s of globaltimer): on expiry the waiting
// role raises MOE_DEVERR_PIPELINE_TIMEOUT, sets a block-wide abort flag that
// releases the other roles, and the block frees its TMEM and returns.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = 128;            // tile rows (permuted tokens)
constexpr int BK = 64;             // k per stage: 64 bf16 = one 128-byte swizzle row
constexpr int UMMA_K = 16;         // k per tcgen05.mma (kind::f16)
constexpr int MMA_N = 256;         // accumulator columns per tile
constexpr int STAGES = 4;
constexpr int A_TILE = BM * BK * 2;            // 16 KiB
constexpr int B_TILE = MMA_N * BK * 2;         // 32 KiB
constexpr int B_HALF = B_TILE / 2;             // 128 rows
constexpr int STAGE_BYTES = A_TILE + B_TILE;   // 48 KiB
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;                 // 2 accumulators x 256 fp32 columns
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 1024;
constexpr unsigned long long kTimeoutNs = 4000000000ull;

// Instruction descriptor (kind::f16): D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15, 16 = 0),
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                            ((uint32_t)(MMA_N >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

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
    const float* topk_w;     // down: gate weights [T*k]
    float* obuf;             // down output [rows, d]
    int rows;                // T*k
    unsigned int* err;       // device error word (MOE_DEVERR_*)
};

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

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait: true when the phase completed, false on abort or timeout.
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kTimeoutNs) {
            *abort_flag = 1;
            atomicOr(err, 1u);
            return false;
        }
    }
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

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(kIdesc), "r"(acc));
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
// Tile enumeration from the expert offsets (identical in every role).

__device__ __forceinline__ int count_tiles(const int* s_off, int E, int n_tiles) {
    int total = 0;
    for (int e = 0; e < E; ++e) total += ((s_off[e + 1] - s_off[e] + BM - 1) / BM) * n_tiles;
    return total;
}

__device__ __forceinline__ void decode_tile(int tile, const int* s_off, int E, int n_tiles, int& e,
                                            int& m_blk, int& n_blk) {
    int base = 0;
    for (e = 0; e < E; ++e) {
        const int mt = (s_off[e + 1] - s_off[e] + BM - 1) / BM;
        const int tiles = mt * n_tiles;
        if (tile < base + tiles) {
            const int local = tile - base;
            n_blk = local / mt;
            m_blk = local - n_blk * mt;
            return;
        }
        base += tiles;
    }
    e = E - 1; m_blk = 0; n_blk = 0;  // not reached for tile < total
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float silu_mul(float a, float b) {
    return __fdividef(a, 1.0f + __expf(-a)) * b;
}

// ---------------------------------------------------------------------------

template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const KParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_TILE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_TILE);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = bars + 2 * STAGES + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_off = reinterpret_cast<int*>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 128);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (threadIdx.x <= p.E) s_off[threadIdx.x] = p.offsets[threadIdx.x];
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total = count_tiles(s_off, p.E, p.n_tiles);
    const int kblocks = (p.Kdim + BK - 1) / BK;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                int e, mb, nb;
                decode_tile(tile, s_off, p.E, p.n_tiles, e, mb, nb);
                const int rowA = s_off[e] + mb * BM;
                const int rowB0 = e * p.b_rows_per_expert + nb * (MODE == kUp ? 128 : 256);
                const int rowB1 = (MODE == kUp) ? rowB0 : rowB0 + 128;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!wait_bounded(smem_u32(&empty[s]), ph ^ 1u, abort_flag, p.err)) { ok = false; break; }
                    const uint32_t fb = smem_u32(&full[s]);
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(smem_u32(sA + s * A_TILE), &tmA, fb, kb * BK, rowA);
                    tma_load_2d(smem_u32(sB + s * B_TILE), &tmB0, fb, kb * BK, rowB0);
                    tma_load_2d(smem_u32(sB + s * B_TILE + B_HALF), &tmB1, fb, kb * BK, rowB1);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++tcount) {
                const uint32_t acc = tcount & 1u;
                const uint32_t use = tcount >> 1;
                if (!wait_bounded(smem_u32(&tempty[acc]), (use & 1u) ^ 1u, abort_flag, p.err)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * MMA_N;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!wait_bounded(smem_u32(&full[s]), ph, abort_flag, p.err)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = sw128_desc(smem_u32(sA + s * A_TILE));
                    const uint64_t bdesc = sw128_desc(smem_u32(sB + s * B_TILE));
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        // advance 16 bf16 = 32 bytes along K inside the swizzle row
                        umma_bf16(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2),
                                  (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&empty[s]));
                }
                if (ok) umma_commit(smem_u32(&tfull[acc]));
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue
        const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
        const int r_in = quad * 32 + lane;
        const uint32_t t_lane = tmem_base + ((uint32_t)(quad * 32) << 16);
        uint32_t tcount = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
            int e, mb, nb;
            decode_tile(tile, s_off, p.E, p.n_tiles, e, mb, nb);
            const uint32_t acc = tcount & 1u;
            const uint32_t use = tcount >> 1;
            // every lane waits; the decision to stop is warp-uniform so the
            // .sync.aligned TMEM loads below always run on a converged warp
            const bool ok = wait_bounded(smem_u32(&tfull[acc]), use & 1u, abort_flag, p.err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int row = s_off[e] + mb * BM + r_in;
            const bool valid = row < s_off[e + 1];
            const uint32_t tacc = t_lane + acc * MMA_N;
            if constexpr (MODE == kUp) {
                __nv_bfloat16* hrow = p.h + (size_t)row * p.n_out;
#pragma unroll 1
                for (int c = 0; c < 128; c += 32) {
                    uint32_t a[32], b[32];
                    tmem_ld32(tacc + c, a);
                    tmem_ld32(tacc + 128 + c, b);
                    tmem_wait_ld();
                    const int col0 = nb * 128 + c;
                    if (valid) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            if (col0 + g * 8 < p.n_out) {
                                uint4 pk;
                                pk.x = pack_bf16x2(silu_mul(__uint_as_float(a[g * 8 + 0]), __uint_as_float(b[g * 8 + 0])),
                                                   silu_mul(__uint_as_float(a[g * 8 + 1]), __uint_as_float(b[g * 8 + 1])));
                                pk.y = pack_bf16x2(silu_mul(__uint_as_float(a[g * 8 + 2]), __uint_as_float(b[g * 8 + 2])),
                                                   silu_mul(__uint_as_float(a[g * 8 + 3]), __uint_as_float(b[g * 8 + 3])));
                                pk.z = pack_bf16x2(silu_mul(__uint_as_float(a[g * 8 + 4]), __uint_as_float(b[g * 8 + 4])),
                                                   silu_mul(__uint_as_float(a[g * 8 + 5]), __uint_as_float(b[g * 8 + 5])));
                                pk.w = pack_bf16x2(silu_mul(__uint_as_float(a[g * 8 + 6]), __uint_as_float(b[g * 8 + 6])),
                                                   silu_mul(__uint_as_float(a[g * 8 + 7]), __uint_as_float(b[g * 8 + 7])));
                                *reinterpret_cast<uint4*>(hrow + col0 + g * 8) = pk;
                            }
                        }
                    }
                }
            } else {
                float wgt = 0.f;
                if (valid) {
                    const int q = p.perm[row];
                    wgt = ((unsigned)q < (unsigned)p.rows) ? p.topk_w[q] : 0.f;
                }
                float* orow = p.obuf + (size_t)row * p.n_out;
#pragma unroll 1
                for (int c = 0; c < MMA_N; c += 32) {
                    uint32_t o[32];
                    tmem_ld32(tacc + c, o);
                    tmem_wait_ld();
                    const int col0 = nb * 256 + c;
                    if (valid) {
#pragma unroll
                        for (int g = 0; g < 8; ++g) {
                            if (col0 + g * 4 < p.n_out) {
                                float4 v;
                                v.x = wgt * __uint_as_float(o[g * 4 + 0]);
                                v.y = wgt * __uint_as_float(o[g * 4 + 1]);
                                v.z = wgt * __uint_as_float(o[g * 4 + 2]);
                                v.w = wgt * __uint_as_float(o[g * 4 + 3]);
                                *reinterpret_cast<float4*>(orow + col0 + g * 4) = v;
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty[acc]));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps through the driver entry point (no libcuda link).

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

// 2-D bf16 row-major [rows, cols] map with a (64 x box_rows) box, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    std::call_once(g_once, init_encode);
    if (!g_encode) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t ensure_smem_attr() {
    static bool done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && done[dev]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e == cudaSuccess && dev < 64) done[dev] = true;
    return e;
}

// Persistent grid: one CTA per SM, or fewer if there cannot be that many tiles.
int gemm_grid(const GroupedGemmArgs& a, int n_tiles) {
    const long long ub = (long long)n_tiles * ((a.rows + BM - 1) / BM + a.E);
    return (int)(ub < a.num_sms ? ub : a.num_sms);
}

}  // namespace

const char* gemm_init_error() {
    std::call_once(g_once, init_encode);
    return g_init_err;
}

cudaError_t launch_up_swiglu(const GroupedGemmArgs& a, const __nv_bfloat16* x_perm,
                             const __nv_bfloat16* W1, const __nv_bfloat16* W3, __nv_bfloat16* h,
                             cudaStream_t s) {
    CUtensorMap mA, mB0, mB1;
    if (!make_map(&mA, x_perm, (uint64_t)a.rows, (uint64_t)a.d, BM) ||
        !make_map(&mB0, W1, (uint64_t)a.E * a.f, (uint64_t)a.d, 128) ||
        !make_map(&mB1, W3, (uint64_t)a.E * a.f, (uint64_t)a.d, 128))
        return cudaErrorInvalidValue;
    KParams p{};
    p.offsets = a.offsets; p.E = a.E; p.n_out = a.f; p.Kdim = a.d;
    p.n_tiles = (a.f + 127) / 128; p.b_rows_per_expert = a.f; p.h = h; p.rows = a.rows;
    p.err = a.err;
    cudaError_t e = ensure_smem_attr<kUp>();
    if (e != cudaSuccess) return e;
    grouped_gemm_kernel<kUp><<<gemm_grid(a, p.n_tiles), NUM_THREADS, SMEM_BYTES, s>>>(mA, mB0, mB1, p);
    return cudaGetLastError();
}

cudaError_t launch_down_scaled(const GroupedGemmArgs& a, const __nv_bfloat16* h,
                               const __nv_bfloat16* W2, const int32_t* perm, const float* topk_w,
                               float* obuf, cudaStream_t s) {
    CUtensorMap mA, mB;
    if (!make_map(&mA, h, (uint64_t)a.rows, (uint64_t)a.f, BM) ||
        !make_map(&mB, W2, (uint64_t)a.E * a.d, (uint64_t)a.f, 128))
        return cudaErrorInvalidValue;
    KParams p{};
    p.offsets = a.offsets; p.E = a.E; p.n_out = a.d; p.Kdim = a.f;
    p.n_tiles = (a.d + 255) / 256; p.b_rows_per_expert = a.d;
    p.perm = perm; p.topk_w = topk_w; p.obuf = obuf; p.rows = a.rows;
    p.err = a.err;
    cudaError_t e = ensure_smem_attr<kDown>();
    if (e != cudaSuccess) return e;
    grouped_gemm_kernel<kDown><<<gemm_grid(a, p.n_tiles), NUM_THREADS, SMEM_BYTES, s>>>(mA, mB, mB, p);
    return cudaGetLastError();
}

}  // namespace moe
