// pointwise_tc.cu -- pointwise (1x1) dgrad on the Blackwell tensor cores.
//
// For a 1x1 filter with stride 1, no padding and one group, dgrad is a plain
// GEMM: dX[M][C] = dY[M][K] * W[K][C] with M = N*H*W, and every address is an
// affine function of (m, k, c) -- dY at m*K + k, W at k*C + c, dX at m*C + c
// ("add the pointwise fast path dgrad was missing", Technical Details and the
// fast-path commit).  Here the K-loop holds no address arithmetic at all: TMA
// moves whole tiles by coordinate and the tensor cores consume them from shared
// memory through descriptors.
//
// Kernel structure (persistent, one CTA per SM, 192 threads):
//   warp 0      TMA producer: dY tile 128 x 64 (K-major) and W tile 64 x BN
//               (C contiguous, i.e. MN-major for the MMA) into a STAGES-deep ring.
//   warp 1      allocates 2*BN TMEM columns, then one lane issues
//               tcgen05.mma (M=128, N=BN, K=16) into one of two accumulators.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (each warp may read the
//               32 TMEM lanes of its quarter), round to bf16 (nearest even),
//               16-byte stores to dX.  The second accumulator lets the MMAs of
//               the next tile run while this one drains.
// Tiles are taken round-robin in (m-block, n-block) order with n fastest, so
// the CTAs working at one time share their dY rows through L2.
//
// Every wait is bounded (common.cuh); on a timeout the kernel records it in the
// status word, raises a CTA-wide abort flag, lets in-flight copies and MMAs land
// and frees its tensor memory before returning.
#include "common.cuh"
#include "host_util.h"
#include "launchers.h"

namespace dgrad {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 192;

template <int BN, int STAGES>
struct PwTcLayout {
    static constexpr int kABytes = kBM * kBK * 2;   // 16 KB
    static constexpr int kBBytes = kBK * BN * 2;    // 8 KB per 64 columns
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kTileBytes = STAGES * kStageBytes;
    static constexpr int kNumBars = 2 * STAGES + 5;  // full, empty, tmem full x2, tmem empty x2, drain
    static constexpr int kBytes = kTileBytes + kNumBars * 8 + 16;
    static constexpr int kAlloc = kBytes + 1024;     // slack to align the tiles to 1024 bytes
    static constexpr uint32_t kTmemCols = 2 * BN;
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    pw_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 __nv_bfloat16* __restrict__ dX, int M, int C, int K, int* status)
{
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    using L = PwTcLayout<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kTileBytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (M + kBM - 1) / kBM;
    const int num_n = (C + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int num_kb = (K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol_b = policy_evict_last();   // W is re-read by every tile
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                const int m_blk = t / num_n;
                const int n_blk = t - m_blk * num_n;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
                    uint8_t* a_tile = smem + stage * L::kStageBytes;
                    uint8_t* b_tile = a_tile + L::kABytes;
                    tma_load_2d(a_tile, &map_a, &full[stage], kb * kBK, m_blk * kBM);
#pragma unroll
                    for (int j = 0; j < BN / 64; ++j)
                        tma_load_2d_hint(b_tile + j * 8192, &map_b, &full[stage], n_blk * BN + j * 64, kb * kBK,
                                         pol_b);
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                report_timeout(status);
                *abort_flag = 1;
            }
            // Let the last copies land before the CTA may exit.
            for (long long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
                const int s = static_cast<int>(i % STAGES);
                const uint32_t par = static_cast<uint32_t>((i / STAGES) & 1);
                if (!mbar_wait(&full[s], par)) {
                    report_timeout(status);
                    *abort_flag = 1;
                }
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, /*b_mn_major=*/true);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + stage * L::kStageBytes);
                    const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        // A: advance 16 k (32 bytes) inside the 128-byte swizzled row.
                        const uint64_t a_desc = sw128_desc(a_addr + kk * 32, 16, 1024);
                        // B: advance 16 k-rows (2 groups of 8 rows of 128 bytes).
                        const uint64_t b_desc = sw128_desc(b_addr + kk * 2048, 8192, 1024);
                        umma_f16(d_tmem, a_desc, b_desc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);   // frees the stage once these MMAs have read it
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);         // accumulator complete
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) {
                report_timeout(status);
                *abort_flag = 1;
            }
            umma_commit(drain);                   // all MMAs issued above have finished
            if (!mbar_wait(drain, 0)) {
                report_timeout(status);
                *abort_flag = 1;
            }
        }
    } else {
        // ----------------------------------------------------------- epilogue
        const int quarter = warp & 3;             // TMEM lanes this warp may read
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
            const int m_blk = t / num_n;
            const int n_blk = t - m_blk * num_n;
            if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int m = m_blk * kBM + row;
            __nv_bfloat16* out_row = dX + static_cast<int64_t>(m) * C;
#pragma unroll 1
            for (int chunk = 0; chunk < BN / 32; ++chunk) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(acc * BN + chunk * 32), v);
                tmem_wait_ld();
                const int col0 = n_blk * BN + chunk * 32;
                if (m < M) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int col = col0 + g * 8;
                        if (col < C) {
                            uint4 o;
                            o.x = float2_to_bf16x2(__uint_as_float(v[g * 8 + 0]), __uint_as_float(v[g * 8 + 1]));
                            o.y = float2_to_bf16x2(__uint_as_float(v[g * 8 + 2]), __uint_as_float(v[g * 8 + 3]));
                            o.z = float2_to_bf16x2(__uint_as_float(v[g * 8 + 4]), __uint_as_float(v[g * 8 + 5]));
                            o.w = float2_to_bf16x2(__uint_as_float(v[g * 8 + 6]), __uint_as_float(v[g * 8 + 7]));
                            *reinterpret_cast<uint4*>(out_row + col) = o;
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (!ok) {
            report_timeout(status);
            *abort_flag = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, L::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Resident-W variant (K <= 512).  Each CTA is pinned to one 128-column slice of
// C and keeps that slice of W (K x 128 bf16, at most 128 KB) in shared memory for
// its whole life, loaded alongside the first tile's k-blocks; after that only dY
// streams through the ring (16 KB per k-block), so the L2->SM traffic per tile is
// the dY tile alone.  The epilogue stages each 128 x 64 bf16 half of the tile in
// shared memory (128-byte swizzle, conflict-free) and writes it with one TMA
// bulk tensor store; the store clips the M and C tails.
constexpr int kResStages = 4;
constexpr int kResMaxKb = 8;   // K <= 512

struct PwResLayout {
    static constexpr int kW = 0;                                  // [kb][2 atoms][64 k][128 B]
    static constexpr int kA = kW + kResMaxKb * 16384;             // [stage][128 rows][128 B]
    static constexpr int kEpi = kA + kResStages * 16384;          // [2][128 rows][128 B]
    static constexpr int kBars = kEpi + 2 * 16384;
    static constexpr int kNumBars = 2 * kResStages + kResMaxKb + 5;
    static constexpr int kBytes = kBars + kNumBars * 8 + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

__global__ void __launch_bounds__(kThreads, 1)
    pw_tc_res_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                     const __grid_constant__ CUtensorMap map_d, int M, int C, int K, int* status)
{
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    using L = PwResLayout;
    constexpr int BN = 128;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
    uint64_t* full = bars;
    uint64_t* empty = bars + kResStages;
    uint64_t* wfull = bars + 2 * kResStages;
    uint64_t* tfull = wfull + kResMaxKb;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (M + kBM - 1) / kBM;
    const int num_n = (C + BN - 1) / BN;
    const int num_kb = (K + kBK - 1) / kBK;
    const int n_blk = blockIdx.x % num_n;
    const int first_m = blockIdx.x / num_n;
    const int m_step = gridDim.x / num_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kResStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int k = 0; k < kResMaxKb; ++k) mbar_init(&wfull[k], 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b);
        tma_prefetch_desc(&map_d);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_first();   // each dY tile is read by num_n CTAs, then dead
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true, first = true;
            for (int m = first_m; m < num_m && ok; m += m_step) {
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], 16384);
                    tma_load_2d_hint(smem + L::kA + stage * 16384, &map_a, &full[stage], kb * kBK, m * kBM,
                                     num_n > 1 ? policy_evict_last() : pol_a);
                    if (first) {
                        mbar_arrive_expect_tx(&wfull[kb], 16384);
                        tma_load_2d(smem + L::kW + kb * 16384, &map_b, &wfull[kb], n_blk * BN, kb * kBK);
                        tma_load_2d(smem + L::kW + kb * 16384 + 8192, &map_b, &wfull[kb], n_blk * BN + 64,
                                    kb * kBK);
                    }
                    ++issued;
                    if (++stage == kResStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                first = false;
            }
            if (!ok) {
                report_timeout(status);
                *abort_flag = 1;
            }
            for (long long i = (issued > kResStages ? issued - kResStages : 0); i < issued; ++i)
                if (!mbar_wait(&full[i % kResStages], static_cast<uint32_t>((i / kResStages) & 1))) {
                    report_timeout(status);
                    *abort_flag = 1;
                }
            if (!first)
                for (int kb = 0; kb < num_kb; ++kb)
                    if (!mbar_wait(&wfull[kb], 0)) {
                        report_timeout(status);
                        *abort_flag = 1;
                    }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, /*b_mn_major=*/true);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true, first = true;
            for (int m = first_m; m < num_m && ok; m += m_step) {
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag) || (first && !mbar_wait(&wfull[kb], 0, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + L::kA + stage * 16384);
                    const uint32_t b_addr = smem_u32(smem + L::kW + kb * 16384);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_f16(d_tmem, sw128_desc(a_addr + kk * 32, 16, 1024),
                                 sw128_desc(b_addr + kk * 2048, 8192, 1024), idesc, (kb | kk) != 0 ? 1u : 0u);
                    umma_commit(&empty[stage]);
                    if (++stage == kResStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
                first = false;
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) {
                report_timeout(status);
                *abort_flag = 1;
            }
            umma_commit(drain);
            if (!mbar_wait(drain, 0)) {
                report_timeout(status);
                *abort_flag = 1;
            }
        }
    } else {
        // Epilogue: 4 warps; warp w reads TMEM lanes 32*(w%4) .. +31 = tile rows.
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const bool issuer = warp == 2 && lane == 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int m = first_m; m < num_m; m += m_step) {
            if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint8_t* buf = smem + L::kEpi + half * 16384;
                if (issuer) bulk_wait_group_read<1>();     // the last store out of this buffer has read it
                named_barrier_sync(1, 128);
                uint32_t v[64];
                tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(acc * BN + half * 64),
                                   *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(acc * BN + half * 64 + 32),
                                   *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                tmem_wait_ld();
                uint8_t* rowp = buf + row * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 o;
                    o.x = float2_to_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1]));
                    o.y = float2_to_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]));
                    o.z = float2_to_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]));
                    o.w = float2_to_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]));
                    *reinterpret_cast<uint4*>(rowp + ((j ^ (row & 7)) << 4)) = o;
                }
                fence_proxy_async_smem();
                named_barrier_sync(1, 128);
                if (issuer) {
                    tma_store_2d(&map_d, buf, n_blk * BN + half * 64, m * kBM);
                    bulk_commit_group();
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (!ok) {
            report_timeout(status);
            *abort_flag = 1;
        }
        if (issuer) bulk_wait_group<0>();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, 2 * BN);
    }
}

// ---------------------------------------------------------------------------
// SM-pair variant (cta_group::2).  Two CTAs of a cluster compute one 256 x 256
// tile of dX: each holds 128 rows of the dY tile and 128 columns of the W tile
// in its own shared memory, the rank-0 CTA issues tcgen05.mma.cta_group::2
// (M = 256, N = 256, K = 16), and each CTA's tensor memory receives its 128 rows
// x 256 columns of the accumulator.  Per k-block each SM loads 32 KB for a
// 128 x 256 slab of output, half the operand bytes per output of a one-SM tile,
// which is what bounds this memory-streaming GEMM.
//   * both CTAs' TMA loads complete on the rank-0 CTA's "full" barrier, whose
//     expected byte count (both halves) the rank-0 producer posts;
//   * the MMA commit is multicast to the "empty" and "tmem full" barriers of
//     both CTAs; both epilogues arrive on the rank-0 "tmem empty" barrier;
//   * the epilogue stages 128 x 64 bf16 chunks in shared memory (128-byte
//     swizzle) and stores them with TMA, which clips the M and C tails;
//   * cluster barriers order barrier initialisation before any remote arrive
//     and keep both CTAs alive until all cross-CTA traffic has landed.
// BN is the pair tile width (256 or 128); each CTA holds BN/2 columns of W.
// The units of one SM pair.  Every pair takes R = tiles / pairs whole tiles
// (t = pair, pair + pairs, ...).  When the L tiles left over fit twice into the
// pairs (2L <= pairs), they are split into 2L halves of BN/2 columns, one per
// pair, so the last round takes about half a tile instead of a whole one on a
// third of the pairs; otherwise the first L pairs take one more whole tile.
struct PwUnit {
    int m_blk, n0, ncols;
};

struct PwSched {
    int num_n, pairs, R, L;
    bool split;
    __device__ __forceinline__ PwSched(int num_tiles, int num_n_, int pairs_, int BN)
    {
        num_n = num_n_;
        pairs = pairs_;
        R = num_tiles / pairs;
        L = num_tiles - R * pairs;
        split = BN == 256 && L > 0 && 2 * L <= pairs;
    }
    __device__ __forceinline__ int count(int pair) const
    {
        return R + (split ? (pair < 2 * L ? 1 : 0) : (pair < L ? 1 : 0));
    }
    __device__ __forceinline__ PwUnit unit(int pair, int k, int BN) const
    {
        PwUnit u;
        if (k < R || !split) {
            const int t = pair + k * pairs;
            u.m_blk = t / num_n;
            u.n0 = (t - u.m_blk * num_n) * BN;
            u.ncols = BN;
        } else {
            const int t = R * pairs + (pair >> 1);
            u.m_blk = t / num_n;
            u.n0 = (t - u.m_blk * num_n) * BN + (pair & 1) * (BN / 2);
            u.ncols = BN / 2;
        }
        return u;
    }
};

template <int BN, int STAGES>
struct PwPairLayout {
    static constexpr int kBHalf = (BN / 2) * kBK * 2;         // this CTA's W columns, one k-block
    static constexpr int kStage = 16384 + kBHalf;            // A 16 KB + W half
    static constexpr int kA = 0;
    static constexpr int kEpi = STAGES * kStage;             // 2 x 16 KB staging
    static constexpr int kBars = kEpi + 2 * 16384;
    static constexpr int kNumBars = 2 * STAGES + 5;
    static constexpr int kBytes = kBars + kNumBars * 8 + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    pw_tc_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const __grid_constant__ CUtensorMap map_d, int M, int C, int K, int* status)
{
    using L = PwPairLayout<BN, STAGES>;
    constexpr int kPairStages = STAGES;
    {
        // While the previous kernel may still run, only L2 prefetches of this CTA's first
        // stages of dY and W: L2 is the point of coherence, so the loads below still see
        // that kernel's writes, and the DRAM reads overlap its tail.
        const int num_n0 = (C + BN - 1) / BN;
        const int pairs0 = static_cast<int>(gridDim.x >> 1);
        const PwSched sched0(((M + 255) / 256) * num_n0, num_n0, pairs0, BN);
        const int pair0 = static_cast<int>(blockIdx.x >> 1);
        if (threadIdx.x == 0 && sched0.count(pair0) > 0) {
            const uint32_t r0 = cluster_ctarank();
            const PwUnit un = sched0.unit(pair0, 0, BN);
            tma_prefetch_desc(&map_a);
            tma_prefetch_desc(&map_b);
            const int nkb = (K + kBK - 1) / kBK < kPairStages ? (K + kBK - 1) / kBK : kPairStages;
            for (int kb = 0; kb < nkb; ++kb) {
                tma_prefetch_l2_2d(&map_a, kb * kBK, un.m_blk * 256 + static_cast<int>(r0) * 128);
                for (int j = 0; j < un.ncols / 128; ++j)
                    tma_prefetch_l2_2d(&map_b, un.n0 + static_cast<int>(r0) * (un.ncols / 2) + j * 64, kb * kBK);
            }
        }
    }
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
    uint64_t* full = bars;                      // used in the rank-0 CTA
    uint64_t* empty = bars + kPairStages;       // each CTA's own
    uint64_t* tfull = bars + 2 * kPairStages;   // each CTA's own
    uint64_t* tempty = tfull + 2;               // used in the rank-0 CTA (256 arrivals)
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const uint32_t rank = cluster_ctarank();
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (M + 255) / 256;
    const int num_n = (C + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int num_kb = (K + kBK - 1) / kBK;
    const int pair = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;
    const PwSched sched(num_tiles, num_n, num_pairs, BN);
    const int nunits = sched.count(pair);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 256);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b);
        tma_prefetch_desc(&map_d);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 2 * BN);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();                              // barriers of both CTAs exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            const uint32_t full0 = leader_addr(&full[0]);
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int k = 0; k < nunits && ok; ++k) {
                const PwUnit un = sched.unit(pair, k, BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // both CTAs' A halves (16 KB each) and W columns (ncols/2 each, 128 bytes per k row)
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (16384 + un.ncols * kBK));
                    uint8_t* a_tile = smem + L::kA + stage * L::kStage;
                    uint8_t* b_tile = a_tile + 16384;
                    const uint32_t fb = full0 + static_cast<uint32_t>(stage * 8);
                    tma_load_2d_pair(a_tile, &map_a, fb, kb * kBK, un.m_blk * 256 + static_cast<int>(rank) * 128);
                    const int ncol = un.n0 + static_cast<int>(rank) * (un.ncols / 2);
                    for (int j = 0; j < un.ncols / 128; ++j)
                        tma_load_2d_pair(b_tile + j * 8192, &map_b, fb, ncol + j * 64, kb * kBK);
                    ++issued;
                    if (++stage == kPairStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                report_timeout(status);
                *abort_flag = 1;
            }
            // the last loads of this CTA land before it may exit: wait until the MMAs
            // that read them have released the stages (multicast commit)
            for (long long i = (issued > kPairStages ? issued - kPairStages : 0); i < issued; ++i)
                if (!mbar_wait(&empty[i % kPairStages], static_cast<uint32_t>((i / kPairStages) & 1))) {
                    report_timeout(status);
                    *abort_flag = 1;
                }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc_full = idesc_bf16_f32(256, BN, /*b_mn_major=*/true);
            constexpr uint32_t idesc_half = idesc_bf16_f32(256, BN / 2, /*b_mn_major=*/true);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int k = 0; k < nunits && ok; ++k) {
                const uint32_t idesc = sched.unit(pair, k, BN).ncols == BN ? idesc_full : idesc_half;
                if (!mbar_wait_cluster(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + L::kA + stage * L::kStage);
                    const uint32_t b_addr = a_addr + 16384;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_f16_pair(d_tmem, sw128_desc(a_addr + kk * 32, 16, 1024),
                                      sw128_desc(b_addr + kk * 2048, 8192, 1024), idesc, (kb | kk) != 0 ? 1u : 0u);
                    umma_commit_pair(&empty[stage]);
                    if (++stage == kPairStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) {
                report_timeout(status);
                *abort_flag = 1;
            }
            umma_commit_pair(drain);             // same CTA-group as the MMAs it tracks
            if (!mbar_wait(drain, 0)) {
                report_timeout(status);
                *abort_flag = 1;
            }
        }
    } else {
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const bool issuer = warp == 2 && lane == 0;
        const uint32_t tempty0 = leader_addr(&tempty[0]);
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int k = 0; k < nunits; ++k) {
            const PwUnit un = sched.unit(pair, k, BN);
            if (!mbar_wait_cluster(&tfull[acc], acc_phase, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int chunk = 0; chunk < un.ncols / 64; ++chunk) {
                uint8_t* buf = smem + L::kEpi + (chunk & 1) * 16384;
                if (issuer) bulk_wait_group_read<1>();
                named_barrier_sync(1, 128);
                uint32_t v[64];
                tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(acc * BN + chunk * 64),
                                   *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(acc * BN + chunk * 64 + 32),
                                   *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                tmem_wait_ld();
                uint8_t* rowp = buf + row * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 o;
                    o.x = float2_to_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1]));
                    o.y = float2_to_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]));
                    o.z = float2_to_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]));
                    o.w = float2_to_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]));
                    *reinterpret_cast<uint4*>(rowp + ((j ^ (row & 7)) << 4)) = o;
                }
                fence_proxy_async_smem();
                named_barrier_sync(1, 128);
                if (issuer) {
                    tma_store_2d(&map_d, buf, un.n0 + chunk * 64, un.m_blk * 256 + static_cast<int>(rank) * 128);
                    bulk_commit_group();
                }
            }
            tc_fence_before();
            mbar_arrive_cluster(tempty0 + static_cast<uint32_t>(acc * 8));   // rank-0 CTA's tmem-empty barrier
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (!ok) {
            report_timeout(status);
            *abort_flag = 1;
        }
        if (issuer) bulk_wait_group<0>();
    }

    tc_fence_before();
    cluster_sync();                              // no CTA leaves while its pair still needs it
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem_base, 2 * BN);
    }
}

// ---------------------------------------------------------------------------
// Split-K variant for small M (few tiles): the K-loop of every (m, n) tile is
// split into S contiguous ranges of k-blocks.  Work unit (m-block, n-block,
// split) computes a partial tile and writes it as fp32 to the workspace
// ws[split][m][c]; a second kernel sums the S partials in split order
// (deterministic: no atomics, nothing to zero) and rounds to bf16 (or f16 when
// F16: f16 operands, the same fp32 partials).  Structure as the streaming
// kernel: TMA producer, MMA issuer, 4 epilogue warps, two TMEM accumulators.
template <int BN, int STAGES, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    pw_tc_splitk_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                        float* __restrict__ ws, int M, int C, int K, int S, int* status)
{
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    using L = PwTcLayout<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kTileBytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (M + kBM - 1) / kBM;
    const int num_n = (C + BN - 1) / BN;
    const int num_units = num_m * num_n * S;
    const int num_kb = (K + kBK - 1) / kBK;
    const int kb_per = (num_kb + S - 1) / S;
    auto unit_range = [&](int u, int& m_blk, int& n_blk, int& kb0, int& kb1) {
        const int ks = u % S;
        const int t = u / S;
        m_blk = t / num_n;
        n_blk = t - m_blk * num_n;
        kb0 = ks * kb_per;
        kb1 = min(num_kb, kb0 + kb_per);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
                int m_blk, n_blk, kb0, kb1;
                unit_range(u, m_blk, n_blk, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
                    uint8_t* a_tile = smem + stage * L::kStageBytes;
                    uint8_t* b_tile = a_tile + L::kABytes;
                    tma_load_2d(a_tile, &map_a, &full[stage], kb * kBK, m_blk * kBM);
#pragma unroll
                    for (int j = 0; j < BN / 64; ++j)
                        tma_load_2d(b_tile + j * 8192, &map_b, &full[stage], n_blk * BN + j * 64, kb * kBK);
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                report_timeout(status);
                *abort_flag = 1;
            }
            for (long long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
                if (!mbar_wait(&full[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1))) {
                    report_timeout(status);
                    *abort_flag = 1;
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = F16 ? idesc_f16_f32(kBM, BN, /*b_mn_major=*/true)
                                           : idesc_bf16_f32(kBM, BN, /*b_mn_major=*/true);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
                int m_blk, n_blk, kb0, kb1;
                unit_range(u, m_blk, n_blk, kb0, kb1);
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + stage * L::kStageBytes);
                    const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_f16(d_tmem, sw128_desc(a_addr + kk * 32, 16, 1024),
                                 sw128_desc(b_addr + kk * 2048, 8192, 1024), idesc,
                                 (kb > kb0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) {
                report_timeout(status);
                *abort_flag = 1;
            }
            umma_commit(drain);
            if (!mbar_wait(drain, 0)) {
                report_timeout(status);
                *abort_flag = 1;
            }
        }
    } else {
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
            int m_blk, n_blk, kb0, kb1;
            unit_range(u, m_blk, n_blk, kb0, kb1);
            const int ks = u % S;
            if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int m = m_blk * kBM + row;
            float* out_row = ws + (static_cast<long long>(ks) * M + m) * C;
#pragma unroll 1
            for (int chunk = 0; chunk < BN / 32; ++chunk) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(acc * BN + chunk * 32), v);
                tmem_wait_ld();
                const int col0 = n_blk * BN + chunk * 32;
                if (m < M) {
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const int col = col0 + g * 4;
                        if (col < C)
                            *reinterpret_cast<uint4*>(out_row + col) =
                                make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (!ok) {
            report_timeout(status);
            *abort_flag = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, L::kTmemCols);
    }
}

// dX[m][c] = round(sum over s of ws[s][m][c]), s in increasing order, rounded once
// to bf16 (or f16 when F16); 8 channels per thread.
template <bool F16>
__global__ void __launch_bounds__(256)
    splitk_reduce_kernel(const float* __restrict__ ws, uint16_t* __restrict__ dX, long long MC, int S, int* status)
{
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    const long long i = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
    if (i >= MC) return;
    float4 a = *reinterpret_cast<const float4*>(ws + i);
    float4 b = *reinterpret_cast<const float4*>(ws + i + 4);
    for (int s = 1; s < S; ++s) {
        const float4 x = *reinterpret_cast<const float4*>(ws + s * MC + i);
        const float4 y = *reinterpret_cast<const float4*>(ws + s * MC + i + 4);
        a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
        b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
    }
    constexpr int EK = F16 ? kF16 : kBF16;
    uint4 o;
    o.x = float2_to_h16x2<EK>(a.x, a.y);
    o.y = float2_to_h16x2<EK>(a.z, a.w);
    o.z = float2_to_h16x2<EK>(b.x, b.y);
    o.w = float2_to_h16x2<EK>(b.z, b.w);
    if (store_ok(dX, MC * 2, dX + i, 16, status)) *reinterpret_cast<uint4*>(dX + i) = o;
}

template <int BN, int STAGES>
cudaError_t launch_bn(const PwArgs& a, const CUtensorMap& map_a, const CUtensorMap& map_b, int num_sms,
                      cudaStream_t stream)
{
    using L = PwTcLayout<BN, STAGES>;
    static_assert(L::kAlloc <= 232448, "shared memory budget");
    auto kern = pw_tc_kernel<BN, STAGES>;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), L::kAlloc);
    if (e != cudaSuccess) return e;
    const int num_tiles = static_cast<int>(((a.M + kBM - 1) / kBM) * ((a.C + BN - 1) / BN));
    const int grid = num_tiles < num_sms ? num_tiles : num_sms;
    {
        const cudaError_t le_ = launch_kernel(kern, dim3(grid), dim3(kThreads), L::kAlloc, stream, 1,
                                             map_a, map_b, static_cast<__nv_bfloat16*>(a.dX),
                                                 static_cast<int>(a.M), static_cast<int>(a.C),
                                                 static_cast<int>(a.K), a.status);
        if (le_ != cudaSuccess) return le_;
    }
    return cudaGetLastError();
}

cudaError_t launch_res(const PwArgs& a, const CUtensorMap& map_a, const CUtensorMap& map_b,
                       const CUtensorMap& map_d, int num_sms, cudaStream_t stream)
{
    using L = PwResLayout;
    static_assert(L::kAlloc <= 232448, "shared memory budget");
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(pw_tc_res_kernel), L::kAlloc);
    if (e != cudaSuccess) return e;
    const int num_m = static_cast<int>((a.M + kBM - 1) / kBM);
    const int num_n = static_cast<int>((a.C + 127) / 128);
    int per_n = num_sms / num_n;
    if (per_n > num_m) per_n = num_m;
    const int grid = per_n * num_n;
    {
        const cudaError_t le_ = launch_kernel(pw_tc_res_kernel, dim3(grid), dim3(kThreads), L::kAlloc, stream, 1,
                                             map_a, map_b, map_d, static_cast<int>(a.M),
                                                            static_cast<int>(a.C), static_cast<int>(a.K),
                                                            a.status);
        if (le_ != cudaSuccess) return le_;
    }
    return cudaGetLastError();
}

template <int BN, int STAGES>
cudaError_t launch_pair(const PwArgs& a, const CUtensorMap& map_a, const CUtensorMap& map_b,
                        const CUtensorMap& map_d, int num_sms, cudaStream_t stream)
{
    using L = PwPairLayout<BN, STAGES>;
    static_assert(L::kAlloc <= 232448, "shared memory budget");
    auto kern = pw_tc_pair_kernel<BN, STAGES>;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), L::kAlloc);
    if (e != cudaSuccess) return e;
    const int num_tiles = static_cast<int>(((a.M + 255) / 256) * ((a.C + BN - 1) / BN));
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L::kAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent: as many pairs as can be resident at once (at most one per tile)
    static int max_clusters = 0;
    if (max_clusters == 0) {
        cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) n = num_sms / 2;
        max_clusters = n;
    }
    int pairs = max_clusters < num_tiles ? max_clusters : num_tiles;
    return launch_kernel(kern, dim3(static_cast<unsigned>(2 * pairs)), dim3(kThreads), L::kAlloc, stream, 2, map_a,
                         map_b, map_d, static_cast<int>(a.M), static_cast<int>(a.C), static_cast<int>(a.K), a.status);
}

}  // namespace

int pointwise_splitk_auto(const PwArgs& a, int num_sms)
{
    const int tiles = static_cast<int>(((a.M + kBM - 1) / kBM) * ((a.C + 127) / 128));
    const int num_kb = static_cast<int>((a.K + kBK - 1) / kBK);
    if (tiles <= 0) return 1;   // empty batch: nothing to split
    int s = (num_sms + tiles - 1) / tiles;
    if (s > num_kb) s = num_kb;
    if (s > 32) s = 32;
    return s < 1 ? 1 : s;
}

size_t pointwise_splitk_workspace_bytes(const PwArgs& a, int splits)
{
    return static_cast<size_t>(splits) * static_cast<size_t>(a.M) * static_cast<size_t>(a.C) * sizeof(float);
}

cudaError_t launch_pointwise_tc_splitk(const PwArgs& a, const CUtensorMap& map_a, const CUtensorMap& map_b,
                                       int splits, float* ws, int num_sms, cudaStream_t stream)
{
    if (a.M <= 0) return cudaSuccess;
    using L = PwTcLayout<128, 6>;
    auto kern = a.f16 ? pw_tc_splitk_kernel<128, 6, true> : pw_tc_splitk_kernel<128, 6, false>;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), L::kAlloc);
    if (e != cudaSuccess) return e;
    const int num_kb = static_cast<int>((a.K + kBK - 1) / kBK);
    const int kb_per = (num_kb + splits - 1) / splits;
    const int S = (num_kb + kb_per - 1) / kb_per;   // no empty split
    const long long units = ((a.M + kBM - 1) / kBM) * ((a.C + 127) / 128) * S;
    const int grid = static_cast<int>(units < num_sms ? units : num_sms);
    {
        const cudaError_t le_ = launch_kernel(kern, dim3(grid), dim3(kThreads), L::kAlloc, stream, 1,
                                             map_a, map_b, ws, static_cast<int>(a.M), static_cast<int>(a.C),
                                                static_cast<int>(a.K), S, a.status);
        if (le_ != cudaSuccess) return le_;
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long MC = a.M * a.C;
    const long long threads = (MC + 7) / 8;
    auto reduce = a.f16 ? splitk_reduce_kernel<true> : splitk_reduce_kernel<false>;
    {
        const cudaError_t le_ = launch_kernel(reduce, dim3(static_cast<unsigned>((threads + 255) / 256)), dim3(256), 0, stream, 1,
                                             ws, static_cast<uint16_t*>(a.dX), MC,
                                                                             S, a.status);
        if (le_ != cudaSuccess) return le_;
    }
    return cudaGetLastError();
}

cudaError_t launch_pointwise_tc_pair(const PwArgs& a, const CUtensorMap& map_a, const CUtensorMap& map_b,
                                     const CUtensorMap& map_d, int bn, int num_sms, cudaStream_t stream)
{
    if (a.M <= 0) return cudaSuccess;
    if (bn == 256) return launch_pair<256, 6>(a, map_a, map_b, map_d, num_sms, stream);
    return launch_pair<128, 8>(a, map_a, map_b, map_d, num_sms, stream);
}

bool pointwise_tc_resident_ok(const PwArgs& a, int num_sms)
{
    return a.K <= 64 * kResMaxKb && (a.C + 127) / 128 <= num_sms / 2;
}

cudaError_t launch_pointwise_tc_resident(const PwArgs& a, const CUtensorMap& map_a, const CUtensorMap& map_b,
                                         const CUtensorMap& map_d, int num_sms, cudaStream_t stream)
{
    if (a.M <= 0) return cudaSuccess;
    if (!pointwise_tc_resident_ok(a, num_sms)) return cudaErrorInvalidValue;
    return launch_res(a, map_a, map_b, map_d, num_sms, stream);
}

cudaError_t launch_pointwise_tc(const PwArgs& a, const CUtensorMap& map_a, const CUtensorMap& map_b, int bn,
                                int num_sms, cudaStream_t stream)
{
    if (a.M <= 0) return cudaSuccess;
    switch (bn) {
    case 64: return launch_bn<64, 8>(a, map_a, map_b, num_sms, stream);
    case 256: return launch_bn<256, 4>(a, map_a, map_b, num_sms, stream);
    default: return launch_bn<128, 6>(a, map_a, map_b, num_sms, stream);
    }
}

}  // namespace dgrad
