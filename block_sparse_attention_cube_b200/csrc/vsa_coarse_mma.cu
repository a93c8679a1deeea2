// The coarse stage's two contractions on the tensor cores (Wan2.2 teardown,
// zharfai.com, section "Video sparse attention selects cubes", part 1: block-
// level attention over the mean-pooled cubes; section "Blackwell changes the
// optimisation problem": dense contractions belong on the fifth-generation
// tensor cores).
//
// The pooled vectors are float32, and the scores decide the selection, so a
// plain bf16 product (8-bit significands) would reorder near-equal cubes.
// Each float32 value x is therefore carried as three bf16 parts
//     hi = bf16(x), mid = bf16(x - hi), lo = bf16(x - hi - mid)
// (x = hi + mid + lo to within 2^-24 |x|, each part rounded to nearest), and
// a product a*b is formed from the six partial products whose size is at
// least 2^-18 |a b|:
//     hi*hi + hi*mid + mid*hi + hi*lo + lo*hi + mid*mid,
// each exact in the float32 accumulator's input (8 x 8 significand bits).
// The dropped terms are below 2^-26 |a b|, so a score carries about the error
// of a float32 dot product.  Six tcgen05 MMAs per 16-channel step replace one;
// on B200 that is still several times the float32 CUDA-core rate.
//
// Scores: one CTA per (b, h, 128 query cubes) loops over the head's key cubes
// in tiles of 128: a TMA producer warp (one lane per bf16 part), an MMA issuer
// warp, and eight epilogue warps that move each 128 x 128 float32 tile from
// tensor memory to the [B, H, C, C] scores (scaled), two tiles in flight (warp
// w: TMEM lane quarter w % 4, key columns 64 (w / 4) .. + 63 of the tile; one
// warp per scheduler was latency-bound at about 1,900 cycles per 32 columns).
// The epilogue stages each warp's 32 x 32 block in shared memory and writes it
// with a TMA store (whole 128-byte lines, rows and columns past C clipped by
// the copy) when C is a multiple of 4; a thread's row written straight from
// registers touches 32 rows per store instruction.  A CTA sees whole score
// rows, so the epilogue also keeps each row's running maximum and sum of
// exponentials (the softmax statistics the coarse output needs), rescaled as
// the maximum grows; the two warps of a row combine theirs at the end.
#include <mutex>

#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "ptx_sm100.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

using namespace ptx;

constexpr int kCmThreads = 320;                 // warps 0-7 epilogue (two per TMEM lane quarter), 8 TMA, 9 MMA
constexpr int kCmEpiWarps = 8;
constexpr int kCmTmaWarp = 8;
constexpr int kCmMmaWarp = 9;
constexpr uint32_t kCmHalf = 128u * 128u;       // 128 rows x 64 bf16 channels, 128-byte swizzled: 16 KB
constexpr uint32_t kCmOffA = 0;                 // query cubes: [part][channel half], up to 6 x 16 KB
constexpr uint32_t kCmOffB = 6u * kCmHalf;      // key cubes: 2 stages x [part] (one channel half), 3 x 16 KB
constexpr uint32_t kCmStage = 3u * kCmHalf;
constexpr int kCmStages = 2;
constexpr uint32_t kCmEBlock = 32u * 128u;      // an epilogue warp's 32 rows x 32 float32 scores, 128-byte swizzled
constexpr uint32_t kCmOffE = kCmOffB + kCmStages * kCmStage;   // [8 warps]
constexpr uint32_t kCmOffStat = kCmOffE + kCmEpiWarps * kCmEBlock;   // [128 rows] float2: the upper half's (m, l)
constexpr uint32_t kCmOffBar = kCmOffStat + 128u * 8u;
enum CmBar : int { kCmBarA = 0, kCmBarBFull = 1, kCmBarBEmpty = 3, kCmBarSFull = 5, kCmBarSEmpty = 7, kCmBarDrain = 9,
                   kCmBarStat = 10, kCmBars = 11 };
constexpr uint32_t kCmOffMisc = kCmOffBar + 8u * kCmBars;          // TMEM address, abort flag
constexpr uint32_t kCmSmem = kCmOffMisc + 16u + 1024u;             // + slack for the 1 KB alignment
static_assert(kCmSmem <= 232448, "shared memory over the 227 KB per-block limit");
constexpr uint32_t kCmTmemCols = 256;                              // two 128-column score buffers
constexpr uint64_t kCmDrainNs = 200000000ull;

// the six partial products (part of the query cube, part of the key cube), largest first:
// (hi, hi), (hi, mid), (mid, hi), (hi, lo), (lo, hi), (mid, mid)
__host__ __device__ constexpr int prod_a(int pr) { return pr == 2 || pr == 5 ? 1 : pr == 4 ? 2 : 0; }
__host__ __device__ constexpr int prod_b(int pr) { return pr == 1 || pr == 5 ? 1 : pr == 3 ? 2 : 0; }

struct CmParams {
    int C, B, H;
    int row_tiles;           // ceil(C / 128)
    float scale;
    float* scores;           // [B, H, C, C]
    float2* stats;           // [B, H, C]: (row maximum, 1 / sum of exp(s - maximum)), or nullptr
    int tma_store;           // 1: scores leave through tm_s (C % 4 == 0), 0: straight from registers
    int* status;             // watchdog word
    uint64_t limit_ns;
};

// x = hi + mid + lo, each part the bf16 nearest to what the larger parts leave (as the pooling pass
// splits the pooled vectors), for two values at once, packed as the bf16 pairs the operands hold (first
// value in the low half): each rounding is one paired conversion, and a part's float value is its bits
// shifted into place.
__device__ __forceinline__ void split3x2(float a, float b, uint32_t& hi, uint32_t& mid, uint32_t& lo) {
    hi = pack_bf16x2(a, b);
    const float ra = a - __uint_as_float(hi << 16), rb = b - __uint_as_float(hi & 0xFFFF0000u);
    mid = pack_bf16x2(ra, rb);
    const float qa = ra - __uint_as_float(mid << 16), qb = rb - __uint_as_float(mid & 0xFFFF0000u);
    lo = pack_bf16x2(qa, qb);
}

__device__ __forceinline__ uint64_t desc_at(uint64_t fixed, uint32_t saddr) {
    return fixed | static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
}

template <int D>
__global__ void __launch_bounds__(kCmThreads, 1)
coarse_scores_mma_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_s, const CmParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base = (raw_u32 + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_u32);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto bar = [&](int i) -> uint32_t { return base + kCmOffBar + 8u * static_cast<uint32_t>(i); };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kCmOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kCmOffMisc + 4);
    const BoundedWait bw{abort_flag, p.status, p.limit_ns};

    const int bh = blockIdx.x / p.row_tiles;
    const int i0 = (blockIdx.x % p.row_tiles) * 128;
    const int C = p.C;
    const int tiles = (C + 127) / 128;
    constexpr int kHalves = D / 64;   // 64-channel halves: one swizzled 128-byte row each

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bar(kCmBarA), 1);
        for (int s = 0; s < kCmStages; ++s) {
            mbar_init(bar(kCmBarBFull + s), 1);
            mbar_init(bar(kCmBarBEmpty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(kCmBarSFull + b), 1);
            mbar_init(bar(kCmBarSEmpty + b), kCmEpiWarps);   // one arrival per epilogue warp
        }
        mbar_init(bar(kCmBarDrain), 1);
        mbar_init(bar(kCmBarStat), 4);   // the four upper-half warps
        fence_mbar_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        if (p.tma_store) prefetch_tensormap(&tm_s);
    }
    if (warp == kCmMmaWarp) {
        tmem_alloc(base + kCmOffMisc, kCmTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto drain_wait = [&](uint32_t b, uint32_t par) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(b, par) && globaltimer() - t0 < kCmDrainNs) {
        }
    };

    if (warp == kCmTmaWarp) {
        // ------------------------------------------------------------ TMA producer (lane i: part i)
        // One thread issuing every copy is held about as long as the copies take, so
        // the three parts of a load go out from three lanes at once.
        constexpr unsigned kPartMask = 0x7u;
        if (lane < 3) {
            bool ok = true;
            uint32_t issued[kCmStages] = {0u, 0u};
            // the CTA's 128 query cubes: three parts x two channel halves (rows past C read as zeros)
            if (lane == 0) mbar_arrive_expect_tx(bar(kCmBarA), 3u * kHalves * kCmHalf);
            __syncwarp(kPartMask);   // lane 0's expect_tx first
            for (int h = 0; h < kHalves; ++h)
                tma_load_4d(base + kCmOffA + (kHalves * lane + h) * kCmHalf, &tm_q, 64 * h, i0, bh, lane,
                            bar(kCmBarA));
            int slot = 0;
            uint32_t phase = 0;
            for (int n = 0; ok && n < tiles; ++n) {
                for (int h = 0; h < kHalves; ++h) {
                    if (!(ok = __all_sync(kPartMask, bw.wait(bar(kCmBarBEmpty + slot), phase ^ 1u)))) break;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(bar(kCmBarBFull + slot), kCmStage);
                        ++issued[slot];
                    }
                    __syncwarp(kPartMask);
                    tma_load_4d(base + kCmOffB + slot * kCmStage + lane * kCmHalf, &tm_k, 64 * h, 128 * n, bh, lane,
                                bar(kCmBarBFull + slot));
                    if (++slot == kCmStages) {
                        slot = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && lane == 0) {
                // copies still in flight land before the CTA exits
                drain_wait(bar(kCmBarA), 0u);
                for (int s = 0; s < kCmStages; ++s)
                    if (issued[s]) drain_wait(bar(kCmBarBFull + s), (issued[s] - 1u) & 1u);
            }
        }
    } else if (warp == kCmMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);   // both operands K-major
            const uint64_t fix = smem_desc_sw128(0, 16u, 1024u);         // 8-row groups 1 KB apart
            bool ok = bw.wait(bar(kCmBarA), 0u);
            bool issued_any = false;
            int slot = 0;
            uint32_t phase = 0;
            for (int n = 0; ok && n < tiles; ++n) {
                const int b = n & 1;
                // the epilogue has read this buffer's previous tile
                if (n >= 2 && !(ok = bw.wait(bar(kCmBarSEmpty + b), ((n >> 1) - 1) & 1))) break;
                for (int h = 0; h < kHalves; ++h) {
                    if (!(ok = bw.wait(bar(kCmBarBFull + slot), phase))) break;
                    tc_fence_after();
                    const uint32_t kb = base + kCmOffB + slot * kCmStage;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                        for (int pr = 0; pr < 6; ++pr) {
                            const uint32_t qa = base + kCmOffA + (kHalves * prod_a(pr) + h) * kCmHalf + kk * 32u;
                            const uint32_t ka = kb + prod_b(pr) * kCmHalf + kk * 32u;
                            mma_bf16_ss(tmem + 128u * b, desc_at(fix, qa), desc_at(fix, ka), idesc,
                                        (h | kk | pr) != 0 ? 1u : 0u);
                        }
                    }
                    mma_commit(bar(kCmBarBEmpty + slot));
                    issued_any = true;
                    if (++slot == kCmStages) {
                        slot = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(bar(kCmBarSFull + b));
            }
            if (issued_any) {
                mma_commit(bar(kCmBarDrain));
                drain_wait(bar(kCmBarDrain), 0u);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue: TMEM -> scores
        constexpr float kLog2e = 1.4426950408889634f;
        const int q = warp & 3, hc = warp >> 2;   // TMEM lane quarter, 64-column half of each tile
        const int r = 32 * q + lane;              // TMEM lane = query row of the tile
        const int gi = i0 + r;
        float* srow = p.scores + (static_cast<int64_t>(bh) * C + (gi < C ? gi : 0)) * C;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
        const uint32_t sb = base + kCmOffE + kCmEBlock * warp;
        float m_run = -INFINITY, l_run = 0.f;   // the row's running maximum and sum of exp(s - m_run)
        bool staged = false;                    // a TMA store of this warp may still read sb
        bool ok = true;
        for (int n = 0; n < tiles; ++n) {
            const int b = n & 1;
            if (!(ok = __all_sync(0xffffffffu, bw.wait(bar(kCmBarSFull + b), (n >> 1) & 1)))) break;
            tc_fence_after();
#pragma unroll 1
            for (int c2 = 0; c2 < 2; ++c2) {
                const int cc = 2 * hc + c2;
                uint32_t v[32];
                tmem_ld32_wait(lane_base + 128u * b + 32u * cc, v);
                const int j0 = 128 * n + 32 * cc;
                float x[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = p.scale * __uint_as_float(v[e]);
                if (j0 + 32 > C) {
                    // keys past C: not stored, and nothing in the statistics
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (j0 + e >= C) x[e] = -INFINITY;
                }
                if (p.stats != nullptr && j0 < C) {
                    float t[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) t[e] = fmaxf(x[e], x[e + 16]);
#pragma unroll
                    for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                        for (int e = 0; e < w; ++e) t[e] = fmaxf(t[e], t[e + w]);
                    const float m_new = fmaxf(m_run, t[0]);
                    const float mb = m_new * kLog2e;
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int e = 0; e < 32; ++e) acc[e & 3] += ex2_approx(fmaf(x[e], kLog2e, -mb));
                    l_run = l_run * ex2_approx((m_run - m_new) * kLog2e) + ((acc[0] + acc[1]) + (acc[2] + acc[3]));
                    m_run = m_new;
                }
                if (p.tma_store) {
                    // the block (rows 32 q.., keys j0..j0+31) through this warp's buffer, once the
                    // previous store has read it; a block wholly past the last row or key is not stored
                    if (j0 >= C || i0 + 32 * q >= C) continue;
                    if (lane == 0 && staged) bulk_wait_group_read<0>();
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t a = sb + lane * 128u + ((static_cast<uint32_t>(c) ^ (lane & 7u)) << 4);
                        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(x[4 * c]),
                                     "f"(x[4 * c + 1]), "f"(x[4 * c + 2]), "f"(x[4 * c + 3])
                                     : "memory");
                    }
                    fence_proxy_async_smem();   // the block becomes visible to the copy engine
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(&tm_s, sb, j0, i0 + 32 * q, bh);
                        bulk_commit_group();
                    }
                    staged = true;
                } else if (gi < C) {
                    if (j0 + 32 <= C && (C & 3) == 0) {
                        float4* dst = reinterpret_cast<float4*>(srow + j0);
#pragma unroll
                        for (int e = 0; e < 8; ++e) dst[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (j0 + e < C) srow[j0 + e] = x[e];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kCmBarSEmpty + b));
        }
        // the stores have left shared memory and reached global memory before the CTA exits
        if (lane == 0 && staged) bulk_wait_group<0>();
        if (p.stats != nullptr) {
            // each row's two halves: (m_a, l_a) and (m_b, l_b) -> m = max, l = l_a 2^(m_a - m) + l_b 2^(m_b - m)
            float2* upper = reinterpret_cast<float2*>(smem + kCmOffStat);
            if (hc == 1) {
                upper[r] = make_float2(m_run, l_run);
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kCmBarStat));   // release: the 32 rows are visible
            } else if (ok && __all_sync(0xffffffffu, bw.wait(bar(kCmBarStat), 0u))) {
                const float2 o = upper[r];
                const float m = fmaxf(m_run, o.x);
                const float l = l_run * ex2_approx((m_run - m) * kLog2e) + o.y * ex2_approx((o.x - m) * kLog2e);
                if (gi < C) p.stats[static_cast<int64_t>(bh) * C + gi] = make_float2(m, 1.0f / l);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kCmMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kCmTmemCols);
    }
}

// ---------------------------------------------------------------- coarse output
// o_coarse = softmax(scores) vbar, as exp(s - m) vbar / l with each row's maximum m and sum l from
// the scores kernel's statistics.  One CTA per (b, h, 128 query cubes): eight converter warps (two
// threads per query row, 32 keys each) turn each 64-key slice of the rows into exp(s - m), split it
// into three bf16 parts and store them K-major with the 128-byte swizzle (the A operand); a TMA warp
// brings the same keys' vbar parts (the B operand, MN-major, one box per lane); an MMA warp issues
// the six partial products per 16-key step into one 128 x D float32 accumulator, which warps 0-3
// scale by 1/l and store.  When C is a multiple of 4, a second TMA warp brings each slice of the 128
// score rows into shared memory (two 32-key boxes, 128-byte swizzled, so that a thread's reads of
// its own row hit every bank once); a thread loading its row straight from global memory touches
// 32 rows per load instruction.  Otherwise each thread loads its row's keys itself, the next
// slice's while it converts the current one.
constexpr uint32_t kPvA = 3u * 128u * 128u;     // P parts of one 64-key slice: 3 x (128 rows x 128 B)
constexpr uint32_t kPvB = 3u * 64u * 256u;      // vbar parts of 64 keys x D = 128: 3 x (2 halves x 8 KB)
constexpr int kPvStages = 2;
constexpr uint32_t kPvOffA = 0;
constexpr uint32_t kPvOffB = kPvOffA + kPvStages * kPvA;
constexpr uint32_t kPvBoxS = 128u * 128u;      // 32 keys x 128 score rows, float32: 16 KB
constexpr uint32_t kPvOffS = kPvOffB + kPvStages * kPvB;   // one slice of scores: [2 key halves]
constexpr uint32_t kPvOffBar = kPvOffS + 2u * kPvBoxS;
enum PvBar : int { kPvBarAFull = 0, kPvBarAEmpty = 2, kPvBarBFull = 4, kPvBarBEmpty = 6, kPvBarSFull = 8,
                   kPvBarSEmpty = 9, kPvBarODone = 10, kPvBarDrain = 11, kPvBars = 12 };
constexpr uint32_t kPvOffMisc = kPvOffBar + 8u * kPvBars;
constexpr uint32_t kPvSmem = kPvOffMisc + 16u + 1024u;
static_assert(kPvSmem <= 232448, "shared memory over the 227 KB per-block limit");
constexpr int kPvConvWarps = 8;                 // warps 0-7 convert (two threads per query row); 0-3 also
constexpr int kPvTmaWarp = 8;                   // run the epilogue (one TMEM lane quarter each)
constexpr int kPvMmaWarp = 9;
constexpr int kPvSWarp = 10;                    // score slices (TMA), when tma_load
constexpr int kPvThreads = 352;

struct PvParams {
    int C, row_tiles;
    const float* scores;      // [B, H, C, C]
    const float2* stats;      // [B, H, C]: (row maximum, 1 / sum of exp(s - maximum))
    float* o_coarse;          // [B, H, C, D]
    int tma_load;             // 1: score slices arrive through tm_s (C % 4 == 0), 0: each thread loads its row
    int* status;
    uint64_t limit_ns;
};

template <int D>
__global__ void __launch_bounds__(kPvThreads, 1)
coarse_pv_mma_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_s,
                     const PvParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base = (raw_u32 + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_u32);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto bar = [&](int i) -> uint32_t { return base + kPvOffBar + 8u * static_cast<uint32_t>(i); };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kPvOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kPvOffMisc + 4);
    const BoundedWait bw{abort_flag, p.status, p.limit_ns};
    constexpr int kHalves = D / 64;
    constexpr uint32_t kPartB = 64u * 128u * kHalves;   // one part of a 64-key vbar slice

    const int bh = blockIdx.x / p.row_tiles;
    const int i0 = (blockIdx.x % p.row_tiles) * 128;
    const int C = p.C;
    const int slices = (C + 63) / 64;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < kPvStages; ++s) {
            mbar_init(bar(kPvBarAFull + s), kPvConvWarps);   // one arrival per converter warp
            mbar_init(bar(kPvBarAEmpty + s), 1);
            mbar_init(bar(kPvBarBFull + s), 1);
            mbar_init(bar(kPvBarBEmpty + s), 1);
        }
        mbar_init(bar(kPvBarSFull), 1);
        mbar_init(bar(kPvBarSEmpty), kPvConvWarps);   // one arrival per converter warp
        mbar_init(bar(kPvBarODone), 1);
        mbar_init(bar(kPvBarDrain), 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_v);
        if (p.tma_load) prefetch_tensormap(&tm_s);
    }
    if (warp == kPvMmaWarp) {
        tmem_alloc(base + kPvOffMisc, 128u);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto drain_wait = [&](uint32_t b, uint32_t par) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(b, par) && globaltimer() - t0 < kCmDrainNs) {
        }
    };

    if (warp == kPvTmaWarp) {
        // ------------------------------------------------------------ vbar parts (lane i: box i)
        constexpr int kBoxes = 3 * kHalves;
        constexpr unsigned kMask = (1u << kBoxes) - 1u;
        if (lane < kBoxes) {
            const int part = lane / kHalves, h = lane % kHalves;
            bool ok = true;
            uint32_t issued[kPvStages] = {0u, 0u};
            for (int n = 0; n < slices; ++n) {
                const int slot = n % kPvStages;
                if (!(ok = __all_sync(kMask, bw.wait(bar(kPvBarBEmpty + slot), ((n / kPvStages) & 1) ^ 1)))) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(kPvBarBFull + slot), 3u * kPartB);
                    ++issued[slot];
                }
                __syncwarp(kMask);   // lane 0's expect_tx first
                tma_load_4d(base + kPvOffB + slot * kPvB + part * kPartB + h * 8192u, &tm_v, 64 * h, 64 * n, bh, part,
                            bar(kPvBarBFull + slot));
            }
            if (!ok && lane == 0)
                for (int s = 0; s < kPvStages; ++s)
                    if (issued[s]) drain_wait(bar(kPvBarBFull + s), (issued[s] - 1u) & 1u);
        }
    } else if (warp == kPvSWarp) {
        // ------------------------------------------------------------ score slices (lane i: keys 32i..32i+31)
        if (p.tma_load && lane < 2) {
            bool ok = true;
            uint32_t issued = 0;
            for (int n = 0; n < slices; ++n) {
                if (!(ok = __all_sync(0x3u, bw.wait(bar(kPvBarSEmpty), (n & 1) ^ 1)))) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(kPvBarSFull), 2u * kPvBoxS);
                    ++issued;
                }
                __syncwarp(0x3u);
                tma_load_3d(base + kPvOffS + lane * kPvBoxS, &tm_s, 64 * n + 32 * lane, i0, bh, bar(kPvBarSFull));
            }
            if (!ok && lane == 0 && issued) drain_wait(bar(kPvBarSFull), (issued - 1u) & 1u);
        }
    } else if (warp == kPvMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);     // P K-major, vbar MN-major
            const uint64_t fix_p = smem_desc_sw128(0, 16u, 1024u);       // K-major, 8-row groups 1 KB apart
            const uint64_t fix_v = smem_desc_sw128(0, 8192u, 1024u);     // MN-major, channel halves 8 KB apart
            bool ok = true, issued_any = false;
            for (int n = 0; ok && n < slices; ++n) {
                const int slot = n % kPvStages;
                const uint32_t par = (n / kPvStages) & 1;
                if (!(ok = bw.wait(bar(kPvBarAFull + slot), par))) break;
                if (!(ok = bw.wait(bar(kPvBarBFull + slot), par))) break;
                tc_fence_after();
                const uint32_t pa = base + kPvOffA + slot * kPvA, vb = base + kPvOffB + slot * kPvB;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                    for (int pr = 0; pr < 6; ++pr) {
                        mma_bf16_ss(tmem, desc_at(fix_p, pa + prod_a(pr) * 16384u + kk * 32u),
                                    desc_at(fix_v, vb + prod_b(pr) * kPartB + kk * 2048u), idesc,
                                    (n | kk | pr) != 0 ? 1u : 0u);
                    }
                }
                mma_commit(bar(kPvBarAEmpty + slot));
                mma_commit(bar(kPvBarBEmpty + slot));
                issued_any = true;
            }
            if (ok) mma_commit(bar(kPvBarODone));
            if (issued_any) {
                mma_commit(bar(kPvBarDrain));
                drain_wait(bar(kPvBarDrain), 0u);
            }
        }
    } else {
        // ------------------------------------------------------------ converters, then the epilogue
        const int r = threadIdx.x & 127, hf = threadIdx.x >> 7;   // query row, half of each 64-key slice
        const int gi = i0 + r;
        const bool real = gi < C;
        const float2 st = real ? p.stats[static_cast<int64_t>(bh) * C + gi] : make_float2(0.f, 0.f);
        constexpr float kLog2e = 1.4426950408889634f;
        const float mb = st.x * kLog2e;   // exp(s - m) = 2^(s log2(e) - m log2(e))
        const float* srow = p.scores + (static_cast<int64_t>(bh) * C + (real ? gi : 0)) * C;
        // keys 64n + 32hf .. + 31 of the row; past C (or a padding row): -inf, whose exp is 0
        auto load = [&](int n, float (&x)[32]) {
            const int jb = 64 * n + 32 * hf;
            if (real && (C & 3) == 0 && jb + 32 <= C) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 t = *reinterpret_cast<const float4*>(srow + jb + 4 * q);
                    x[4 * q] = t.x;
                    x[4 * q + 1] = t.y;
                    x[4 * q + 2] = t.z;
                    x[4 * q + 3] = t.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = (real && jb + e < C) ? srow[jb + e] : -INFINITY;
            }
        };
        bool ok = true;
        float nxt[32];
        if (!p.tma_load) load(0, nxt);
        for (int n = 0; n < slices; ++n) {
            float cur[32];
            if (p.tma_load) {
                if (!(ok = __all_sync(0xffffffffu, bw.wait(bar(kPvBarSFull), n & 1)))) break;
                const uint32_t src = base + kPvOffS + hf * kPvBoxS + r * 128u;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t a = src + ((static_cast<uint32_t>(c) ^ (r & 7u)) << 4);
                    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                 : "=f"(cur[4 * c]), "=f"(cur[4 * c + 1]), "=f"(cur[4 * c + 2]), "=f"(cur[4 * c + 3])
                                 : "r"(a)
                                 : "memory");
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kPvBarSEmpty));   // release: the slice is read
                // keys past C arrive as zeros from the copy; they weigh nothing
                const int jb = 64 * n + 32 * hf;
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (jb + e >= C) cur[e] = -INFINITY;
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) cur[e] = nxt[e];
                if (n + 1 < slices) load(n + 1, nxt);
            }
            const int slot = n % kPvStages;
            if (!(ok = __all_sync(0xffffffffu, bw.wait(bar(kPvBarAEmpty + slot), ((n / kPvStages) & 1) ^ 1)))) break;
            uint8_t* a = smem + kPvOffA + slot * kPvA + r * 128;
#pragma unroll
            for (int cq = 0; cq < 4; ++cq) {              // 16-byte chunk c = 4hf + cq: 8 keys
                uint32_t hw[4], mw[4], lw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    split3x2(ex2_approx(fmaf(cur[8 * cq + 2 * e], kLog2e, -mb)),
                             ex2_approx(fmaf(cur[8 * cq + 2 * e + 1], kLog2e, -mb)), hw[e], mw[e], lw[e]);
                const int sc = ((4 * hf + cq) ^ (r & 7)) * 16;   // the 128-byte swizzle of row r
                *reinterpret_cast<uint4*>(a + sc) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4*>(a + 16384 + sc) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
                *reinterpret_cast<uint4*>(a + 32768 + sc) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
            fence_proxy_async_smem();   // the stores become visible to the tensor cores
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kPvBarAFull + slot));
        }
        // warps 0-3 (rows 32 w .. 32 w + 31: their TMEM lane quarter) store the result
        if (warp < 4 && ok && __all_sync(0xffffffffu, bw.wait(bar(kPvBarODone), 0u))) {
            tc_fence_after();
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * warp) << 16);
            float* orow = p.o_coarse + (static_cast<int64_t>(bh) * C + (real ? gi : 0)) * D;
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t v[32];
                tmem_ld32_wait(lane_base + 32u * cc, v);
                if (real) {
                    float4* dst = reinterpret_cast<float4*>(orow + 32 * cc);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(__uint_as_float(v[4 * e]) * st.y, __uint_as_float(v[4 * e + 1]) * st.y,
                                             __uint_as_float(v[4 * e + 2]) * st.y,
                                             __uint_as_float(v[4 * e + 3]) * st.y);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kPvMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 128u);
    }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 cm_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// Split parts [3][B*H][C][D] bf16 as (D, C, B*H, part): box 64 channels x `rows` cubes, 128-byte swizzle.
bool encode_parts(CUtensorMap* m, const uint16_t* parts, const Dims& d, uint32_t rows) {
    auto fn = cm_encode_fn();
    if (!fn) return false;
    const cuuint64_t bh = static_cast<cuuint64_t>(d.B) * d.H;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d.D), static_cast<cuuint64_t>(d.C), bh, 3u};
    const cuuint64_t row = static_cast<cuuint64_t>(d.D) * 2u;
    const cuuint64_t strides[3] = {row, row * d.C, row * d.C * bh};
    const cuuint32_t box[4] = {64u, rows, 1u, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(parts), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scores [B*H][C][C] float32 as (C keys, C rows, B*H): box 32 keys x `rows` rows, 128-byte swizzle
// (the scores epilogue's staged blocks, the coarse output's slices).  Needs C % 4 == 0 (16-byte row
// pitch) and a 16-byte aligned base.
bool encode_scores(CUtensorMap* m, const float* scores, const Dims& d, uint32_t rows) {
    auto fn = cm_encode_fn();
    if (!fn || (d.C & 3) != 0 || (reinterpret_cast<uintptr_t>(scores) & 15u) != 0) return false;
    const cuuint64_t bh = static_cast<cuuint64_t>(d.B) * d.H;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d.C), static_cast<cuuint64_t>(d.C), bh};
    const cuuint64_t row = static_cast<cuuint64_t>(d.C) * 4u;
    const cuuint64_t strides[2] = {row, row * d.C};
    const cuuint32_t box[3] = {32u, rows, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(scores), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t split_parts_elems(const Dims& d) { return 3u * static_cast<size_t>(d.B) * d.H * d.C * d.D; }

cudaError_t launch_coarse_scores_mma(const Dims& d, const uint16_t* q_parts, const uint16_t* k_parts, float scale,
                                     float* scores, float* stats, cudaStream_t s, const char** why) {
    if (d.D != 128 && d.D != 64) return cudaErrorInvalidValue;
    CUtensorMap tq, tk, ts;
    if (!encode_parts(&tq, q_parts, d, 128u) || !encode_parts(&tk, k_parts, d, 128u)) {
        if (why) *why = "cuTensorMapEncodeTiled failed for the split pooled vectors";
        return cudaErrorInvalidValue;
    }
    // the TMA store where the layout allows it; otherwise the epilogue writes from registers
    const bool tma_store = encode_scores(&ts, scores, d, 32u);
    if (!tma_store) ts = tq;   // a valid map that the kernel never uses
    static int configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (!(dev >= 0 && dev < 64 && configured[dev])) {
        e = cudaFuncSetAttribute(coarse_scores_mma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kCmSmem));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(coarse_scores_mma_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(kCmSmem));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = 1;
    }
    CmParams p{};
    p.C = d.C;
    p.B = d.B;
    p.H = d.H;
    p.row_tiles = (d.C + 127) / 128;
    p.scale = scale;
    p.scores = scores;
    p.stats = reinterpret_cast<float2*>(stats);
    p.tma_store = tma_store ? 1 : 0;
    p.status = status_word();
    p.limit_ns = kWaitLimitNs;
    if (!p.status) {
        if (why) *why = "watchdog word unavailable";
        return cudaErrorInvalidValue;
    }
    const int64_t grid = static_cast<int64_t>(d.B) * d.H * p.row_tiles;
    if (grid > 0x7FFFFFFFll) return cudaErrorInvalidValue;
    if (d.D == 128) coarse_scores_mma_kernel<128><<<static_cast<unsigned>(grid), kCmThreads, kCmSmem, s>>>(tq, tk, ts, p);
    else coarse_scores_mma_kernel<64><<<static_cast<unsigned>(grid), kCmThreads, kCmSmem, s>>>(tq, tk, ts, p);
    return cudaGetLastError();
}

cudaError_t launch_coarse_pv_mma(const Dims& d, const float* scores, const float* stats, const uint16_t* v_parts,
                                 float* o_coarse, cudaStream_t s, const char** why) {
    if (d.D != 128 && d.D != 64) return cudaErrorInvalidValue;
    CUtensorMap tv, ts;
    if (!encode_parts(&tv, v_parts, d, 64u)) {
        if (why) *why = "cuTensorMapEncodeTiled failed for the split pooled values";
        return cudaErrorInvalidValue;
    }
    // score slices by TMA where the layout allows it; otherwise each converter thread loads its row
    const bool tma_load = encode_scores(&ts, scores, d, 128u);
    if (!tma_load) ts = tv;   // a valid map that the kernel never uses
    static int configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (!(dev >= 0 && dev < 64 && configured[dev])) {
        e = cudaFuncSetAttribute(coarse_pv_mma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kPvSmem));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(coarse_pv_mma_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(kPvSmem));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = 1;
    }
    PvParams p{};
    p.C = d.C;
    p.row_tiles = (d.C + 127) / 128;
    p.scores = scores;
    p.stats = reinterpret_cast<const float2*>(stats);
    p.o_coarse = o_coarse;
    p.tma_load = tma_load ? 1 : 0;
    p.status = status_word();
    p.limit_ns = kWaitLimitNs;
    if (!p.status) {
        if (why) *why = "watchdog word unavailable";
        return cudaErrorInvalidValue;
    }
    const int64_t grid = static_cast<int64_t>(d.B) * d.H * p.row_tiles;
    if (grid > 0x7FFFFFFFll) return cudaErrorInvalidValue;
    if (d.D == 128) coarse_pv_mma_kernel<128><<<static_cast<unsigned>(grid), kPvThreads, kPvSmem, s>>>(tv, ts, p);
    else coarse_pv_mma_kernel<64><<<static_cast<unsigned>(grid), kPvThreads, kPvSmem, s>>>(tv, ts, p);
    return cudaGetLastError();
}

}  // namespace vsa
