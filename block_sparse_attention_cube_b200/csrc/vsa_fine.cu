// Fine stage of Video Sparse Attention on sm_100a tensor cores.
//
// Method (Wan2.2 teardown, zharfai.com, section "Video sparse attention
// selects cubes", part 2): every 64-token query cube attends, token by token,
// to the tokens of the key/value cubes selected for it; padded key tokens are
// excluded.  With every cube selected this is dense bidirectional attention
// softmax(q k^T / sqrt(d)) v (Wan2.1 acceleration article, bafh001.com,
// section 4.2).
//
// Design (re-derived for B200, not taken from the pages' Hopper/Triton
// kernels):
//  * Work item = (b, h, pair of query cubes 2p and 2p+1): 128 query rows, the
//    M = 128 of one tcgen05.mma.  The pair walks the merged, ordered union of
//    its two selection lists; at each step one 64-token key cube is loaded and
//    the rows of a cube that did not select it are masked (dense attention
//    selects every cube for both, so no row is ever masked there).
//  * Roles (warp specialisation, teardown section "Blackwell changes the
//    optimisation problem"): warp 0 issues TMA loads (Q pair, then K and V
//    cubes through a 4-deep ring with separate K and V barriers so that K
//    slots recycle as soon as QK^T is done); warp 1 allocates tensor memory
//    and one thread issues the MMAs; warps 2..5 (one per TMEM lane quarter)
//    run the softmax and the epilogue, one query row per thread.
//  * Tensor memory: two 128x64 fp32 score buffers (QK^T of step s+1 runs
//    while the softmax of step s reads the other) and a 128xD fp32 output
//    accumulator.
//  * Softmax: online, in the log2 domain, with a lazily updated row maximum
//    (rescaling the accumulator only when the maximum grows by more than
//    2^8); P is rounded to bf16 and written to shared memory in the operand
//    layout; the denominator sums the float32 probabilities.  Teardown section
//    "Fixed-max softmax is a numerical contract": subtracting any common
//    constant leaves softmax unchanged; here the constant is bounded so no
//    exponent overflows.
//  * Persistent CTAs (teardown section "Persistent kernel removes repeated
//    start-up cost"): one CTA per SM walks the work items of consecutive
//    heads, so the K/V of a head stay in L2 while all its query pairs use them.
//  * Every barrier wait is bounded; on expiry the CTA records VSA_ERR_TIMEOUT,
//    drains its own copies and MMAs, frees tensor memory and exits.
#include <cmath>
#include <climits>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "ptx_sm100.cuh"
#include "vsa_internal.h"

namespace vsa {

__device__ int g_vsa_status;   // watchdog word (VSA_OK or VSA_ERR_TIMEOUT)

namespace {

using namespace ptx;

constexpr int kThreads = 192;
constexpr int kStages = 4;
constexpr uint32_t kQBytes = 32768;     // 128 rows x 256 B (two 128-B column halves)
constexpr uint32_t kKVBytes = 16384;    // 64 rows x 256 B
constexpr uint32_t kPBytes = 16384;     // 128 rows x 128 B
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + 2 * kQBytes;
constexpr uint32_t kOffV = kOffK + kStages * kKVBytes;
constexpr uint32_t kOffP = kOffV + kStages * kKVBytes;
constexpr uint32_t kOffBar = kOffP + kPBytes;
// barrier slots
constexpr int kBarQFull = 0;                    // [2]
constexpr int kBarQEmpty = 2;                   // [2]
constexpr int kBarKFull = 4;                    // [kStages]
constexpr int kBarKEmpty = kBarKFull + kStages;
constexpr int kBarVFull = kBarKEmpty + kStages;
constexpr int kBarVEmpty = kBarVFull + kStages;
constexpr int kBarSFull = kBarVEmpty + kStages; // [2]
constexpr int kBarSEmpty = kBarSFull + 2;       // [2]
constexpr int kBarPFull = kBarSEmpty + 2;
constexpr int kBarPVDone = kBarPFull + 1;
constexpr int kBarDrain = kBarPVDone + 1;
constexpr int kNumBars = kBarDrain + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;   // tmem slot (4 B) + abort flag (4 B)
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;     // + alignment slack
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;     // S buffer b at column 64*b
constexpr uint32_t kColO = 128;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s for draining after an abort

struct FineParams {
    const int32_t* idx;   // [B, H, C, k] or nullptr (all cubes)
    uint16_t* o;          // [B, H, Npad, D]
    float* lse;           // [B, H, Npad] or nullptr
    int k;
    int H, C, Cx, Cy, T, X, Y;
    int npairs;
    int64_t Npad;
    int64_t items;
    int32_t oob_row;      // a row index outside the tiled tensors (TMA fills zeros)
    float c_log2;         // scale * log2(e)
    int* status;
    uint64_t limit_ns;
};

// Ordered union of the selection lists of the two query cubes of a pair.
// Entries outside [0, C) are visited as the empty cube C.  Every entry of
// either list is consumed exactly once, duplicates included.
struct PairWalk {
    const int32_t* a;
    const int32_t* b;
    int k, C;
    bool dense, has_b;
    int ia, ib;

    __device__ __forceinline__ int head(const int32_t* l, int i, bool present) const {
        if (!present) return INT_MAX;
        if (dense) return i < C ? i : INT_MAX;
        if (i >= k) return INT_MAX;
        const int v = __ldg(l + i);
        return (v < 0 || v >= C) ? C : v;
    }
    __device__ __forceinline__ bool next(int& cube, uint32_t& flags) {
        const int ha = head(a, ia, true), hb = head(b, ib, has_b);
        if (ha == INT_MAX && hb == INT_MAX) return false;
        cube = min(ha, hb);
        flags = (ha == cube ? 1u : 0u) | (hb == cube ? 2u : 0u);
        ia += (flags & 1u) ? 1 : 0;
        ib += (flags & 2u) ? 1 : 0;
        return true;
    }
};

struct Item {
    int64_t bh;
    int cube_a, cube_b;
    bool has_b;
};

__device__ __forceinline__ Item decode_item(int64_t it, const FineParams& p) {
    Item r;
    const int pair = static_cast<int>(it % p.npairs);
    r.bh = it / p.npairs;
    r.cube_a = 2 * pair;
    r.cube_b = 2 * pair + 1;
    r.has_b = r.cube_b < p.C;
    return r;
}

__device__ __forceinline__ PairWalk make_walk(const Item& item, const FineParams& p) {
    PairWalk w;
    w.dense = p.idx == nullptr;
    w.k = p.k;
    w.C = p.C;
    w.has_b = item.has_b;
    const int32_t* base = w.dense ? nullptr : p.idx + item.bh * p.C * static_cast<int64_t>(p.k);
    w.a = w.dense ? nullptr : base + static_cast<int64_t>(item.cube_a) * p.k;
    w.b = (w.dense || !item.has_b) ? nullptr : base + static_cast<int64_t>(item.cube_b) * p.k;
    w.ia = 0;
    w.ib = 0;
    return w;
}

// Bit o is set when offset o of cube j holds a real token.
__device__ __forceinline__ uint64_t cube_key_mask(int j, const FineParams& p) {
    if (j < 0 || j >= p.C) return 0ull;
    const int ct = j / (p.Cx * p.Cy), cx = (j / p.Cy) % p.Cx, cy = j % p.Cy;
    const int nt = min(4, p.T - 4 * ct), nx = min(4, p.X - 4 * cx), ny = min(4, p.Y - 4 * cy);
    if (nt == 4 && nx == 4 && ny == 4) return ~0ull;
    const uint64_t my = static_cast<uint64_t>((1u << ny) - 1u) * 0x1111111111111111ull;
    uint32_t ex = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (i < nx) ex |= 0xFu << (4 * i);
    const uint64_t mx = static_cast<uint64_t>(ex) * 0x0001000100010001ull;
    uint64_t mt = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (i < nt) mt |= 0xFFFFull << (16 * i);
    return my & mx & mt;
}

__device__ __forceinline__ int32_t tile_row(const Item& item, int cube, const FineParams& p) {
    if (cube < 0 || cube >= p.C) return p.oob_row;
    return static_cast<int32_t>(item.bh * p.Npad + static_cast<int64_t>(cube) * 64);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fine_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const FineParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base = (raw_u32 + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_u32);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto bar = [&](int i) -> uint32_t { return base + kOffBar + 8u * static_cast<uint32_t>(i); };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    const BoundedWait bw{abort_flag, p.status, p.limit_ns};

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(kBarQFull + i), 1);
            mbar_init(bar(kBarQEmpty + i), 1);
            mbar_init(bar(kBarSFull + i), 1);
            mbar_init(bar(kBarSEmpty + i), 128);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(kBarKFull + s), 1);
            mbar_init(bar(kBarKEmpty + s), 1);
            mbar_init(bar(kBarVFull + s), 1);
            mbar_init(bar(kBarVEmpty + s), 1);
        }
        mbar_init(bar(kBarPFull), 128);
        mbar_init(bar(kBarPVDone), 1);
        mbar_init(bar(kBarDrain), 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(base + kOffMisc, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    constexpr uint32_t kRowBytesQ = 128u * D * 2u;   // bytes of one Q pair load
    constexpr uint32_t kRowBytesKV = 64u * D * 2u;   // bytes of one K or V cube load

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t q_issued[2] = {0, 0}, k_issued[kStages] = {}, v_issued[kStages] = {};
            int64_t g = 0;
            int n_item = 0;
            bool ok = true;
            for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x, ++n_item) {
                const Item item = decode_item(it, p);
                const int qb = n_item & 1;
                if (!(ok = bw.wait(bar(kBarQEmpty + qb), ((n_item >> 1) & 1) ^ 1))) break;
                mbar_arrive_expect_tx(bar(kBarQFull + qb), kRowBytesQ);
                ++q_issued[qb];
                const uint32_t qdst = base + kOffQ + qb * kQBytes;
                const int32_t ra = tile_row(item, item.cube_a, p);
                const int32_t rb = item.has_b ? tile_row(item, item.cube_b, p) : p.oob_row;
                tma_load_2d(qdst, &tm_q, 0, ra, bar(kBarQFull + qb));
                tma_load_2d(qdst + 8192, &tm_q, 0, rb, bar(kBarQFull + qb));
                if (D == 128) {
                    tma_load_2d(qdst + 16384, &tm_q, 64, ra, bar(kBarQFull + qb));
                    tma_load_2d(qdst + 24576, &tm_q, 64, rb, bar(kBarQFull + qb));
                }
                PairWalk w = make_walk(item, p);
                int cube;
                uint32_t flags;
                while (w.next(cube, flags)) {
                    const int st = static_cast<int>(g % kStages);
                    const uint32_t par = static_cast<uint32_t>((g / kStages) & 1) ^ 1u;
                    const int32_t row = tile_row(item, cube, p);
                    if (!(ok = bw.wait(bar(kBarKEmpty + st), par))) break;
                    mbar_arrive_expect_tx(bar(kBarKFull + st), kRowBytesKV);
                    ++k_issued[st];
                    const uint32_t kdst = base + kOffK + st * kKVBytes;
                    tma_load_2d(kdst, &tm_k, 0, row, bar(kBarKFull + st));
                    if (D == 128) tma_load_2d(kdst + 8192, &tm_k, 64, row, bar(kBarKFull + st));
                    if (!(ok = bw.wait(bar(kBarVEmpty + st), par))) break;
                    mbar_arrive_expect_tx(bar(kBarVFull + st), kRowBytesKV);
                    ++v_issued[st];
                    const uint32_t vdst = base + kOffV + st * kKVBytes;
                    tma_load_2d(vdst, &tm_v, 0, row, bar(kBarVFull + st));
                    if (D == 128) tma_load_2d(vdst + 8192, &tm_v, 64, row, bar(kBarVFull + st));
                    ++g;
                }
            }
            if (!ok) {
                // wait for this CTA's own copies still in flight before exiting
                const BoundedWait dw{abort_flag, p.status, kDrainLimitNs};
                auto drain = [&](uint32_t b, uint32_t issued) {
                    if (issued == 0) return;
                    const uint32_t par = (issued - 1u) & 1u;
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(b, par) && globaltimer() - t0 < dw.limit_ns) {
                    }
                };
                for (int i = 0; i < 2; ++i) drain(bar(kBarQFull + i), q_issued[i]);
                for (int s = 0; s < kStages; ++s) {
                    drain(bar(kBarKFull + s), k_issued[s]);
                    drain(bar(kBarVFull + s), v_issued[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);   // Q (K-major) x K^T (K-major)
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);    // P (K-major) x V (MN-major)
            int64_t g = 0;
            int n_item = 0;
            bool ok = true;
            bool issued_any = false;
            auto issue_pv = [&](int64_t gs, bool first) -> bool {
                if (!bw.wait(bar(kBarPFull), static_cast<uint32_t>(gs & 1))) return false;
                const int st = static_cast<int>(gs % kStages);
                if (!bw.wait(bar(kBarVFull + st), static_cast<uint32_t>((gs / kStages) & 1))) return false;
                tc_fence_after();
                const uint32_t pa = base + kOffP;
                const uint32_t vb = base + kOffV + st * kKVBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t adesc = smem_desc_sw128(pa + kk * 32u, 16u, 1024u);
                    const uint64_t bdesc = smem_desc_sw128(vb + kk * 2048u, 8192u, 1024u);
                    mma_bf16_ss(tmem + kColO, adesc, bdesc, idesc_o, (first && kk == 0) ? 0u : 1u);
                }
                mma_commit(bar(kBarPVDone));
                mma_commit(bar(kBarVEmpty + st));
                return true;
            };
            for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x, ++n_item) {
                const Item item = decode_item(it, p);
                const int qb = n_item & 1;
                if (!(ok = bw.wait(bar(kBarQFull + qb), (n_item >> 1) & 1))) break;
                PairWalk w = make_walk(item, p);
                int cube;
                uint32_t flags;
                int64_t s = 0;
                while (ok && w.next(cube, flags)) {
                    const int64_t gs = g + s;
                    const int st = static_cast<int>(gs % kStages);
                    const int sb = static_cast<int>(gs & 1);
                    if (!(ok = bw.wait(bar(kBarKFull + st), static_cast<uint32_t>((gs / kStages) & 1)))) break;
                    if (!(ok = bw.wait(bar(kBarSEmpty + sb), static_cast<uint32_t>(((gs >> 1) & 1) ^ 1)))) break;
                    tc_fence_after();
                    const uint32_t qa = base + kOffQ + qb * kQBytes;
                    const uint32_t kb = base + kOffK + st * kKVBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t koff = (kk >> 2) * 8192u + (kk & 3) * 32u;
                        const uint64_t adesc = smem_desc_sw128(qa + (kk >> 2) * 16384u + (kk & 3) * 32u, 16u, 1024u);
                        const uint64_t bdesc = smem_desc_sw128(kb + koff, 16u, 1024u);
                        mma_bf16_ss(tmem + kColS + 64u * sb, adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    issued_any = true;
                    mma_commit(bar(kBarSFull + sb));
                    mma_commit(bar(kBarKEmpty + st));
                    if (s > 0) ok = issue_pv(gs - 1, s == 1);
                    ++s;
                }
                if (!ok) break;
                mma_commit(bar(kBarQEmpty + qb));
                if (s > 0) ok = issue_pv(g + s - 1, s == 1);
                g += s;
            }
            if (issued_any) {
                // all MMAs of this CTA complete before tensor memory is freed
                mma_commit(bar(kBarDrain));
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(bar(kBarDrain), 0) && globaltimer() - t0 < kDrainLimitNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int row = q * 32 + lane;          // query row of the pair, 0..127
        const int half = q >> 1;                // 0: first cube, 1: second cube
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        uint8_t* prow = smem + kOffP + row * 128;
        const float c = p.c_log2;
        int64_t g = 0;
        bool ok = true;
        auto wait_all = [&](uint32_t b, uint32_t par) -> bool {
            const bool mine = bw.wait(b, par);
            return __all_sync(0xffffffffu, mine);
        };
        for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x) {
            const Item item = decode_item(it, p);
            PairWalk w = make_walk(item, p);
            float m_run = -INFINITY, l_run = 0.f;
            int cube;
            uint32_t flags;
            while (w.next(cube, flags)) {
                const int sb = static_cast<int>(g & 1);
                if (!(ok = wait_all(bar(kBarSFull + sb), static_cast<uint32_t>((g >> 1) & 1)))) break;
                tc_fence_after();
                const bool active = (flags >> half) & 1u;    // warp-uniform
                uint32_t sa[32], sbv[32];
                if (active) {
                    tmem_ld32(tmem + lane_addr + kColS + 64u * sb, sa);
                    tmem_ld32(tmem + lane_addr + kColS + 64u * sb + 32u, sbv);
                    tmem_wait_ld();
                }
                tc_fence_before();
                mbar_arrive(bar(kBarSEmpty + sb));

                uint32_t pk[32];
                bool rescale_o = false;
                float alpha_o = 1.f;     // factor applied to this row of O (1 unless rescaled)
                if (active) {
                    const uint64_t vm = cube_key_mask(cube, p);
                    float mt = -INFINITY;
                    if (vm == ~0ull) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) mt = fmaxf(mt, fmaxf(__uint_as_float(sa[j]), __uint_as_float(sbv[j])));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            if ((vm >> j) & 1ull) mt = fmaxf(mt, __uint_as_float(sa[j]));
                            if ((vm >> (j + 32)) & 1ull) mt = fmaxf(mt, __uint_as_float(sbv[j]));
                        }
                    }
                    const float mts = mt * c;
                    if (mts > m_run + kRescaleLog2) {
                        // before the row's first valid key, O and l hold nothing for it
                        if (m_run != -INFINITY) {
                            alpha_o = ex2_approx(m_run - mts);
                            rescale_o = true;
                            l_run *= alpha_o;
                        } else {
                            l_run = 0.f;
                        }
                        m_run = mts;
                    }
                    const float neg_m = -m_run;
                    float lsum = 0.f;
                    if (m_run == -INFINITY) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) pk[j] = 0u;
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            float p0 = ex2_approx(fmaf(__uint_as_float(sa[2 * j]), c, neg_m));
                            float p1 = ex2_approx(fmaf(__uint_as_float(sa[2 * j + 1]), c, neg_m));
                            float p2 = ex2_approx(fmaf(__uint_as_float(sbv[2 * j]), c, neg_m));
                            float p3 = ex2_approx(fmaf(__uint_as_float(sbv[2 * j + 1]), c, neg_m));
                            if (vm != ~0ull) {
                                if (!((vm >> (2 * j)) & 1ull)) p0 = 0.f;
                                if (!((vm >> (2 * j + 1)) & 1ull)) p1 = 0.f;
                                if (!((vm >> (2 * j + 32)) & 1ull)) p2 = 0.f;
                                if (!((vm >> (2 * j + 33)) & 1ull)) p3 = 0.f;
                            }
                            pk[j] = pack_bf16x2(p0, p1);
                            pk[16 + j] = pack_bf16x2(p2, p3);
                            lsum += (p0 + p1) + (p2 + p3);
                        }
                    }
                    l_run += lsum;
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) pk[j] = 0u;
                }

                // the P buffer and the O accumulator are free once PV of the previous step is done
                if (g > 0 && !(ok = wait_all(bar(kBarPVDone), static_cast<uint32_t>((g - 1) & 1)))) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale_o)) {
#pragma unroll
                    for (int ch = 0; ch < D / 32; ++ch) {
                        uint32_t o[32];
                        const uint32_t ta = tmem + lane_addr + kColO + 32u * ch;
                        tmem_ld32(ta, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha_o);
                        tmem_st32(ta, o);
                    }
                    tmem_wait_st();
                }
                // P row: 64 bf16 = 8 chunks of 16 B, 128-byte swizzle (chunk c at c ^ (row & 7))
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint4 v = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
                    *reinterpret_cast<uint4*>(prow + ((ch ^ (row & 7)) << 4)) = v;
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(bar(kBarPFull));
                ++g;
            }
            if (!ok) break;
            // ---------------- epilogue: O / l and log-sum-exp of this item's rows
            if (!(ok = wait_all(bar(kBarPVDone), static_cast<uint32_t>((g - 1) & 1)))) break;
            tc_fence_after();
            const bool store = (half == 0) || item.has_b;
            const int cube_row = (half == 0) ? item.cube_a : item.cube_b;
            const int64_t grow = item.bh * p.Npad + static_cast<int64_t>(cube_row) * 64 + (row & 63);
            const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_addr + kColO + 32u * ch, o);
                tmem_wait_ld();
                if (store) {
                    uint32_t w16[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        w16[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * inv_l, __uint_as_float(o[2 * j + 1]) * inv_l);
                    uint4* dst = reinterpret_cast<uint4*>(p.o + grow * D + 32 * ch);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(w16[4 * v], w16[4 * v + 1], w16[4 * v + 2], w16[4 * v + 3]);
                }
            }
            if (store && p.lse != nullptr)
                p.lse[grow] = l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

__global__ void wait_probe_kernel(int* status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar_storage;
    __shared__ int abort_flag;
    const uint32_t b = smem_u32(&bar_storage);
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(b, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const BoundedWait bw{&abort_flag, status, limit_ns};
    (void)bw.wait(b, 0);   // nothing arrives: gives up after limit_ns
    __syncthreads();
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool encode_rows(CUtensorMap* m, const void* ptr, int D, int64_t rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2u};
    const cuuint32_t box[2] = {64u, 64u};
    const cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t set_smem_attr() {
    static int done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(fine_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = 1;
    return e;
}

}  // namespace

int* status_word() {
    static int* ptrs[64] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_vsa_status) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int*>(a);
    }
    return ptrs[dev];
}

cudaError_t launch_fine(const Dims& d, const uint16_t* qt, const uint16_t* kt, const uint16_t* vt,
                        const int32_t* idx, int k, float scale, uint16_t* o_fine, float* lse, cudaStream_t s,
                        const char** why) {
    CUtensorMap tq, tk, tv;
    if (!encode_rows(&tq, qt, d.D, d.rows) || !encode_rows(&tk, kt, d.D, d.rows) ||
        !encode_rows(&tv, vt, d.D, d.rows)) {
        if (why) *why = "cuTensorMapEncodeTiled failed for a tiled Q/K/V tensor";
        return cudaErrorInvalidValue;
    }
    FineParams p{};
    p.idx = idx;
    p.o = o_fine;
    p.lse = lse;
    p.k = idx ? k : d.C;
    p.H = d.H;
    p.C = d.C;
    p.Cx = d.Cx;
    p.Cy = d.Cy;
    p.T = d.T;
    p.X = d.X;
    p.Y = d.Y;
    p.npairs = (d.C + 1) / 2;
    p.Npad = d.Npad;
    p.items = static_cast<int64_t>(d.B) * d.H * p.npairs;
    p.oob_row = static_cast<int32_t>(d.rows);
    p.c_log2 = scale * 1.4426950408889634f;
    p.status = status_word();
    p.limit_ns = kWaitLimitNs;
    if (!p.status) {
        if (why) *why = "watchdog word unavailable";
        return cudaErrorInvalidValue;
    }
    const int grid = static_cast<int>(p.items < sm_count() ? p.items : sm_count());
    cudaError_t e;
    if (d.D == 128) {
        if ((e = set_smem_attr<128>()) != cudaSuccess) return e;
        fine_kernel<128><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, p);
    } else {
        if ((e = set_smem_attr<64>()) != cudaSuccess) return e;
        fine_kernel<64><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, p);
    }
    return cudaGetLastError();
}

cudaError_t launch_wait_probe(uint64_t limit_ns, cudaStream_t s) {
    int* st = status_word();
    if (!st) return cudaErrorInvalidValue;
    wait_probe_kernel<<<1, 32, 0, s>>>(st, limit_ns);
    return cudaGetLastError();
}

}  // namespace vsa
