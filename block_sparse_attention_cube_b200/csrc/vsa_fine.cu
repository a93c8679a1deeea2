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
//  * Work item = (b, h, group of four query cubes).  The four cubes form two
//    128-row tiles (the M = 128 of one tcgen05.mma), A = cubes 0-1 and
//    B = cubes 2-3 of the group, which share one K/V stream: the item walks
//    the merged, ordered union of the four selection lists and each step
//    loads one 64-token key cube.  Rows of a cube that did not select the
//    step's cube are masked; a tile none of whose cubes selected it skips the
//    step (no MMA, no softmax).  Dense attention selects every cube for every
//    row, so nothing is masked or skipped.  Groups are four consecutive
//    entries of an optional per-head permutation of the query cubes (vsa_group
//    orders cubes with similar selections next to each other).
//  * Roles (warp specialisation, teardown section "Blackwell changes the
//    optimisation problem"): warp 0 issues TMA loads (the Q group, then K and V
//    cubes through a 4-deep ring with separate K and V barriers so a K slot
//    recycles as soon as QK^T is done); warp 1 allocates all 512 tensor-memory
//    columns and one thread issues the MMAs; warps 2..5 run the softmax and
//    epilogue of tile A and warps 6..9 those of tile B, one query row per
//    thread (warp w reads TMEM lane quarter w % 4).
//  * Tensor memory, per tile: two 128x64 fp32 score buffers (QK^T of a later
//    step runs while the softmax reads the other) and a 128xD fp32 output
//    accumulator.  The softmax writes P (bf16) over the first 32 columns of
//    the score buffer it read, and PV takes its A operand from there, so P
//    never goes through shared memory; the buffer is released by the commit
//    of that PV.
//  * Softmax: online, in the log2 domain, with a lazily updated row maximum
//    (the accumulator is rescaled only when the maximum grows by more than
//    2^8); P is rounded to bf16; the denominator sums the float32
//    probabilities.  Teardown section
//    "Fixed-max softmax is a numerical contract": subtracting any common
//    constant leaves softmax unchanged; here the constant is bounded so no
//    exponent overflows.
//  * Persistent CTAs (teardown section "Persistent kernel removes repeated
//    start-up cost"): one CTA per SM walks the work items of consecutive
//    heads, so the K/V of a head stay in L2 while its query groups use them.
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

constexpr int kThreads = 320;          // producer warp, MMA warp, 2 x 4 softmax warps
constexpr int kStages = 4;
constexpr uint32_t kQTileBytes = 32768;   // 128 rows x 256 B (two 128-B column halves)
constexpr uint32_t kKVBytes = 16384;      // 64 rows x 256 B
constexpr uint32_t kOffQ = 0;                                  // [2 tiles]
constexpr uint32_t kOffK = kOffQ + 2 * kQTileBytes;            // [kStages]
constexpr uint32_t kOffV = kOffK + kStages * kKVBytes;         // [kStages]
constexpr uint32_t kOffBar = kOffV + kStages * kKVBytes;
// barrier slots
constexpr int kBarQFull = 0;
constexpr int kBarQEmpty = 1;
constexpr int kBarKFull = 2;                       // [kStages]
constexpr int kBarKEmpty = kBarKFull + kStages;
constexpr int kBarVFull = kBarKEmpty + kStages;
constexpr int kBarVEmpty = kBarVFull + kStages;
constexpr int kBarSFull = kBarVEmpty + kStages;    // [tile][buffer]
constexpr int kBarSEmpty = kBarSFull + 4;          // [tile][buffer]
constexpr int kBarPFull = kBarSEmpty + 4;          // [tile][buffer]
constexpr int kBarPVDone = kBarPFull + 4;          // [tile][buffer]
constexpr int kBarDrain = kBarPVDone + 4;
constexpr int kNumBars = kBarDrain + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;   // tmem slot (4 B) + abort flag (4 B)
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;     // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTileCols = 256;   // per tile: S buffers at +0 and +64 (P over their first 32), O at +128
constexpr uint32_t kColO = 128;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s for draining after an abort

struct FineParams {
    const int32_t* idx;     // [B, H, C, k] or nullptr (all cubes)
    const int32_t* order;   // [B, H, C] permutation of query cubes, or nullptr (identity)
    uint16_t* o;            // [B, H, Npad, D]
    float* lse;             // [B, H, Npad] or nullptr
    int k;
    int C, Ct, Cx, Cy, T, X, Y;
    int ngroups;            // ceil(C / 4)
    uint64_t magic_cxcy;    // floor(2^48 / (Cx*Cy)) + 1: exact j / (Cx*Cy) for j < 2^24
    uint64_t magic_cy;      // floor(2^48 / Cy) + 1
    int64_t Npad;
    int64_t items;
    int32_t oob_row;        // a row index outside the tiled tensors (TMA fills zeros)
    float c_log2;           // scale * log2(e)
    int* status;
    uint64_t limit_ns;
};

__device__ __forceinline__ uint32_t div_magic(uint32_t j, uint64_t magic) {
    return static_cast<uint32_t>((static_cast<uint64_t>(j) * magic) >> 48);
}

// The four query cubes of one work item (slot j < 0 when absent).
struct Item {
    int64_t bh;
    int cube[4];
    uint32_t present;   // bit j set when slot j holds a query cube
};

__device__ __forceinline__ Item decode_item(int64_t it, const FineParams& p) {
    Item r;
    const int g = static_cast<int>(it % p.ngroups);
    r.bh = it / p.ngroups;
    r.present = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int pos = 4 * g + j;
        int c = -1;
        if (pos < p.C) {
            c = p.order ? __ldg(p.order + r.bh * p.C + pos) : pos;
            if (c < 0 || c >= p.C) c = -1;
        }
        r.cube[j] = c;
        r.present |= (c >= 0 ? 1u : 0u) << j;
    }
    return r;
}

// Ordered union of the selection lists of the group's query cubes.  Entries
// outside [0, C) are visited as the empty cube C.  Every entry of every list
// is consumed exactly once, duplicates included.  `flags` bit j is set when
// slot j's list holds the step's cube.
struct GroupWalk {
    const int32_t* lst[4];
    int pos[4];
    int k, C;
    uint32_t present;
    bool dense;

    __device__ __forceinline__ int head(int j) const {
        if (!((present >> j) & 1u)) return INT_MAX;
        if (dense) return pos[j] < C ? pos[j] : INT_MAX;
        if (pos[j] >= k) return INT_MAX;
        const int v = __ldg(lst[j] + pos[j]);
        return (v < 0 || v >= C) ? C : v;
    }
    __device__ __forceinline__ bool next(int& cube, uint32_t& flags) {
        int h[4];
        int m = INT_MAX;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            h[j] = head(j);
            m = min(m, h[j]);
        }
        if (m == INT_MAX) return false;
        cube = m;
        flags = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (h[j] == m) {
                flags |= 1u << j;
                ++pos[j];
            }
        }
        return true;
    }
};

__device__ __forceinline__ GroupWalk make_walk(const Item& item, const FineParams& p) {
    GroupWalk w;
    w.dense = p.idx == nullptr;
    w.k = p.k;
    w.C = p.C;
    w.present = item.present;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        w.pos[j] = 0;
        w.lst[j] = (w.dense || item.cube[j] < 0)
                       ? nullptr
                       : p.idx + (item.bh * p.C + item.cube[j]) * static_cast<int64_t>(p.k);
    }
    return w;
}

// Bit o is set when offset o of cube j holds a real token.
__device__ __forceinline__ uint64_t cube_key_mask(int j, const FineParams& p) {
    if (j < 0 || j >= p.C) return 0ull;
    const uint32_t ct = div_magic(static_cast<uint32_t>(j), p.magic_cxcy);
    const uint32_t rem = static_cast<uint32_t>(j) - ct * static_cast<uint32_t>(p.Cx * p.Cy);
    const uint32_t cx = div_magic(rem, p.magic_cy);
    const uint32_t cy = rem - cx * static_cast<uint32_t>(p.Cy);
    const int nt = min(4, p.T - 4 * static_cast<int>(ct));
    const int nx = min(4, p.X - 4 * static_cast<int>(cx));
    const int ny = min(4, p.Y - 4 * static_cast<int>(cy));
    if ((nt & nx & ny) == 4) return ~0ull;
    const uint64_t my = static_cast<uint64_t>((1u << ny) - 1u) * 0x1111111111111111ull;
    const uint32_t ex = (0xFFFFu >> (16 - 4 * nx));                  // nx nibbles of 0xF
    const uint64_t mx = static_cast<uint64_t>(ex) * 0x0001000100010001ull;
    const uint64_t mt = (nt == 4) ? ~0ull : ((1ull << (16 * nt)) - 1ull);
    return my & mx & mt;
}

__device__ __forceinline__ int32_t tile_row(int64_t bh, int cube, const FineParams& p) {
    if (cube < 0 || cube >= p.C) return p.oob_row;
    return static_cast<int32_t>(bh * p.Npad + static_cast<int64_t>(cube) * 64);
}

__device__ __forceinline__ float max64(const uint32_t (&s)[64]) {
    float m[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        m[i] = fmaxf(fmaxf(__uint_as_float(s[4 * i]), __uint_as_float(s[4 * i + 1])),
                     fmaxf(__uint_as_float(s[4 * i + 2]), __uint_as_float(s[4 * i + 3])));
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
    return m[0];
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
        mbar_init(bar(kBarQFull), 1);
        mbar_init(bar(kBarQEmpty), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(kBarKFull + s), 1);
            mbar_init(bar(kBarKEmpty + s), 1);
            mbar_init(bar(kBarVFull + s), 1);
            mbar_init(bar(kBarVEmpty + s), 1);
        }
        // Per-buffer barriers keep every producer at most one phase ahead of its
        // consumer (P(n+2) needs S(n+2), which needs PV(n) to have read P(n)),
        // so waiting on a phase parity never aliases an older phase.
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar(kBarSFull + i), 1);
            mbar_init(bar(kBarSEmpty + i), 1);   // released by the commit after the PV that read its P
            mbar_init(bar(kBarPFull + i), 128);
            mbar_init(bar(kBarPVDone + i), 1);
        }
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

    constexpr uint32_t kBytesQ = 4u * 64u * D * 2u;   // one Q group load
    constexpr uint32_t kBytesKV = 64u * D * 2u;       // one K or V cube load

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t q_issued = 0, k_issued[kStages] = {}, v_issued[kStages] = {};
            int64_t g = 0;
            int n_item = 0;
            bool ok = true;
            for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x, ++n_item) {
                const Item item = decode_item(it, p);
                if (!(ok = bw.wait(bar(kBarQEmpty), (n_item & 1) ^ 1))) break;
                mbar_arrive_expect_tx(bar(kBarQFull), kBytesQ);
                ++q_issued;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t dst = base + kOffQ + (j >> 1) * kQTileBytes + (j & 1) * 8192u;
                    const int32_t row = tile_row(item.bh, item.cube[j], p);
                    tma_load_2d(dst, &tm_q, 0, row, bar(kBarQFull));
                    if (D == 128) tma_load_2d(dst + 16384, &tm_q, 64, row, bar(kBarQFull));
                }
                GroupWalk w = make_walk(item, p);
                int cube;
                uint32_t flags;
                while (w.next(cube, flags)) {
                    const int st = static_cast<int>(g % kStages);
                    const uint32_t par = static_cast<uint32_t>((g / kStages) & 1) ^ 1u;
                    const int32_t row = tile_row(item.bh, cube, p);
                    if (!(ok = bw.wait(bar(kBarKEmpty + st), par))) break;
                    mbar_arrive_expect_tx(bar(kBarKFull + st), kBytesKV);
                    ++k_issued[st];
                    const uint32_t kdst = base + kOffK + st * kKVBytes;
                    tma_load_2d(kdst, &tm_k, 0, row, bar(kBarKFull + st));
                    if (D == 128) tma_load_2d(kdst + 8192, &tm_k, 64, row, bar(kBarKFull + st));
                    if (!(ok = bw.wait(bar(kBarVEmpty + st), par))) break;
                    mbar_arrive_expect_tx(bar(kBarVFull + st), kBytesKV);
                    ++v_issued[st];
                    const uint32_t vdst = base + kOffV + st * kKVBytes;
                    tma_load_2d(vdst, &tm_v, 0, row, bar(kBarVFull + st));
                    if (D == 128) tma_load_2d(vdst + 8192, &tm_v, 64, row, bar(kBarVFull + st));
                    ++g;
                }
            }
            if (!ok) {
                // wait for this CTA's own copies still in flight before exiting
                auto drain = [&](uint32_t b, uint32_t issued) {
                    if (issued == 0) return;
                    const uint32_t par = (issued - 1u) & 1u;
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(b, par) && globaltimer() - t0 < kDrainLimitNs) {
                    }
                };
                drain(bar(kBarQFull), q_issued);
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
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);    // P (TMEM, K-major) x V (MN-major)
            int64_t g = 0;
            uint32_t n_s[2] = {0, 0}, n_p[2] = {0, 0};   // per-tile counts of S and PV steps issued
            int n_item = 0;
            bool ok = true, issued_any = false;
            bool pv_started[2] = {false, false};
            // PV of step `gp` for the tiles active in `fl`, then release its V stage
            auto issue_pv = [&](uint32_t fl, int64_t gp) -> bool {
                const int st = static_cast<int>(gp % kStages);
                bool v_ready = false;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (!((fl >> (2 * t)) & 3u)) continue;
                    if (!bw.wait(bar(kBarPFull + 2 * t + (n_p[t] & 1u)), (n_p[t] >> 1) & 1u)) return false;
                    if (!v_ready) {
                        if (!bw.wait(bar(kBarVFull + st), static_cast<uint32_t>((gp / kStages) & 1))) return false;
                        v_ready = true;
                    }
                    tc_fence_after();
                    const uint32_t sb = n_p[t] & 1u;   // P of this step sits over its S buffer
                    const uint32_t pa = tmem + t * kTileCols + 64u * sb;
                    const uint32_t vb = base + kOffV + st * kKVBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bdesc = smem_desc_sw128(vb + kk * 2048u, 8192u, 1024u);
                        mma_bf16_ts(tmem + t * kTileCols + kColO, pa + 8u * kk, bdesc, idesc_o,
                                    (!pv_started[t] && kk == 0) ? 0u : 1u);
                    }
                    pv_started[t] = true;
                    mma_commit(bar(kBarPVDone + 2 * t + sb));   // also covers every earlier MMA
                    mma_commit(bar(kBarSEmpty + 2 * t + sb));
                    ++n_p[t];
                }
                mma_commit(bar(kBarVEmpty + st));
                return true;
            };
            for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x, ++n_item) {
                const Item item = decode_item(it, p);
                if (!(ok = bw.wait(bar(kBarQFull), n_item & 1))) break;
                pv_started[0] = pv_started[1] = false;
                GroupWalk w = make_walk(item, p);
                int cube;
                uint32_t flags, prev_flags = 0;
                int64_t prev_g = -1;
                while (ok && w.next(cube, flags)) {
                    const int st = static_cast<int>(g % kStages);
                    if (!(ok = bw.wait(bar(kBarKFull + st), static_cast<uint32_t>((g / kStages) & 1)))) break;
                    const uint32_t kb = base + kOffK + st * kKVBytes;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (!((flags >> (2 * t)) & 3u)) continue;
                        const uint32_t sb = n_s[t] & 1u;
                        if (!(ok = bw.wait(bar(kBarSEmpty + 2 * t + sb), ((n_s[t] >> 1) & 1u) ^ 1u))) break;
                        tc_fence_after();
                        const uint32_t qa = base + kOffQ + t * kQTileBytes;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t adesc =
                                smem_desc_sw128(qa + (kk >> 2) * 16384u + (kk & 3) * 32u, 16u, 1024u);
                            const uint64_t bdesc = smem_desc_sw128(kb + (kk >> 2) * 8192u + (kk & 3) * 32u, 16u, 1024u);
                            mma_bf16_ss(tmem + t * kTileCols + 64u * sb, adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
                        }
                        issued_any = true;
                        mma_commit(bar(kBarSFull + 2 * t + sb));
                        ++n_s[t];
                    }
                    if (!ok) break;
                    mma_commit(bar(kBarKEmpty + st));
                    if (prev_g >= 0 && !(ok = issue_pv(prev_flags, prev_g))) break;
                    prev_flags = flags;
                    prev_g = g;
                    ++g;
                }
                if (!ok) break;
                mma_commit(bar(kBarQEmpty));
                if (prev_g >= 0 && !(ok = issue_pv(prev_flags, prev_g))) break;
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
        const int tile = (warp - 2) >> 2;        // 0: warps 2..5, 1: warps 6..9
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int row = q * 32 + lane;           // query row of the tile, 0..127
        const int slot = 2 * tile + (q >> 1);    // query-cube slot of the group
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t tcol = tmem + tile * kTileCols;
        const uint32_t bar_sfull = bar(kBarSFull + 2 * tile);
        const uint32_t bar_pfull = bar(kBarPFull + 2 * tile), bar_pvdone = bar(kBarPVDone + 2 * tile);
        const float c = p.c_log2;
        uint32_t n = 0;   // steps this tile has taken part in (same count as the MMA issuer's)
        bool ok = true;
        auto wait_all = [&](uint32_t b, uint32_t par) -> bool {
            const bool mine = bw.wait(b, par);
            return __all_sync(0xffffffffu, mine);
        };
        const uint32_t tile_mask = 3u << (2 * tile);
        for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x) {
            const Item item = decode_item(it, p);
            GroupWalk w = make_walk(item, p);
            float m_run = -INFINITY, l_run = 0.f;
            uint32_t steps = 0;
            int cube;
            uint32_t flags;
            while (w.next(cube, flags)) {
                if (!(flags & tile_mask)) continue;    // tile skips this step
                const uint32_t sb = n & 1u;
                if (!(ok = wait_all(bar_sfull + 8u * sb, (n >> 1) & 1u))) break;
                tc_fence_after();
                const bool active = (flags >> slot) & 1u;    // warp-uniform
                uint32_t s[64];
                if (active) tmem_ld64_wait(tcol + lane_addr + 64u * sb, s);

                // s[] is reused in place: after the exponentials s[0..31] hold P as bf16 pairs
                bool rescale_o = false;
                float alpha_o = 1.f;     // factor applied to this row of O (1 unless rescaled)
                if (active) {
                    const uint64_t vm = cube_key_mask(cube, p);
                    if (vm != ~0ull) {
                        const uint32_t ninf = __float_as_uint(-INFINITY);
#pragma unroll
                        for (int j = 0; j < 64; ++j)
                            if (!((vm >> j) & 1ull)) s[j] = ninf;
                    }
                    const float mts = max64(s) * c;
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
                    if (m_run == -INFINITY) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) s[j] = 0u;
                    } else {
                        const float neg_m = -m_run;
                        float acc[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float p0 = ex2_approx(fmaf(__uint_as_float(s[2 * j]), c, neg_m));
                            const float p1 = ex2_approx(fmaf(__uint_as_float(s[2 * j + 1]), c, neg_m));
                            acc[j & 7] += p0 + p1;
                            s[j] = pack_bf16x2(p0, p1);   // s[j] was consumed at iteration j/2 <= j
                        }
                        l_run += ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) s[j] = 0u;
                }

                if (__any_sync(0xffffffffu, rescale_o)) {
                    // the O accumulator is stable once the tile's previous PV (n-1) is done
                    if (n > 0 && !(ok = wait_all(bar_pvdone + 8u * ((n - 1) & 1u), ((n - 1) >> 1) & 1u))) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int ch = 0; ch < D / 32; ++ch) {
                        uint32_t o[32];
                        const uint32_t ta = tcol + lane_addr + kColO + 32u * ch;
                        tmem_ld32_wait(ta, o);
#pragma unroll
                        for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha_o);
                        tmem_st32(ta, o);
                    }
                }
                // P (bf16 pairs in s[0..31]) over the first 32 columns of this step's S buffer
                tmem_st32(tcol + lane_addr + 64u * sb, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_pfull + 8u * sb);
                ++n;
                ++steps;
            }
            if (!ok) break;
            if (steps == 0) continue;   // the tile holds no query cube of this group
            // ---------------- epilogue: O / l and log-sum-exp of this tile's rows
            // the commit of PV(n-1) covers every earlier MMA of the CTA
            if (!(ok = wait_all(bar_pvdone + 8u * ((n - 1) & 1u), ((n - 1) >> 1) & 1u))) break;
            tc_fence_after();
            const int cube_row = item.cube[slot];
            const bool store = cube_row >= 0;
            const int64_t grow = item.bh * p.Npad + static_cast<int64_t>(store ? cube_row : 0) * 64 + (row & 63);
            const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
#pragma unroll 1
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t o[32];
                tmem_ld32_wait(tcol + lane_addr + kColO + 32u * ch, o);
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

uint64_t magic48(uint32_t d) { return ((uint64_t{1} << 48) / d) + 1; }

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
                        const int32_t* idx, int k, const int32_t* order, float scale, uint16_t* o_fine,
                        float* lse, cudaStream_t s, const char** why) {
    CUtensorMap tq, tk, tv;
    if (!encode_rows(&tq, qt, d.D, d.rows) || !encode_rows(&tk, kt, d.D, d.rows) ||
        !encode_rows(&tv, vt, d.D, d.rows)) {
        if (why) *why = "cuTensorMapEncodeTiled failed for a tiled Q/K/V tensor";
        return cudaErrorInvalidValue;
    }
    FineParams p{};
    p.idx = idx;
    p.order = order;
    p.o = o_fine;
    p.lse = lse;
    p.k = idx ? k : d.C;
    p.C = d.C;
    p.Ct = d.Ct;
    p.Cx = d.Cx;
    p.Cy = d.Cy;
    p.T = d.T;
    p.X = d.X;
    p.Y = d.Y;
    p.ngroups = (d.C + 3) / 4;
    p.magic_cxcy = magic48(static_cast<uint32_t>(d.Cx * d.Cy));
    p.magic_cy = magic48(static_cast<uint32_t>(d.Cy));
    p.Npad = d.Npad;
    p.items = static_cast<int64_t>(d.B) * d.H * p.ngroups;
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
