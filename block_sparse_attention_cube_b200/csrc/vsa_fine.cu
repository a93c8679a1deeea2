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
//    the merged, ordered union of the four selection lists, two key cubes
//    (128 keys, the N of QK^T) per step.  Rows of a cube that did not select
//    one of the step's cubes mask that cube's 64 columns; a tile none of whose
//    cubes selected either cube skips the step (no MMA, no softmax).  Dense
//    attention selects every cube for every row, so nothing is masked or
//    skipped.  Groups are four consecutive entries of an optional per-head
//    permutation of the query cubes (vsa_group orders cubes with similar
//    selections next to each other).
//  * Roles (warp specialisation, teardown section "Blackwell changes the
//    optimisation problem"): warp 0 issues TMA loads (the Q group, then the
//    step's K cubes through a 3-deep ring and V cubes through a separate
//    2-deep ring, so K slots recycle as soon as QK^T is done); warp 1
//    allocates all 512 tensor-memory columns and one thread issues the MMAs;
//    warps 2..5 run the softmax and epilogue of tile A and warps 6..9 those
//    of tile B, one query row per thread (warp w reads TMEM lane quarter w%4).
//  * Tensor memory, per tile: one 128x128 fp32 score buffer and a 128xD fp32
//    output accumulator.  The softmax writes P (bf16) over the first 64
//    columns of the scores it read and PV takes its A operand from there.
//    MMAs issued by one thread execute in order, so the next QK^T into the
//    buffer is issued right after the PV that reads its P.  The issue order
//    per step, S_A(i), PV_B(i-1), S_B(i), PV_A(i), lets each tile's softmax
//    run while the tensor cores work on the other tile.
//  * Softmax: online, in the log2 domain.  The running maximum starts at the
//    row's first tile maximum and moves only when a step's probabilities would
//    exceed 2^64 (the bound that keeps every later sum finite); moving it
//    rescales the accumulator, the denominator and any P already stored.  The
//    scores of step i arrive only after the tile's PV of step i-1 completed,
//    so the accumulator is stable then.  P is rounded to bf16; the
//    denominator sums the float32 probabilities; exponent arguments use
//    packed f32x2 FMA.  Teardown section "Fixed-max
//    softmax is a numerical contract": subtracting any common constant leaves
//    softmax unchanged; here the constant is bounded so no exponent overflows.
//  * Persistent CTAs (teardown section "Persistent kernel removes repeated
//    start-up cost"): one CTA per SM walks the work items of consecutive
//    heads, so the K/V of a head stay in L2 while its query groups use them.
//  * Every barrier wait is bounded; on expiry the CTA records VSA_ERR_TIMEOUT,
//    drains its own copies and MMAs, frees tensor memory and exits.  Each
//    barrier's producer can run at most one phase ahead of its consumer, so a
//    wait on a phase parity never aliases an older phase.
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
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kQTileBytes = 32768;   // 128 rows x 256 B (two 128-B column halves)
constexpr uint32_t kKVBytes = 32768;      // two cubes: [d 0-63: cube a, cube b][d 64-127: cube a, cube b]
constexpr uint32_t kOffQ = 0;                                  // [2 tiles]
constexpr uint32_t kOffK = kOffQ + 2 * kQTileBytes;            // [kKStages]
constexpr uint32_t kOffV = kOffK + kKStages * kKVBytes;        // [kVStages]
constexpr uint32_t kOffBar = kOffV + kVStages * kKVBytes;
// barrier slots
constexpr int kBarQFull = 0;
constexpr int kBarQEmpty = 1;
constexpr int kBarKFull = 2;                        // [kKStages]
constexpr int kBarKEmpty = kBarKFull + kKStages;
constexpr int kBarVFull = kBarKEmpty + kKStages;    // [kVStages]
constexpr int kBarVEmpty = kBarVFull + kVStages;
constexpr int kBarSFull = kBarVEmpty + kVStages;    // [tile]
constexpr int kBarPFull = kBarSFull + 2;            // [tile]
constexpr int kBarPVDone = kBarPFull + 2;           // [tile]
constexpr int kBarDrain = kBarPVDone + 2;
constexpr int kNumBars = kBarDrain + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;   // tmem slot (4 B) + abort flag (4 B)
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;     // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTileCols = 256;   // per tile: S at +0 (P over its first 64 columns), O at +128
constexpr uint32_t kColO = 128;
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

// Ordered union of the selection lists of the group's query cubes, two cubes
// per step.  Entries outside [0, C) are visited as the empty cube C.  Every
// entry of every list is consumed exactly once, duplicates included.  In
// `flags`, bit j (cube a) or bit 4 + j (cube b) is set when slot j's list
// holds that cube; cube b is -1 (empty, no flags) when the union runs out.
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
    __device__ __forceinline__ bool next1(int& cube, uint32_t& flags) {
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
    __device__ __forceinline__ bool next(int& cube_a, int& cube_b, uint32_t& flags) {
        uint32_t fa, fb = 0;
        if (!next1(cube_a, fa)) return false;
        if (!next1(cube_b, fb)) {
            cube_b = -1;
            fb = 0;
        }
        flags = fa | (fb << 4);
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

__device__ __forceinline__ bool tile_active(uint32_t flags, int t) { return (flags & (0x33u << (2 * t))) != 0u; }

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

// Scores of columns whose bit in `vm` is clear become -inf.
__device__ __forceinline__ void mask64(uint32_t (&s)[64], uint64_t vm) {
    if (vm == ~0ull) return;
    const uint32_t ninf = __float_as_uint(-INFINITY);
#pragma unroll
    for (int j = 0; j < 64; ++j)
        if (!((vm >> j) & 1ull)) s[j] = ninf;
}

__device__ __forceinline__ float max64(const uint32_t (&s)[64]) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = __uint_as_float(s[i]);
#pragma unroll
    for (int j = 8; j < 64; ++j) m[j & 7] = fmaxf(m[j & 7], __uint_as_float(s[j]));
    return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])), fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

constexpr float kSumLimit = 18446744073709551616.0f;   // 2^64: bound on any probability

// Maximum over both cubes' masked scores of this row: cube a in columns
// [taddr, taddr + 64) (skipped when vm_a is 0), cube b in [taddr + 64, taddr + 128).
// Warp-collective TMEM loads; used on a row's first step and on overflow only,
// so kept out of line.
__device__ __noinline__ float tile_max(uint32_t taddr, uint64_t vm_a, uint64_t vm_b) {
    uint32_t s[64];
    float m = -INFINITY;
    if (vm_a) {
        tmem_ld64_wait(taddr, s);
        mask64(s, vm_a);
        m = max64(s);
    }
    tmem_ld64_wait(taddr + 64u, s);
    mask64(s, vm_b);
    return fmaxf(m, max64(s));
}

// Probabilities 2^(s*c - m) of one cube's 64 masked scores: returned packed as
// 32 bf16 pairs in pk, their float32 sum as the result.
__device__ __forceinline__ float probs_half(uint32_t taddr, uint64_t vm, float c, float m, uint32_t (&pk)[32]) {
    uint32_t s[64];
    tmem_ld64_wait(taddr, s);
    mask64(s, vm);
    const uint64_t c2 = f32x2(c, c), nm2 = f32x2(-m, -m);
    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const uint64_t t = fma_f32x2(f32x2(__uint_as_float(s[2 * j]), __uint_as_float(s[2 * j + 1])), c2, nm2);
        float t0, t1;
        f32x2_split(t, t0, t1);
        const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
        acc[j & 3] = add_f32x2(acc[j & 3], f32x2(p0, p1));
        pk[j] = pack_bf16x2(p0, p1);
    }
    const uint64_t a2 = add_f32x2(add_f32x2(acc[0], acc[1]), add_f32x2(acc[2], acc[3]));
    float lo, hi;
    f32x2_split(a2, lo, hi);
    return lo + hi;
}

// Multiply `chunks` x 32 float32 columns of this row's tensor memory by alpha.
__device__ __forceinline__ void scale_tmem_f32(uint32_t taddr, int chunks, float alpha) {
#pragma unroll 1
    for (int ch = 0; ch < chunks; ++ch) {
        uint32_t o[32];
        tmem_ld32_wait(taddr + 32u * ch, o);
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
        tmem_st32(taddr + 32u * ch, o);
    }
}

// Multiply 32 columns of bf16 pairs (this row's stored P of one cube) by alpha.
__device__ __forceinline__ void scale_tmem_bf16(uint32_t taddr, float alpha) {
    uint32_t o[32];
    tmem_ld32_wait(taddr, o);
#pragma unroll
    for (int j = 0; j < 32; ++j)
        o[j] = pack_bf16x2(__uint_as_float(o[j] << 16) * alpha, __uint_as_float(o[j] & 0xFFFF0000u) * alpha);
    tmem_st32(taddr, o);
}

// Rare path of a cube half whose probabilities overflowed for some row of the
// warp: those rows move their maximum to the tile maximum and rescale O, l and
// (for half 1) the stored P of half 0; every row then recomputes the half and
// stores its P.  Warp-collective; returns the row's new sum.
struct RowState {
    float sum, m, l;   // the half's new sum, the row maximum and denominator after the move
};

template <int D>
__device__ __noinline__ RowState move_max_and_redo(uint32_t tcol, int h, uint64_t vm_a, uint64_t vm_b, float c,
                                                   bool over, bool row_active, float m_run, float l_run) {
    // half 1: only cube b's scores count (half 0's columns hold P by now)
    const float tmax = (h ? tile_max(tcol, 0ull, vm_b) : tile_max(tcol, vm_a, vm_b)) * c;
    float alpha = 1.f;
    if (over) {
        const float m_new = fmaxf(m_run, tmax);
        alpha = ex2_approx(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
    }
    // the tile's previous PV completed before these scores were committed
    scale_tmem_f32(tcol + kColO, D / 32, alpha);
    if (h == 1) scale_tmem_bf16(tcol, alpha);   // half 0's P is already stored
    uint32_t pk[32];
    float sum = 0.f;
    if (row_active) {
        sum = probs_half(tcol + 64u * h, h ? vm_b : vm_a, c, m_run, pk);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) pk[j] = 0u;
    }
    tmem_st32(tcol + 32u * h, pk);
    return RowState{sum, m_run, l_run};
}

// Shared-memory descriptor for a 1024-byte-aligned 128-byte-swizzled operand:
// the fixed fields once, the start address per use.
__device__ __forceinline__ uint64_t desc_at(uint64_t fixed, uint32_t saddr) {
    return fixed | static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
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
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(bar(kBarKFull + s), 1);
            mbar_init(bar(kBarKEmpty + s), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(bar(kBarVFull + s), 1);
            mbar_init(bar(kBarVEmpty + s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(kBarSFull + t), 1);
            mbar_init(bar(kBarPFull + t), 128);
            mbar_init(bar(kBarPVDone + t), 1);
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
    constexpr uint32_t kBytesKV = 2u * 64u * D * 2u;  // one step's two K (or V) cubes

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t q_issued = 0, k_issued[kKStages] = {}, v_issued[kVStages] = {};
            int64_t g = 0;
            int n_item = 0;
            bool ok = true;
            // two cubes into one stage: [d 0-63: a | b][d 64-127: a | b], 8 KB per box
            auto load_pair = [&](const CUtensorMap* m, uint32_t dst, int32_t ra, int32_t rb, uint32_t b) {
                tma_load_2d(dst, m, 0, ra, b);
                tma_load_2d(dst + 8192, m, 0, rb, b);
                if (D == 128) {
                    tma_load_2d(dst + 16384, m, 64, ra, b);
                    tma_load_2d(dst + 24576, m, 64, rb, b);
                }
            };
            for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x, ++n_item) {
                const Item item = decode_item(it, p);
                if (!(ok = bw.wait(bar(kBarQEmpty), (n_item & 1) ^ 1))) break;
                mbar_arrive_expect_tx(bar(kBarQFull), kBytesQ);
                ++q_issued;
                for (int t = 0; t < 2; ++t)
                    load_pair(&tm_q, base + kOffQ + t * kQTileBytes, tile_row(item.bh, item.cube[2 * t], p),
                              tile_row(item.bh, item.cube[2 * t + 1], p), bar(kBarQFull));
                GroupWalk w = make_walk(item, p);
                int ca, cb;
                uint32_t flags;
                while (w.next(ca, cb, flags)) {
                    const int32_t ra = tile_row(item.bh, ca, p), rb = tile_row(item.bh, cb, p);
                    const int ks = static_cast<int>(g % kKStages);
                    if (!(ok = bw.wait(bar(kBarKEmpty + ks), static_cast<uint32_t>((g / kKStages) & 1) ^ 1u))) break;
                    mbar_arrive_expect_tx(bar(kBarKFull + ks), kBytesKV);
                    ++k_issued[ks];
                    load_pair(&tm_k, base + kOffK + ks * kKVBytes, ra, rb, bar(kBarKFull + ks));
                    const int vs = static_cast<int>(g % kVStages);
                    if (!(ok = bw.wait(bar(kBarVEmpty + vs), static_cast<uint32_t>((g / kVStages) & 1) ^ 1u))) break;
                    mbar_arrive_expect_tx(bar(kBarVFull + vs), kBytesKV);
                    ++v_issued[vs];
                    load_pair(&tm_v, base + kOffV + vs * kKVBytes, ra, rb, bar(kBarVFull + vs));
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
                for (int s = 0; s < kKStages; ++s) drain(bar(kBarKFull + s), k_issued[s]);
                for (int s = 0; s < kVStages; ++s) drain(bar(kBarVFull + s), v_issued[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);   // Q (K-major) x K^T (K-major)
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);     // P (TMEM, K-major) x V (MN-major)
            const uint64_t fix_k = smem_desc_sw128(0, 16u, 1024u);         // K-major, 8-row groups 1 KB apart
            const uint64_t fix_v = smem_desc_sw128(0, 16384u, 1024u);      // MN-major, d halves 16 KB apart
            int64_t g = 0;
            uint32_t n_s[2] = {0, 0}, n_p[2] = {0, 0};   // per-tile S and PV steps issued
            int n_item = 0;
            bool ok = true, issued_any = false;
            bool acc[2] = {false, false};                 // O of the tile already holds this item's sum
            auto issue_s = [&](int t, int ks) {
                const uint32_t qa = base + kOffQ + t * kQTileBytes;
                const uint32_t kb = base + kOffK + ks * kKVBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                    mma_bf16_ss(tmem + t * kTileCols, desc_at(fix_k, qa + off), desc_at(fix_k, kb + off), idesc_s,
                                kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(kBarSFull + t));
                ++n_s[t];
                issued_any = true;
            };
            // PV of tile t for the step whose V sits in stage vs (waits for its P and V)
            auto issue_pv = [&](int t, int64_t gs) -> bool {
                const int vs = static_cast<int>(gs % kVStages);
                if (!bw.wait(bar(kBarPFull + t), n_p[t] & 1u)) return false;
                if (!bw.wait(bar(kBarVFull + vs), static_cast<uint32_t>((gs / kVStages) & 1))) return false;
                tc_fence_after();
                const uint32_t vb = base + kOffV + vs * kKVBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tmem + t * kTileCols + kColO, tmem + t * kTileCols + 8u * kk,
                                desc_at(fix_v, vb + kk * 2048u), idesc_o, (!acc[t] && kk == 0) ? 0u : 1u);
                acc[t] = true;
                mma_commit(bar(kBarPVDone + t));
                ++n_p[t];
                return true;
            };
            for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x, ++n_item) {
                const Item item = decode_item(it, p);
                if (!(ok = bw.wait(bar(kBarQFull), n_item & 1))) break;
                acc[0] = acc[1] = false;
                GroupWalk w = make_walk(item, p);
                int ca, cb;
                uint32_t flags;
                bool pend_b = false;   // PV of tile B for the previous step still to issue
                int64_t g_prev = -1;
                while (w.next(ca, cb, flags)) {
                    const int ks = static_cast<int>(g % kKStages);
                    if (!(ok = bw.wait(bar(kBarKFull + ks), static_cast<uint32_t>((g / kKStages) & 1)))) break;
                    tc_fence_after();
                    const bool act_a = tile_active(flags, 0), act_b = tile_active(flags, 1);
                    if (act_a) issue_s(0, ks);                                  // S_A(i)
                    if (pend_b && !(ok = issue_pv(1, g_prev))) break;           // PV_B(i-1)
                    if (g_prev >= 0) mma_commit(bar(kBarVEmpty + static_cast<int>(g_prev % kVStages)));
                    if (act_b) issue_s(1, ks);                                  // S_B(i)
                    mma_commit(bar(kBarKEmpty + ks));
                    if (act_a && !(ok = issue_pv(0, g))) break;                 // PV_A(i)
                    pend_b = act_b;
                    g_prev = g;
                    ++g;
                }
                if (!ok) break;
                mma_commit(bar(kBarQEmpty));
                if (pend_b && !(ok = issue_pv(1, g_prev))) break;
                if (g_prev >= 0) mma_commit(bar(kBarVEmpty + static_cast<int>(g_prev % kVStages)));
            }
            if (issued_any) {
                // all MMAs of this CTA complete before tensor memory is freed
                mma_commit(bar(kBarDrain));
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(bar(kBarDrain), 0) && globaltimer() - t0 < kDrainLimitNs) {
                }
            }
            (void)n_s;
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int tile = (warp - 2) >> 2;        // 0: warps 2..5, 1: warps 6..9
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int row = q * 32 + lane;           // query row of the tile, 0..127
        const int slot = 2 * tile + (q >> 1);    // query-cube slot of the group
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t tcol = tmem + tile * kTileCols + lane_addr;
        const uint32_t bar_sfull = bar(kBarSFull + tile), bar_pfull = bar(kBarPFull + tile);
        const uint32_t bar_pvdone = bar(kBarPVDone + tile);
        const float c = p.c_log2;
        uint32_t n = 0;   // steps this tile has taken part in (same count as the MMA issuer's)
        bool ok = true;
        auto wait_all = [&](uint32_t b, uint32_t par) -> bool {
            const bool mine = bw.wait(b, par);
            return __all_sync(0xffffffffu, mine);
        };
        for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x) {
            const Item item = decode_item(it, p);
            GroupWalk w = make_walk(item, p);
            float m_run = -INFINITY, l_run = 0.f;
            uint32_t steps = 0;
            int ca, cb;
            uint32_t flags;
            while (w.next(ca, cb, flags)) {
                if (!tile_active(flags, tile)) continue;      // the tile skips this step
                if (!(ok = wait_all(bar_sfull, n & 1u))) break;
                tc_fence_after();
                // warp-uniform: this warp's rows belong to one query cube
                const uint64_t vm_a = ((flags >> slot) & 1u) ? cube_key_mask(ca, p) : 0ull;
                const uint64_t vm_b = ((flags >> (4 + slot)) & 1u) ? cube_key_mask(cb, p) : 0ull;
                const bool row_active = (vm_a | vm_b) != 0ull;   // warp-uniform
                // the row's first step with keys: the running maximum starts at the tile maximum
                if (row_active && m_run == -INFINITY) {
                    m_run = tile_max(tcol, vm_a, vm_b) * c;
                    l_run = 0.f;
                }
                // P per cube half h, from the scores in columns [64h, 64h + 64), stored as bf16
                // pairs over columns [32h, 32h + 32).  A half whose probabilities would exceed
                // 2^64 (the lazy maximum fell far behind) moves the maximum up first; the
                // scores of both halves are intact until half 0's P is stored.
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    uint32_t pk[32];
                    float sum = 0.f;
                    const uint64_t vm = h ? vm_b : vm_a;
                    if (row_active) sum = probs_half(tcol + 64u * h, vm, c, m_run, pk);
                    const bool over = !(sum <= kSumLimit);
                    if (__any_sync(0xffffffffu, over)) {
                        const RowState r = move_max_and_redo<D>(tcol, h, vm_a, vm_b, c, over, row_active, m_run, l_run);
                        sum = r.sum;
                        m_run = r.m;
                        l_run = r.l;
                    } else {
                        if (!row_active) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) pk[j] = 0u;
                        }
                        tmem_st32(tcol + 32u * h, pk);
                    }
                    l_run += sum;
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_pfull);
                ++n;
                ++steps;
            }
            if (!ok) break;
            if (steps == 0) continue;   // the tile holds no query cube of this group
            // ---------------- epilogue: O / l and log-sum-exp of this tile's rows
            // PV(n-2) completed before S(n-1) was committed, so this parity cannot alias
            if (!(ok = wait_all(bar_pvdone, (n - 1) & 1u))) break;
            tc_fence_after();
            const int cube_row = item.cube[slot];
            const bool store = cube_row >= 0;
            const int64_t grow = item.bh * p.Npad + static_cast<int64_t>(store ? cube_row : 0) * 64 + (row & 63);
            const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
#pragma unroll 1
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t o[32];
                tmem_ld32_wait(tcol + kColO + 32u * ch, o);
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
