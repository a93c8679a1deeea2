// Fine stage of Video Sparse Attention on sm_100a tensor cores.
//
// Method (Wan2.2 teardown, zharfai.com, section "Video sparse attention
// selects cubes", part 2): every 64-token query cube attends, token by token,
// to the tokens of the key/value cubes selected for it; padded key tokens are
// excluded.  With every cube selected this is dense bidirectional attention
// softmax(q k^T / sqrt(d)) v (Wan2.1 acceleration article, bafh001.com,
// section 4.2), which does not depend on the token order at all.
//
// Design (re-derived for B200, not taken from the pages' Hopper/Triton
// kernels):
//  * A "block" is 64 tokens of one (batch, head).  Three ways to fetch one
//    with TMA (one 64-row x 128-byte box per 64 channels):
//      tiled  - a cube of the cube-major tiled tensor [B, H, Npad, D];
//      cubes  - the same cube gathered straight from the projection layout
//               [B, N, H, D] by a 5-D box (64 channels x 4 y x 4 x x 4 t),
//               padded positions zero-filled by the copy engine, so no
//               tiling pass is needed;
//      tokens - 64 consecutive tokens of [B, N, H, D] (dense attention over
//               the real tokens only, no padding).
//  * Work item = (b, h, group of four query blocks).  The four blocks form
//    two 128-row tiles (the M = 128 of one tcgen05.mma), A = blocks 0-1 and
//    B = blocks 2-3, which share one K/V stream: the item walks the merged,
//    ordered union of the four selection lists, two key blocks (128 keys,
//    the N of QK^T) per step.  Rows of a block that did not select one of the
//    step's blocks mask that block's 64 columns; a tile none of whose blocks
//    selected either block skips the step.  Dense attention selects every
//    block for every row.  Groups are four consecutive entries of an optional
//    per-head permutation of the query cubes (vsa_group orders cubes with
//    similar selections next to each other).
//  * Roles (warp specialisation, teardown section "Blackwell changes the
//    optimisation problem"): warp 16 walks the selections and issues TMA (the
//    Q group, then the step's K blocks and V blocks through two 2-deep rings,
//    so K slots recycle as soon as QK^T is done); for sparse selections it
//    publishes each step (its two key blocks and which query blocks selected
//    them) in an 8-deep shared-memory ring, so no other role repeats the
//    walk.  Warp 17 allocates all 512 tensor-memory columns and one thread
//    issues the MMAs.  Warps 0..15 run the softmax and epilogue, one query row
//    per thread, two warps per TMEM lane quarter of a tile: one takes the
//    first 64 of a step's 128 key columns, the other the last 64, so a tile's
//    softmax runs as two halves in parallel (warp w reads lane quarter w%4).
//    The two agree on each row's running maximum and add their row sums
//    through a double-buffered shared slot guarded by a two-arrival mbarrier.
//  * Tensor memory, per tile: one 128x128 fp32 score buffer and a 128xD fp32
//    output accumulator.  Each half's softmax writes its P (bf16 pairs) over
//    the first 32 columns of its own 64 score columns, and PV takes its A
//    operand from there.  MMAs issued by one thread execute in order, so the
//    next QK^T into the buffer is issued right after the PV that reads its P.
//    The issue order per step, S_A(i), PV_B(i-1), S_B(i), PV_A(i), lets each
//    tile's softmax run while the tensor cores work on the other tile.
//  * Softmax: online, in the log2 domain.  The running maximum starts at the
//    maximum of the row's first scores (over both halves) and moves only when
//    a step's probabilities in either half would exceed 2^64 (the bound that
//    keeps every later sum finite); moving it rescales the accumulator and the
//    denominators and recomputes the step, whose P is stored only once both
//    halves agree.  The scores of step i arrive only after the tile's PV of
//    step i-1 completed, so the accumulator is stable then.  P is rounded to
//    bf16; the denominator sums the float32 probabilities.  Teardown section
//    "Fixed-max softmax is a numerical contract": subtracting any common
//    constant leaves softmax unchanged; here the constant is bounded so no
//    exponent overflows.
//  * Epilogue: O / l either to the tiled output (plus log-sum-exp), or, fused,
//    the gated merge of part 3 of the method, g_c * O_c[cube] + g_f * O / l,
//    written straight to the token's row of [B, N, H, D] (the untiling).
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

constexpr int kThreads = 576;          // 2 tiles x 2 halves x 4 softmax warps, then the TMA and MMA warps
constexpr int kTmaWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kRing = 8;               // published steps (sparse selections)
constexpr uint32_t kQTileBytes = 32768;   // 128 rows x 256 B (two 128-B column halves)
constexpr uint32_t kKVBytes = 32768;      // two blocks: [d 0-63: block a, block b][d 64-127: block a, block b]
constexpr uint32_t kOffQ = 0;                                  // [2 tiles]
constexpr uint32_t kOffK = kOffQ + 2 * kQTileBytes;            // [kKStages]
constexpr uint32_t kOffV = kOffK + kKStages * kKVBytes;        // [kVStages]
constexpr uint32_t kOffRec = kOffV + kVStages * kKVBytes;      // [kRing] x 16 B
constexpr uint32_t kOffXch = kOffRec + kRing * 16;             // [2 buffers][2 tiles][4 quarters][2 halves][32] floats
constexpr uint32_t kXchBytes = 2 * 2 * 4 * 2 * 32 * 4;
constexpr uint32_t kOffBar = kOffXch + kXchBytes;
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
constexpr int kBarRecFull = kBarPVDone + 2;         // [kRing]
constexpr int kBarRecEmpty = kBarRecFull + kRing;   // [kRing]
constexpr int kBarPair = kBarRecEmpty + kRing;      // [tile * 4 + lane quarter]: the two half warps
constexpr int kBarDrain = kBarPair + 8;
constexpr int kNumBars = kBarDrain + 1;
constexpr uint32_t kRecConsumers = 1 + 16;          // the MMA thread and the sixteen softmax warps
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;   // tmem slot (4 B) + abort flag (4 B)
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;     // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTileCols = 256;   // per tile: S at +0 (P over its first 64 columns), O at +128
constexpr uint32_t kColO = 128;
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s for draining after an abort
static_assert(kSmemBytes <= 232448, "shared memory over the 227 KB per-block limit");

enum LoadMode : int { kLoadTiled = 0, kLoadCubes = 1, kLoadTokens = 2 };

struct FineParams {
    const int32_t* idx;     // [B, H, C, k] or nullptr (every block)
    const int32_t* order;   // [B, H, C] permutation of query cubes, or nullptr (identity)
    const uint2* steps;     // precomputed steps [items][steps_stride] (schedule_kernel), or nullptr (walk here)
    int64_t steps_stride;
    uint16_t* o;            // tiled O [B, H, Npad, D], or the merged output [B, N, H, D] (fused)
    float* lse;             // [B, H, Npad] or nullptr (tiled output only)
    const float* o_coarse;  // [B, H, C, D] or nullptr (fused only; no coarse term)
    const uint16_t* g_coarse;   // [B, N, H] or nullptr (gate 0)
    const uint16_t* g_fine;     // [B, N, H] or nullptr (gate 1)
    int k;                  // selections per query block (nblk when idx is nullptr)
    int B, H;
    int nblk;               // blocks per head: C (cube modes) or ceil(N / 64) (token mode)
    int C, Ct, Cx, Cy, T, X, Y;
    int64_t N;
    int group;              // query blocks per work item: 4 (two tiles, fine_kernel) or 2 (one tile, fine_tile_kernel)
    int ngroups;            // ceil(nblk / group)
    uint64_t magic_cxcy;    // floor(2^48 / (Cx*Cy)) + 1: exact j / (Cx*Cy) for j < 2^24
    uint64_t magic_cy;      // floor(2^48 / Cy) + 1
    uint64_t magic_cx;      // floor(2^48 / Cx) + 1
    uint64_t mask_t, mask_x, mask_y;   // real offsets of a cube in the last cube layer along t, x, y
    int64_t Npad;
    int64_t items;
    int32_t oob_row;        // a row index outside the tiled tensors (TMA fills zeros)
    float c_log2;           // scale * log2(e)
    int* status;
    uint64_t limit_ns;
    int* overflow;          // fine_tile_kernel: set to 1 when a probability bound was exceeded (or nullptr)
    int* work;              // fine_tile_kernel: item counter, zero at launch (nullptr: every gridDim.x-th item)
    const int* run_if;      // fine_kernel: return at once unless *run_if != 0 (or nullptr: always run)
};

__device__ __forceinline__ uint32_t div_magic(uint32_t j, uint64_t magic) {
    return static_cast<uint32_t>((static_cast<uint64_t>(j) * magic) >> 48);
}

// The query blocks of one work item (slot j < 0 when absent; slots past p.group are absent).
struct Item {
    int64_t bh;
    int b, h;
    int blk[4];
    uint32_t present;   // bit j set when slot j holds a query block
};

// Item counts fit in 31 bits (make_params' callers check), so the divisions are 32-bit ones.
__device__ __forceinline__ Item decode_item(int64_t it, const FineParams& p) {
    Item r;
    const uint32_t itu = static_cast<uint32_t>(it), ng = static_cast<uint32_t>(p.ngroups);
    const uint32_t bh = itu / ng, nh = static_cast<uint32_t>(p.H);
    const int g = static_cast<int>(itu - bh * ng);
    const uint32_t b = bh / nh;
    r.bh = bh;
    r.b = static_cast<int>(b);
    r.h = static_cast<int>(bh - b * nh);
    r.present = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int pos = p.group * g + j;
        int c = -1;
        if (j < p.group && pos < p.nblk) {
            c = p.order ? __ldg(p.order + r.bh * p.C + pos) : pos;
            if (c < 0 || c >= p.nblk) c = -1;
        }
        r.blk[j] = c;
        r.present |= (c >= 0 ? 1u : 0u) << j;
    }
    return r;
}

// One step of an item: key blocks a and b (b = -1 when the union ran out; an
// index outside [0, nblk) is the empty block), bit j (block a) or 4 + j
// (block b) of `flags` set when query slot j selected it, `last` on the
// item's final step.
struct StepRec {
    int32_t ca, cb;
    uint32_t flags;
    uint32_t last;
};

__device__ __forceinline__ StepRec dense_step(int s, uint32_t present, int nblk) {
    StepRec r;
    r.ca = 2 * s;
    r.cb = 2 * s + 1 < nblk ? 2 * s + 1 : -1;
    r.flags = present | (r.cb >= 0 ? present << 4 : 0u);
    r.last = 2 * s + 2 >= nblk ? 1u : 0u;
    return r;
}

// Ordered union of the selection lists of the group's query blocks, two
// blocks per step (run by the producer lane only).  Entries outside [0, C)
// are visited as the empty block C.  Every entry of every list is consumed
// exactly once, duplicates included.
struct GroupWalk {
    const int32_t* lst[4];
    int pos[4];
    int k, C;
    uint32_t present;

    __device__ __forceinline__ int head(int j) const {
        if (!((present >> j) & 1u) || pos[j] >= k) return INT_MAX;
        const int v = __ldg(lst[j] + pos[j]);
        return (v < 0 || v >= C) ? C : v;
    }
    __device__ __forceinline__ bool next1(int& blk, uint32_t& flags) {
        int h[4];
        int m = INT_MAX;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            h[j] = head(j);
            m = min(m, h[j]);
        }
        if (m == INT_MAX) return false;
        blk = m;
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
    __device__ __forceinline__ bool done() const {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (((present >> j) & 1u) && pos[j] < k) return false;
        return true;
    }
    // Next step of the union; false once it is exhausted.
    __device__ __forceinline__ bool next(StepRec& r) {
        uint32_t fa, fb = 0;
        int a, b;
        if (!next1(a, fa)) return false;
        if (!next1(b, fb)) {
            b = -1;
            fb = 0;
        }
        r.ca = a;
        r.cb = b;
        r.flags = fa | (fb << 4);
        r.last = done() ? 1u : 0u;
        return true;
    }
};

__device__ __forceinline__ GroupWalk make_walk(const Item& item, const FineParams& p) {
    GroupWalk w;
    w.k = p.k;
    w.C = p.C;
    w.present = item.present;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        w.pos[j] = 0;
        w.lst[j] = item.blk[j] < 0 ? p.idx : p.idx + (item.bh * p.C + item.blk[j]) * static_cast<int64_t>(p.k);
    }
    return w;
}

// Entries of the union in three passes: those only tile A's query blocks
// selected, then only tile B's, then both tiles' (pairing like with like
// leaves fewer tiles half-used in a step).
struct TileWalk {
    GroupWalk w0, w;
    int pass;
    __device__ __forceinline__ bool next_entry(int& blk, uint32_t& fl) {
        for (;;) {
            if (!w.next1(blk, fl)) {
                if (++pass == 3) return false;
                w = w0;
                continue;
            }
            const int pat = ((fl & 3u) ? 1 : 0) | ((fl & 12u) ? 2 : 0);
            if (pat == pass + 1) return true;
        }
    }
};

// A step record in global memory: x = block a | block b << 16 (0xFFFF: none),
// y = flags | last << 31.
__device__ __forceinline__ uint2 encode_step(const StepRec& r) {
    const uint32_t a = r.ca < 0 ? 0xFFFFu : static_cast<uint32_t>(r.ca);
    const uint32_t b = r.cb < 0 ? 0xFFFFu : static_cast<uint32_t>(r.cb);
    return make_uint2(a | (b << 16), r.flags | (r.last << 31));
}

__device__ __forceinline__ StepRec decode_step(uint2 e) {
    StepRec r;
    const uint32_t a = e.x & 0xFFFFu, b = e.x >> 16;
    r.ca = a == 0xFFFFu ? -1 : static_cast<int32_t>(a);
    r.cb = b == 0xFFFFu ? -1 : static_cast<int32_t>(b);
    r.flags = e.y & 0xFFu;
    r.last = e.y >> 31;
    return r;
}

__device__ __forceinline__ bool tile_active(uint32_t flags, int t) { return (flags & (0x33u << (2 * t))) != 0u; }

// Bit o is set when offset o of key block j holds a real token.
template <int LM>
__device__ __forceinline__ uint64_t key_mask(int j, const FineParams& p) {
    if (j < 0 || j >= p.nblk) return 0ull;
    if (LM == kLoadTokens) {
        const int64_t left = p.N - 64ll * j;
        return left >= 64 ? ~0ull : ((1ull << left) - 1ull);
    }
    uint64_t m = ~0ull;
    const uint32_t q = div_magic(static_cast<uint32_t>(j), p.magic_cy);          // j / Cy
    if (static_cast<int>(static_cast<uint32_t>(j) - q * static_cast<uint32_t>(p.Cy)) == p.Cy - 1) m &= p.mask_y;
    const uint32_t ct = div_magic(q, p.magic_cx);                                  // j / (Cx*Cy)
    if (static_cast<int>(q - ct * static_cast<uint32_t>(p.Cx)) == p.Cx - 1) m &= p.mask_x;
    if (static_cast<int>(ct) == p.Ct - 1) m &= p.mask_t;
    return m;
}

// One 64-row x 64-channel box of block j (channels [d0, d0 + 64)) into dst.
// Blocks outside [0, nblk) are fetched from fully out-of-range coordinates,
// which the copy engine fills with zeros (and still counts in full).
template <int LM, int D>
__device__ __forceinline__ void load_block(const CUtensorMap* m, uint32_t dst, int j, int d0, uint32_t bar,
                                           const Item& it, const FineParams& p) {
    const bool valid = j >= 0 && j < p.nblk;
    if (LM == kLoadTiled) {
        const int32_t row = valid ? static_cast<int32_t>(it.bh * p.Npad + static_cast<int64_t>(j) * 64) : p.oob_row;
        tma_load_2d(dst, m, d0, row, bar);
    } else if (LM == kLoadCubes) {
        if (valid) {
            const uint32_t q = div_magic(static_cast<uint32_t>(j), p.magic_cy);
            const uint32_t ct = div_magic(q, p.magic_cx);
            const int cy = j - static_cast<int>(q) * p.Cy;
            const int cx = static_cast<int>(q) - static_cast<int>(ct) * p.Cx;
            tma_load_5d(dst, m, it.h * D + d0, 4 * cy, 4 * cx, 4 * static_cast<int>(ct), it.b, bar);
        } else {
            tma_load_5d(dst, m, d0, 0, 0, 0, p.B, bar);
        }
    } else {
        if (valid) tma_load_3d(dst, m, it.h * D + d0, 64 * j, it.b, bar);
        else tma_load_3d(dst, m, d0, 0, p.B, bar);
    }
}

constexpr float kSumLimit = 18446744073709551616.0f;   // 2^64: bound on any probability

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

// Scores of columns whose bit in `vm` is clear become -inf (32 columns).
__device__ __forceinline__ void mask32(uint32_t (&s)[32], uint32_t vm) {
    if (vm == 0xFFFFFFFFu) return;
    const uint32_t ninf = __float_as_uint(-INFINITY);
#pragma unroll
    for (int j = 0; j < 32; ++j)
        if (!((vm >> j) & 1u)) s[j] = ninf;
}

__device__ __forceinline__ float max32(const uint32_t (&s)[32]) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = __uint_as_float(s[i]);
#pragma unroll
    for (int j = 8; j < 32; ++j) m[j & 7] = fmaxf(m[j & 7], __uint_as_float(s[j]));
    return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])), fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

// Probabilities 2^(s*c - m) of 32 masked scores: 16 bf16 pairs into pk, their
// float32 sum returned.
__device__ __forceinline__ float probs32(const uint32_t (&s)[32], float c, float m, uint32_t* pk) {
    const uint64_t c2 = f32x2(c, c), nm2 = f32x2(-m, -m);
    uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const uint64_t t = fma_f32x2(f32x2(__uint_as_float(s[2 * j]), __uint_as_float(s[2 * j + 1])), c2, nm2);
        float t0, t1;
        f32x2_split(t, t0, t1);
        const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
        acc[j & 1] = add_f32x2(acc[j & 1], f32x2(p0, p1));
        pk[j] = pack_bf16x2(p0, p1);
    }
    float lo, hi;
    f32x2_split(add_f32x2(acc[0], acc[1]), lo, hi);
    return lo + hi;
}

// Masked maximum (times c) of this warp's 64 score columns at tS.  Warp-collective.
__device__ __forceinline__ float half_max(uint32_t tS, uint64_t vm, float c) {
    float m = -INFINITY;
#pragma unroll 1
    for (int ch = 0; ch < 2; ++ch) {
        uint32_t sc[32];
        tmem_ld32_wait(tS + 32u * ch, sc);
        mask32(sc, static_cast<uint32_t>(vm >> (32 * ch)));
        m = fmaxf(m, max32(sc));
    }
    return m * c;
}

// Probabilities of this warp's 64 score columns at tS, as 32 bf16 pairs in
// pk; their float32 sum returned.  Warp-collective.
__device__ __forceinline__ float half_probs(uint32_t tS, uint64_t vm, float c, float m, uint32_t (&pk)[32]) {
    float sum = 0.f;
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
        uint32_t sc[32];
        tmem_ld32_wait(tS + 32u * ch, sc);
        mask32(sc, static_cast<uint32_t>(vm >> (32 * ch)));
        sum += probs32(sc, c, m, pk + 16 * ch);
    }
    return sum;
}

// Shared-memory descriptor for a 1024-byte-aligned 128-byte-swizzled operand:
// the fixed fields once, the start address per use.
__device__ __forceinline__ uint64_t desc_at(uint64_t fixed, uint32_t saddr) {
    return fixed | static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
}

// Position of a ring (or stage) counter: slot and phase parity.
struct RingPos {
    int slot;
    uint32_t phase;
    template <int N>
    __device__ __forceinline__ void advance() {
        if (++slot == N) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

template <int D, int LM, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
fine_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const FineParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base = (raw_u32 + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_u32);

    // a re-run launched behind fine_tile_kernel does nothing unless that kernel's probabilities overflowed
    if (p.run_if != nullptr && *p.run_if == 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto bar = [&](int i) -> uint32_t { return base + kOffBar + 8u * static_cast<uint32_t>(i); };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    StepRec* ring = reinterpret_cast<StepRec*>(smem + kOffRec);
    const BoundedWait bw{abort_flag, p.status, p.limit_ns};
    const bool dense = p.idx == nullptr;

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
            mbar_init(bar(kBarPFull + t), 8);   // one arrival per softmax warp of the tile
            mbar_init(bar(kBarPVDone + t), 1);
        }
        for (int r = 0; r < kRing; ++r) {
            mbar_init(bar(kBarRecFull + r), 1);
            mbar_init(bar(kBarRecEmpty + r), kRecConsumers);
        }
        for (int i = 0; i < 8; ++i) mbar_init(bar(kBarPair + i), 2);
        mbar_init(bar(kBarDrain), 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(base + kOffMisc, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    constexpr uint32_t kBytesQ = 4u * 64u * D * 2u;   // one Q group load
    constexpr uint32_t kBytesKV = 2u * 64u * D * 2u;  // one step's two K (or V) blocks

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ walk + TMA producer
        if (lane == 0) {
            uint32_t q_issued = 0, k_issued[kKStages] = {}, v_issued[kVStages] = {};
            RingPos kp{0, 0}, vp{0, 0}, rp{0, 0};
            int n_item = 0;
            bool ok = true;
            for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x, ++n_item) {
                const Item item = decode_item(it, p);
                auto load_pair = [&](const CUtensorMap* m, uint32_t dst, int ja, int jb, uint32_t b) {
                    load_block<LM, D>(m, dst, ja, 0, b, item, p);
                    load_block<LM, D>(m, dst + 8192, jb, 0, b, item, p);
                    if (D == 128) {
                        load_block<LM, D>(m, dst + 16384, ja, 64, b, item, p);
                        load_block<LM, D>(m, dst + 24576, jb, 64, b, item, p);
                    }
                };
                if (!(ok = bw.wait(bar(kBarQEmpty), (n_item & 1) ^ 1))) break;
                mbar_arrive_expect_tx(bar(kBarQFull), kBytesQ);
                ++q_issued;
                for (int t = 0; t < 2; ++t)
                    load_pair(&tm_q, base + kOffQ + t * kQTileBytes, item.blk[2 * t], item.blk[2 * t + 1],
                              bar(kBarQFull));
                GroupWalk w = make_walk(item, p);
                for (int s = 0;; ++s) {
                    StepRec r;
                    if (dense) {
                        r = dense_step(s, item.present, p.nblk);
                    } else {
                        if (p.steps != nullptr) {
                            // a record is trusted no further than the buffer's bounds: blocks
                            // past the grid read as the empty cube, and the last slot ends the item
                            r = decode_step(__ldg(p.steps + it * p.steps_stride + s));
                            r.ca = min(r.ca, p.C);
                            r.cb = min(r.cb, p.C);
                            if (s + 1 >= p.steps_stride) r.last = 1u;
                        } else if (!w.next(r)) {
                            // an item none of whose slots holds a query block (an order
                            // entry out of range) still publishes one empty step
                            r = StepRec{-1, -1, 0u, 1u};
                        }
                        if (!(ok = bw.wait(bar(kBarRecEmpty + rp.slot), rp.phase ^ 1u))) break;
                        ring[rp.slot] = r;
                        mbar_arrive(bar(kBarRecFull + rp.slot));   // release: the record is visible
                        rp.advance<kRing>();
                    }
                    if (!(ok = bw.wait(bar(kBarKEmpty + kp.slot), kp.phase ^ 1u))) break;
                    mbar_arrive_expect_tx(bar(kBarKFull + kp.slot), kBytesKV);
                    ++k_issued[kp.slot];
                    load_pair(&tm_k, base + kOffK + kp.slot * kKVBytes, r.ca, r.cb, bar(kBarKFull + kp.slot));
                    kp.advance<kKStages>();
                    if (!(ok = bw.wait(bar(kBarVEmpty + vp.slot), vp.phase ^ 1u))) break;
                    mbar_arrive_expect_tx(bar(kBarVFull + vp.slot), kBytesKV);
                    ++v_issued[vp.slot];
                    load_pair(&tm_v, base + kOffV + vp.slot * kKVBytes, r.ca, r.cb, bar(kBarVFull + vp.slot));
                    vp.advance<kVStages>();
                    if (r.last) break;
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
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);   // Q (K-major) x K^T (K-major)
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);     // P (TMEM, K-major) x V (MN-major)
            const uint64_t fix_k = smem_desc_sw128(0, 16u, 1024u);         // K-major, 8-row groups 1 KB apart
            const uint64_t fix_v = smem_desc_sw128(0, 16384u, 1024u);      // MN-major, d halves 16 KB apart
            RingPos kp{0, 0}, vp{0, 0}, rp{0, 0};
            uint32_t n_p[2] = {0, 0};   // per-tile PV steps issued
            int n_item = 0;
            bool ok = true, issued_any = false;
            bool acc[2] = {false, false};   // O of the tile already holds this item's sum
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
                issued_any = true;
            };
            // PV of tile t for the step whose V sits in stage v (waits for its P and V)
            auto issue_pv = [&](int t, RingPos v) -> bool {
                if (!bw.wait(bar(kBarPFull + t), n_p[t] & 1u)) return false;
                if (!bw.wait(bar(kBarVFull + v.slot), v.phase)) return false;
                tc_fence_after();
                const uint32_t vb = base + kOffV + v.slot * kKVBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    // P of key half h sits in the first 32 columns of that half's scores
                    mma_bf16_ts(tmem + t * kTileCols + kColO, tmem + t * kTileCols + (kk >> 2) * 64u + (kk & 3) * 8u,
                                desc_at(fix_v, vb + kk * 2048u), idesc_o, (!acc[t] && kk == 0) ? 0u : 1u);
                acc[t] = true;
                mma_commit(bar(kBarPVDone + t));
                ++n_p[t];
                return true;
            };
            for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x, ++n_item) {
                const uint32_t present = dense ? decode_item(it, p).present : 0u;
                if (!(ok = bw.wait(bar(kBarQFull), n_item & 1))) break;
                acc[0] = acc[1] = false;
                bool pend_b = false;   // PV of tile B for the previous step still to issue
                bool have_prev = false;
                RingPos v_prev{0, 0};
                for (int s = 0;; ++s) {
                    StepRec r;
                    if (dense) {
                        r = dense_step(s, present, p.nblk);
                    } else {
                        if (!(ok = bw.wait(bar(kBarRecFull + rp.slot), rp.phase))) break;
                        r = ring[rp.slot];
                        mbar_arrive(bar(kBarRecEmpty + rp.slot));
                        rp.advance<kRing>();
                    }
                    if (!(ok = bw.wait(bar(kBarKFull + kp.slot), kp.phase))) break;
                    tc_fence_after();
                    const bool act_a = tile_active(r.flags, 0), act_b = tile_active(r.flags, 1);
                    if (act_a) issue_s(0, kp.slot);                               // S_A(i)
                    if (pend_b && !(ok = issue_pv(1, v_prev))) break;             // PV_B(i-1)
                    if (have_prev) mma_commit(bar(kBarVEmpty + v_prev.slot));
                    if (act_b) issue_s(1, kp.slot);                               // S_B(i)
                    mma_commit(bar(kBarKEmpty + kp.slot));
                    kp.advance<kKStages>();
                    if (act_a && !(ok = issue_pv(0, vp))) break;                  // PV_A(i)
                    pend_b = act_b;
                    have_prev = true;
                    v_prev = vp;
                    vp.advance<kVStages>();
                    if (r.last) break;
                }
                if (!ok) break;
                mma_commit(bar(kBarQEmpty));
                if (pend_b && !(ok = issue_pv(1, v_prev))) break;
                if (have_prev) mma_commit(bar(kBarVEmpty + v_prev.slot));
            }
            if (issued_any) {
                // all MMAs of this CTA complete before tensor memory is freed
                mma_commit(bar(kBarDrain));
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(bar(kBarDrain), 0) && globaltimer() - t0 < kDrainLimitNs) {
                }
            }
        }
    } else if (warp < kTmaWarp) {
        // ------------------------------------------------------------ softmax + epilogue
        // Warps 0..15.  Two warps share each TMEM lane quarter of a tile, one per
        // 64-column half of a step's 128 scores, so a tile's softmax runs as two
        // independent halves.  The pair agrees on each row's maximum (first scores,
        // overflow) and adds its row sums through a double-buffered shared slot
        // guarded by a two-arrival mbarrier (every wait bounded).
        const int sidx = warp;
        const int tile = sidx >> 3;              // 0: warps 0..7, 1: warps 8..15
        const int half = (sidx >> 2) & 1;        // which 64 of the step's 128 key columns
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int row = q * 32 + lane;           // query row of the tile, 0..127
        const int slot = 2 * tile + (q >> 1);    // query-block slot of the group
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t tS = tmem + tile * kTileCols + lane_addr + 64u * half;   // scores; P over its first 32 columns
        const uint32_t tO = tmem + tile * kTileCols + lane_addr + kColO + (D / 2) * half;   // this warp's channels
        const uint32_t bar_sfull = bar(kBarSFull + tile), bar_pfull = bar(kBarPFull + tile);
        const uint32_t bar_pvdone = bar(kBarPVDone + tile);
        const uint32_t bar_pair = bar(kBarPair + tile * 4 + q);
        float* xbuf = reinterpret_cast<float*>(smem + kOffXch);
        const float c = p.c_log2;
        uint32_t n = 0;    // steps this tile has taken part in (same count as the MMA issuer's)
        uint32_t xn = 0;   // exchanges of this pair
        RingPos rp{0, 0};
        bool ok = true;
        auto wait_all = [&](uint32_t b, uint32_t par) -> bool {
            const bool mine = bw.wait(b, par);
            return __all_sync(0xffffffffu, mine);
        };
        // Gives the partner warp this lane's value and returns the partner's for the same row.
        auto exchange = [&](float mine, float& other) -> bool {
            float* slot_base = xbuf + (((xn & 1u) * 2 + tile) * 4 + q) * 64;
            slot_base[half * 32 + lane] = mine;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_pair);   // release: the warp's 32 values are visible
            const bool got = wait_all(bar_pair, xn & 1u);
            ++xn;
            other = slot_base[(half ^ 1) * 32 + lane];
            return got;
        };
        for (int64_t it = blockIdx.x; ok && it < p.items; it += gridDim.x) {
            const Item item = decode_item(it, p);
            float m_run = -INFINITY, l_run = 0.f;   // m_run is the same in both warps of the pair
            uint32_t steps = 0;
            for (int s = 0;; ++s) {
                StepRec r;
                if (dense) {
                    r = dense_step(s, item.present, p.nblk);
                } else {
                    if (!(ok = wait_all(bar(kBarRecFull + rp.slot), rp.phase))) break;
                    r = ring[rp.slot];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(kBarRecEmpty + rp.slot));
                    rp.advance<kRing>();
                }
                if (tile_active(r.flags, tile)) {
                    // warp-uniform: this warp's rows belong to one query block
                    const uint64_t vm_a = ((r.flags >> slot) & 1u) ? key_mask<LM>(r.ca, p) : 0ull;
                    const uint64_t vm_b = ((r.flags >> (4 + slot)) & 1u) ? key_mask<LM>(r.cb, p) : 0ull;
                    const uint64_t vm = half ? vm_b : vm_a;
                    if (!(ok = wait_all(bar_sfull, n & 1u))) break;
                    tc_fence_after();
                    uint32_t pk[32];
                    if ((vm_a | vm_b) != 0ull) {   // the same in both warps of the pair
                        if (__any_sync(0xffffffffu, m_run == -INFINITY)) {
                            // the row's first scores: the maximum over both halves
                            const float mx = vm ? half_max(tS, vm, c) : -INFINITY;
                            float omx;
                            if (!(ok = exchange(mx, omx))) break;
                            if (m_run == -INFINITY) m_run = fmaxf(mx, omx);
                        }
                        float sum = 0.f;
                        if (vm) {
                            sum = half_probs(tS, vm, c, m_run, pk);
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) pk[j] = 0u;
                        }
                        float osum;
                        if (!(ok = exchange(sum, osum))) break;
                        // A probability above 2^64 in either half (the maximum fell far
                        // behind): both warps raise it to the step's maximum, rescale what
                        // they accumulated (each its half of O) and recompute.  The scores
                        // are intact, since no P of this step is stored yet.
                        if (__any_sync(0xffffffffu, !(sum <= kSumLimit) || !(osum <= kSumLimit))) {
                            const float mx = vm ? half_max(tS, vm, c) : -INFINITY;
                            float omx;
                            if (!(ok = exchange(mx, omx))) break;
                            const float m_new = fmaxf(m_run, fmaxf(mx, omx));
                            const float alpha = ex2_approx(m_run - m_new);
                            m_run = m_new;
                            l_run *= alpha;
                            // the tile's previous PV completed before these scores were committed
                            scale_tmem_f32(tO, D / 64, alpha);
                            if (vm) sum = half_probs(tS, vm, c, m_run, pk);
                        }
                        l_run += sum;
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) pk[j] = 0u;
                    }
                    tmem_st32(tS, pk);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_pfull);
                    ++n;
                    ++steps;
                }
                if (r.last) break;
            }
            if (!ok) break;
            if (steps == 0) continue;   // the tile holds no query block of this group (both warps)
            // ---------------- epilogue of this warp's rows and channels
            // PV(n-2) completed before S(n-1) was committed, so this parity cannot alias
            if (!(ok = wait_all(bar_pvdone, (n - 1) & 1u))) break;
            tc_fence_after();
            float ol;
            if (!(ok = exchange(l_run, ol))) break;
            const float l_tot = half ? (ol + l_run) : (l_run + ol);   // one order in both warps
            const int blk = item.blk[slot];
            const int o_ = row & 63;
            const int d0 = (D / 2) * half;
            const float inv_l = l_tot > 0.f ? 1.0f / l_tot : 0.f;
            if (!FUSED) {
                const bool store = blk >= 0;
                const int64_t grow = item.bh * p.Npad + static_cast<int64_t>(store ? blk : 0) * 64 + o_;
#pragma unroll 1
                for (int ch = 0; ch < D / 64; ++ch) {
                    uint32_t o[32];
                    tmem_ld32_wait(tO + 32u * ch, o);
                    if (store) {
                        uint32_t w16[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            w16[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * inv_l,
                                                 __uint_as_float(o[2 * j + 1]) * inv_l);
                        uint4* dst = reinterpret_cast<uint4*>(p.o + grow * D + d0 + 32 * ch);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            dst[v] = make_uint4(w16[4 * v], w16[4 * v + 1], w16[4 * v + 2], w16[4 * v + 3]);
                    }
                }
                if (store && half == 0 && p.lse != nullptr)
                    p.lse[grow] = l_tot > 0.f ? (m_run + log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
            } else {
                // token of this row, and the cube whose coarse output it merges
                int64_t tok = -1;
                int cube = 0;
                if (blk >= 0) {
                    if (LM == kLoadTokens) {
                        tok = 64ll * blk + o_;
                        if (tok >= p.N) {
                            tok = -1;
                        } else if (p.o_coarse != nullptr) {
                            const int64_t xy = static_cast<int64_t>(p.X) * p.Y;
                            const int tt = static_cast<int>(tok / xy);
                            const int rem = static_cast<int>(tok - tt * xy);
                            const int xx = rem / p.Y, yy = rem - (rem / p.Y) * p.Y;
                            cube = ((tt >> 2) * p.Cx + (xx >> 2)) * p.Cy + (yy >> 2);
                        }
                    } else {
                        const uint32_t qd = div_magic(static_cast<uint32_t>(blk), p.magic_cy);
                        const uint32_t ct = div_magic(qd, p.magic_cx);
                        const int cy = blk - static_cast<int>(qd) * p.Cy;
                        const int cx = static_cast<int>(qd) - static_cast<int>(ct) * p.Cx;
                        const int tt = 4 * static_cast<int>(ct) + (o_ >> 4);
                        const int xx = 4 * cx + ((o_ >> 2) & 3), yy = 4 * cy + (o_ & 3);
                        if (tt < p.T && xx < p.X && yy < p.Y)
                            tok = (static_cast<int64_t>(tt) * p.X + xx) * p.Y + yy;
                        cube = blk;
                    }
                }
                const bool store = tok >= 0;
                float gc = 0.f, gf = 1.f;
                const float* ocr = nullptr;
                const int64_t grow = (static_cast<int64_t>(item.b) * p.N + (store ? tok : 0)) * p.H + item.h;
                if (store) {
                    if (p.g_coarse) gc = __uint_as_float(static_cast<uint32_t>(__ldg(p.g_coarse + grow)) << 16);
                    if (p.g_fine) gf = __uint_as_float(static_cast<uint32_t>(__ldg(p.g_fine + grow)) << 16);
                    if (p.o_coarse) ocr = p.o_coarse + (item.bh * p.C + cube) * D;
                }
                const float sf = gf * inv_l;
#pragma unroll 1
                for (int ch = 0; ch < D / 64; ++ch) {
                    uint32_t o[32];
                    tmem_ld32_wait(tO + 32u * ch, o);
                    if (store) {
                        float v[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(o[j]) * sf;
                        if (ocr != nullptr) {
                            const float4* oc4 = reinterpret_cast<const float4*>(ocr + d0 + 32 * ch);
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const float4 cv = __ldg(oc4 + j);
                                v[4 * j] = fmaf(gc, cv.x, v[4 * j]);
                                v[4 * j + 1] = fmaf(gc, cv.y, v[4 * j + 1]);
                                v[4 * j + 2] = fmaf(gc, cv.z, v[4 * j + 2]);
                                v[4 * j + 3] = fmaf(gc, cv.w, v[4 * j + 3]);
                            }
                        }
                        uint32_t w16[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) w16[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                        uint4* dst = reinterpret_cast<uint4*>(p.o + grow * D + d0 + 32 * ch);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[v4] = make_uint4(w16[4 * v4], w16[4 * v4 + 1], w16[4 * v4 + 2], w16[4 * v4 + 3]);
                    }
                }
            }
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ====================================================================== one-tile kernel
// fine_tile_kernel: the fused fine stage with one 128-row tile per work item
// (two query blocks) and three score buffers in tensor memory, so that three
// steps of the same tile are in flight at once: while one group of softmax
// warps turns step i's scores into probabilities, the tensor core computes
// the scores of steps i+1 and i+2 into the other two buffers.  Two threads
// issue the MMAs, one the QK^T products (S) and one the PV products, because
// one thread issues an M128N128K16 MMA only every ~95 cycles, against ~68 for
// the tensor core to run it.
//
// Roles (640 threads): warps 0-11 are three softmax groups of four warps
// (group g owns score buffer g and takes the steps s with s % 3 == g; warp
// 4g + q reads TMEM lane quarter q); warp 12 loads the tile's Q and per step
// two K blocks through a 3-deep ring; warp 15 loads per step two V blocks
// through a 2-deep ring; warp 13 allocates tensor memory and issues S(s) into
// buffer s % 3 once PV(s - 3) has drained it; warp 14 issues PV(s) into the
// output accumulator once group s % 3 has stored P(s); warps 16-19 write the
// output (warp 16 + q: lane quarter q).
//
// Loads: a thread that issues TMA copies is held for roughly as long as the
// copies take to land (about 1,300 cycles for a step's 32 KB of K, measured
// with clock stamps), so one thread issuing K and V in turn paced the whole
// pipeline: V(s) waits for PV(s - 2), and K(s + 1) queued behind it.  K and V
// therefore have producers of their own, and the four 8 KB boxes of a load
// (two blocks x two 64-channel halves) are issued by four lanes at once.
//
// Tensor memory: buffers at columns 0, 128 and 256 (128 fp32 scores for a
// step's 128 keys; P, as bf16 pairs, over the first 64 columns), the output
// accumulator at 384.
//
// Softmax with a fixed maximum per row (Wan2.2 teardown, zharfai.com, section
// "Fixed-max softmax is a numerical contract"): the maximum of a row's first
// selected scores is kept for the whole item, so the three groups need no
// exchange per step; each keeps its own partial row sum and the epilogue adds
// the three.
//
// Epilogue: warps 16-19 merge and store the item's output while the three
// softmax groups go on to the next item, which they start as soon as their
// steps of this one are done; the first PV of the next item waits only until
// the epilogue warps have read O out of tensor memory.  The epilogue fetches
// its inputs (gates, the coarse outputs of the tile's query cubes) while the
// item's steps run.  Because the groups run one item ahead of the epilogue,
// the per-item maxima, row sums and their barriers come in two sets, used by
// even and odd items.  The epilogue waits for the
// item's last PV on a barrier committed once per item: a wait by parity on
// the last step's PV-done barrier would pass early whenever that buffer's
// previous PV were still pending (a parity wait returns at once when the
// barrier is one phase behind).  A group that has no step in an item (items
// of one or two steps) depends on nothing in it, so each group also waits,
// before item n, until the epilogue has read item n - 2's row sums (SetFree):
// no group runs more than one item ahead of the epilogue.
//
// Work items are claimed, not dealt: the Q/K producer takes the CTA's first
// item as blockIdx.x and every later one from a counter in the caller's
// memory (the second word of the overflow pair), then publishes each index in
// a four-slot shared-memory ring that every other role reads.  Items differ in
// length (the union of two selections: 16 to 32 steps at top-k 32), and a fixed
// deal of every 148th item left the longest CTA about 4% behind the mean at
// Wan 480p; claimed in order, items still run about 148 apart, so the K and V
// cubes that neighbouring query cubes share stay in L2.  The next index is
// claimed one item early, so its atomic's latency is hidden.
//
// A probability above 2^64 (a later score far above the first
// maximum) or a non-finite sum raises the overflow word, and the caller then
// runs fine_kernel, whose online maximum is rescaled per step, over the whole
// stage again: the teardown's guard that re-runs a tile with online rescaling.
constexpr int kTThreads = 640;
constexpr int kTVWarp = 15;
constexpr int kTEpiWarp = 16;                                     // warps 16-19: the epilogue
constexpr int kTTmaWarp = 12;
constexpr int kTSWarp = 13;
constexpr int kTPVWarp = 14;
constexpr int kTBufs = 3;
constexpr int kTKStages = 3;
constexpr int kTVStages = 2;
constexpr uint32_t kTOffQ = 0;                                   // one tile: 128 rows x 256 B
constexpr uint32_t kTOffK = kTOffQ + kQTileBytes;                // [kTKStages]
constexpr uint32_t kTOffV = kTOffK + kTKStages * kKVBytes;       // [kTVStages]
constexpr uint32_t kTOffM = kTOffV + kTVStages * kKVBytes;       // [2 items][128] each row's fixed maximum
constexpr uint32_t kTOffL = kTOffM + 2 * 128 * 4;                // [2 items][kTBufs][128] each group's row sums
constexpr uint32_t kTOffOC = kTOffL + 2 * kTBufs * 128 * 4;      // [4 epilogue warps][128] coarse outputs
constexpr int kTItemRing = 4;                                    // items published ahead of the last reader
constexpr uint32_t kTOffItem = kTOffOC + 4 * 128 * 4;            // [kTItemRing] int32 item indices
constexpr uint32_t kTOffBar = kTOffItem + kTItemRing * 4;
constexpr int kTBarQFull = 0;
constexpr int kTBarQEmpty = 1;
constexpr int kTBarKFull = 2;                                    // [kTKStages]
constexpr int kTBarKEmpty = kTBarKFull + kTKStages;
constexpr int kTBarVFull = kTBarKEmpty + kTKStages;             // [kTVStages]
constexpr int kTBarVEmpty = kTBarVFull + kTVStages;
constexpr int kTBarSFull = kTBarVEmpty + kTVStages;             // [kTBufs]
constexpr int kTBarPFull = kTBarSFull + kTBufs;                  // [kTBufs], four arrivals
constexpr int kTBarPVDone = kTBarPFull + kTBufs;                 // [kTBufs]
constexpr int kTBarMReady = kTBarPVDone + kTBufs;                // [2 items][2 query blocks], two arrivals
constexpr int kTBarEpi = kTBarMReady + 4;                        // [2 items], twelve arrivals
constexpr int kTBarOFree = kTBarEpi + 2;                         // four arrivals (the epilogue warps)
constexpr int kTBarODone = kTBarOFree + 1;                       // the item's last PV complete (one commit per item)
constexpr int kTBarSetFree = kTBarODone + 1;                     // [2 items], four arrivals: the set is read
constexpr int kTBarDrain = kTBarSetFree + 2;                     // [2 issuers]
constexpr int kTBarItemFull = kTBarDrain + 2;                    // [kTItemRing]
constexpr int kTBarItemEmpty = kTBarItemFull + kTItemRing;       // [kTItemRing], kTItemReaders arrivals
constexpr int kTNumBars = kTBarItemEmpty + kTItemRing;
// readers of each published item: the S and PV issuers, the V producer, the twelve softmax warps and
// the four epilogue warps
constexpr uint32_t kTItemReaders = 1 + 1 + 1 + 12 + 4;
constexpr uint32_t kTOffMisc = kTOffBar + kTNumBars * 8;         // tmem slot (4 B) + abort flag (4 B)
constexpr uint32_t kTSmemBytes = kTOffMisc + 16 + 1024;
constexpr uint32_t kTColO = 384;
static_assert(kTSmemBytes <= 232448, "shared memory over the 227 KB per-block limit");

// Step s of item it: computed (dense) or read from the precomputed list.
__device__ __forceinline__ StepRec tile_step(const FineParams& p, int64_t it, int s, uint32_t present) {
    if (p.idx == nullptr) return dense_step(s, present, p.nblk);
    StepRec r = decode_step(__ldg(p.steps + it * p.steps_stride + s));
    r.ca = min(r.ca, p.C);
    r.cb = min(r.cb, p.C);
    if (s + 1 >= p.steps_stride) r.last = 1u;
    return r;
}

template <int D, int LM>
__global__ void __launch_bounds__(kTThreads, 1)
fine_tile_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const FineParams p) {
    static_assert(LM == kLoadCubes || LM == kLoadTokens, "token-layout inputs only");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base = (raw_u32 + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_u32);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto bar = [&](int i) -> uint32_t { return base + kTOffBar + 8u * static_cast<uint32_t>(i); };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kTOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kTOffMisc + 4);
    float* m_row = reinterpret_cast<float*>(smem + kTOffM);
    float* l_part = reinterpret_cast<float*>(smem + kTOffL);
    float* oc_s = reinterpret_cast<float*>(smem + kTOffOC);
    const BoundedWait bw{abort_flag, p.status, p.limit_ns};

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bar(kTBarQFull), 1);
        mbar_init(bar(kTBarQEmpty), 1);
        for (int s = 0; s < kTKStages; ++s) {
            mbar_init(bar(kTBarKFull + s), 1);
            mbar_init(bar(kTBarKEmpty + s), 1);
        }
        for (int s = 0; s < kTVStages; ++s) {
            mbar_init(bar(kTBarVFull + s), 1);
            mbar_init(bar(kTBarVEmpty + s), 1);
        }
        for (int b = 0; b < kTBufs; ++b) {
            mbar_init(bar(kTBarSFull + b), 1);
            mbar_init(bar(kTBarPFull + b), 4);    // the four warps of group b
            mbar_init(bar(kTBarPVDone + b), 1);
        }
        for (int i = 0; i < 4; ++i) mbar_init(bar(kTBarMReady + i), 2);   // the two warps of a query block
        mbar_init(bar(kTBarEpi + 0), 12);
        mbar_init(bar(kTBarEpi + 1), 12);
        mbar_init(bar(kTBarOFree), 4);
        mbar_init(bar(kTBarODone), 1);
        mbar_init(bar(kTBarSetFree + 0), 4);
        mbar_init(bar(kTBarSetFree + 1), 4);
        mbar_init(bar(kTBarDrain + 0), 1);
        mbar_init(bar(kTBarDrain + 1), 1);
        for (int i = 0; i < kTItemRing; ++i) {
            mbar_init(bar(kTBarItemFull + i), 1);
            mbar_init(bar(kTBarItemEmpty + i), kTItemReaders);
        }
        fence_mbar_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == kTSWarp) {
        tmem_alloc(base + kTOffMisc, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    constexpr uint32_t kBytesQ = 2u * 64u * D * 2u;   // one tile's Q
    constexpr uint32_t kBytesKV = 2u * 64u * D * 2u;  // one step's two K (or V) blocks
    auto drain_wait = [&](uint32_t b, uint32_t par) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(b, par) && globaltimer() - t0 < kDrainLimitNs) {
        }
    };

    constexpr int kBoxes = D == 128 ? 4 : 2;
    constexpr unsigned kBoxMask = (1u << kBoxes) - 1u;
    volatile int32_t* item_ring = reinterpret_cast<volatile int32_t*>(smem + kTOffItem);
    // The n-th item of this CTA for the lanes of `mask` (lane 0 among them): every lane waits for it
    // and reads it, lane 0 then releases the slot.  -1: no item is left.
    auto take_item = [&](int n, unsigned mask, int64_t& it) -> bool {
        const int slot = n % kTItemRing;
        const uint32_t par = static_cast<uint32_t>(n / kTItemRing) & 1u;
        if (!__all_sync(mask, bw.wait(bar(kTBarItemFull + slot), par))) return false;
        it = item_ring[slot];
        __syncwarp(mask);
        if (lane == 0) mbar_arrive(bar(kTBarItemEmpty + slot));   // release: the index is read
        return true;
    };
    if (warp == kTTmaWarp) {
        // ------------------------------------------------------------ Q and K producer (lane i: box i)
        if (lane < kBoxes) {
            uint32_t q_issued = 0, k_issued[kTKStages] = {};
            RingPos kp{0, 0};
            bool ok = true;
            int64_t claimed = blockIdx.x;   // lane 0: the item this CTA takes next
            for (int n_item = 0; ok; ++n_item) {
                // publish the item (or -1 once none is left) and claim the one after it
                int32_t it32 = -1;
                if (lane == 0) {
                    const int slot = n_item % kTItemRing;
                    ok = bw.wait(bar(kTBarItemEmpty + slot), (static_cast<uint32_t>(n_item / kTItemRing) & 1u) ^ 1u);
                    if (ok) {
                        it32 = claimed < p.items ? static_cast<int32_t>(claimed) : -1;
                        item_ring[slot] = it32;
                        mbar_arrive(bar(kTBarItemFull + slot));   // release: the index is visible
                        if (it32 >= 0)
                            claimed = p.work != nullptr ? static_cast<int64_t>(gridDim.x) + atomicAdd(p.work, 1)
                                                        : claimed + gridDim.x;
                    }
                }
                ok = __shfl_sync(kBoxMask, ok ? 1 : 0, 0) != 0;
                it32 = __shfl_sync(kBoxMask, it32, 0);
                if (!ok || it32 < 0) break;
                const int64_t it = it32;
                const Item item = decode_item(it, p);
                auto load_pair = [&](const CUtensorMap* m, uint32_t dst, int ja, int jb, uint32_t b) {
                    __syncwarp(kBoxMask);   // lane 0's expect_tx first
                    load_block<LM, D>(m, dst + 8192u * lane, (lane & 1) ? jb : ja, 64 * (lane >> 1), b, item, p);
                };
                if (!(ok = __all_sync(kBoxMask, bw.wait(bar(kTBarQEmpty), (n_item & 1) ^ 1)))) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(kTBarQFull), kBytesQ);
                    ++q_issued;
                }
                load_pair(&tm_q, base + kTOffQ, item.blk[0], item.blk[1], bar(kTBarQFull));
                for (int s = 0;; ++s) {
                    const StepRec r = tile_step(p, it, s, item.present);
                    if (!(ok = __all_sync(kBoxMask, bw.wait(bar(kTBarKEmpty + kp.slot), kp.phase ^ 1u)))) break;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(bar(kTBarKFull + kp.slot), kBytesKV);
                        ++k_issued[kp.slot];
                    }
                    load_pair(&tm_k, base + kTOffK + kp.slot * kKVBytes, r.ca, r.cb, bar(kTBarKFull + kp.slot));
                    kp.advance<kTKStages>();
                    if (r.last) break;
                }
            }
            if (!ok && lane == 0) {
                // wait for this CTA's own copies still in flight before exiting
                if (q_issued) drain_wait(bar(kTBarQFull), (q_issued - 1u) & 1u);
                for (int s = 0; s < kTKStages; ++s)
                    if (k_issued[s]) drain_wait(bar(kTBarKFull + s), (k_issued[s] - 1u) & 1u);
            }
        }
    } else if (warp == kTSWarp) {
        // ------------------------------------------------------------ S = Q K^T issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);   // Q (K-major) x K^T (K-major)
            const uint64_t fix_k = smem_desc_sw128(0, 16u, 1024u);         // K-major, 8-row groups 1 KB apart
            RingPos kp{0, 0};
            uint32_t uses[kTBufs] = {0u, 0u, 0u};   // S issued into each buffer so far
            bool ok = true, issued_any = false;
            for (int n_item = 0; ok; ++n_item) {
                int64_t it;
                if (!(ok = take_item(n_item, 1u, it)) || it < 0) break;
                const uint32_t present = decode_item(it, p).present;
                if (!(ok = bw.wait(bar(kTBarQFull), n_item & 1))) break;
                for (int s = 0;; ++s) {
                    const StepRec r = tile_step(p, it, s, present);
                    const int b = s % kTBufs;
                    // the buffer's previous P must have been read by its PV
                    if (uses[b] > 0 && !(ok = bw.wait(bar(kTBarPVDone + b), (uses[b] - 1u) & 1u))) break;
                    if (!(ok = bw.wait(bar(kTBarKFull + kp.slot), kp.phase))) break;
                    tc_fence_after();
                    const uint32_t qa = base + kTOffQ, kb = base + kTOffK + kp.slot * kKVBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                        mma_bf16_ss(tmem + 128u * b, desc_at(fix_k, qa + off), desc_at(fix_k, kb + off), idesc_s,
                                    kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(kTBarSFull + b));
                    mma_commit(bar(kTBarKEmpty + kp.slot));
                    issued_any = true;
                    ++uses[b];
                    kp.advance<kTKStages>();
                    if (r.last) break;
                }
                if (!ok) break;
                mma_commit(bar(kTBarQEmpty));
            }
            if (issued_any) {
                mma_commit(bar(kTBarDrain + 0));
                drain_wait(bar(kTBarDrain + 0), 0u);
            }
        }
    } else if (warp == kTPVWarp) {
        // ------------------------------------------------------------ O += P V issuer
        if (lane == 0) {
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);     // P (TMEM, K-major) x V (MN-major)
            const uint64_t fix_v = smem_desc_sw128(0, 16384u, 1024u);      // MN-major, d halves 16 KB apart
            RingPos vp{0, 0};
            uint32_t waits[kTBufs] = {0u, 0u, 0u};   // P-full phases consumed per buffer
            bool ok = true, issued_any = false;
            for (int n_item = 0; ok; ++n_item) {
                int64_t it;
                if (!(ok = take_item(n_item, 1u, it)) || it < 0) break;
                const uint32_t present = decode_item(it, p).present;
                for (int s = 0;; ++s) {
                    const StepRec r = tile_step(p, it, s, present);
                    const int b = s % kTBufs;
                    // the item's first PV overwrites O: the previous item's epilogue must have read it
                    if (s == 0 && n_item > 0 && !(ok = bw.wait(bar(kTBarOFree), (n_item - 1) & 1))) break;
                    if (!(ok = bw.wait(bar(kTBarPFull + b), waits[b] & 1u))) break;
                    ++waits[b];
                    if (!(ok = bw.wait(bar(kTBarVFull + vp.slot), vp.phase))) break;
                    tc_fence_after();
                    const uint32_t vb = base + kTOffV + vp.slot * kKVBytes;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tmem + kTColO, tmem + 128u * b + 8u * kk, desc_at(fix_v, vb + kk * 2048u), idesc_o,
                                    (s > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(bar(kTBarPVDone + b));
                    mma_commit(bar(kTBarVEmpty + vp.slot));
                    issued_any = true;
                    vp.advance<kTVStages>();
                    if (r.last) {
                        mma_commit(bar(kTBarODone));   // O of the item is complete
                        break;
                    }
                }
                if (!ok) break;
            }
            if (issued_any) {
                mma_commit(bar(kTBarDrain + 1));
                drain_wait(bar(kTBarDrain + 1), 0u);
            }
        }
    } else if (warp == kTVWarp) {
        // ------------------------------------------------------------ V producer (lane i: box i)
        if (lane < kBoxes) {
            uint32_t v_issued[kTVStages] = {};
            RingPos vp{0, 0};
            bool ok = true;
            for (int n_item = 0; ok; ++n_item) {
                int64_t it;
                if (!(ok = take_item(n_item, kBoxMask, it)) || it < 0) break;
                const Item item = decode_item(it, p);
                for (int s = 0;; ++s) {
                    const StepRec r = tile_step(p, it, s, item.present);
                    if (!(ok = __all_sync(kBoxMask, bw.wait(bar(kTBarVEmpty + vp.slot), vp.phase ^ 1u)))) break;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(bar(kTBarVFull + vp.slot), kBytesKV);
                        ++v_issued[vp.slot];
                    }
                    __syncwarp(kBoxMask);
                    const uint32_t dst = base + kTOffV + vp.slot * kKVBytes;
                    load_block<LM, D>(&tm_v, dst + 8192u * lane, (lane & 1) ? r.cb : r.ca, 64 * (lane >> 1),
                                      bar(kTBarVFull + vp.slot), item, p);
                    vp.advance<kTVStages>();
                    if (r.last) break;
                }
            }
            if (!ok && lane == 0) {
                for (int s = 0; s < kTVStages; ++s)
                    if (v_issued[s]) drain_wait(bar(kTBarVFull + s), (v_issued[s] - 1u) & 1u);
            }
        }
    } else if (warp >= kTEpiWarp) {
        // ------------------------------------------------------------ epilogue warpgroup
        const int q = warp & 3;                  // TMEM lane quarter
        const int row = q * 32 + lane;           // query row of the tile, 0..127
        const int slot = q >> 1;                 // query block of the row
        const uint32_t tO = tmem + kTColO + (static_cast<uint32_t>(q * 32) << 16);
        float* oc_w = oc_s + (warp - kTEpiWarp) * 128;   // this warp's query cube's coarse output
        bool ok = true;
        auto wait_all = [&](uint32_t b, uint32_t par) -> bool {
            const bool mine = bw.wait(b, par);
            return __all_sync(0xffffffffu, mine);
        };
        // token of this row (-1: none) and, for the token layout, its cube
        auto row_token = [&](const Item& item, int& cube) -> int64_t {
            const int blk = item.blk[slot];
            const int o_ = row & 63;
            int64_t tok = -1;
            cube = 0;
            if (blk >= 0) {
                if (LM == kLoadTokens) {
                    tok = 64ll * blk + o_;
                    if (tok >= p.N) {
                        tok = -1;
                    } else if (p.o_coarse != nullptr) {
                        const int64_t xy = static_cast<int64_t>(p.X) * p.Y;
                        const int tt = static_cast<int>(tok / xy);
                        const int rem = static_cast<int>(tok - tt * xy);
                        const int xx = rem / p.Y, yy = rem - (rem / p.Y) * p.Y;
                        cube = ((tt >> 2) * p.Cx + (xx >> 2)) * p.Cy + (yy >> 2);
                    }
                } else {
                    const uint32_t qd = div_magic(static_cast<uint32_t>(blk), p.magic_cy);
                    const uint32_t ct = div_magic(qd, p.magic_cx);
                    const int cy = blk - static_cast<int>(qd) * p.Cy;
                    const int cx = static_cast<int>(qd) - static_cast<int>(ct) * p.Cx;
                    const int tt = 4 * static_cast<int>(ct) + (o_ >> 4);
                    const int xx = 4 * cx + ((o_ >> 2) & 3), yy = 4 * cy + (o_ & 3);
                    if (tt < p.T && xx < p.X && yy < p.Y) tok = (static_cast<int64_t>(tt) * p.X + xx) * p.Y + yy;
                    cube = blk;
                }
            }
            return tok;
        };
        for (int n_item = 0; ok; ++n_item) {
            int64_t it;
            if (!(ok = take_item(n_item, 0xffffffffu, it)) || it < 0) break;
            const Item item = decode_item(it, p);
            const int ip = n_item & 1;
            const uint32_t ipar = static_cast<uint32_t>(n_item >> 1) & 1u;
            const float* l_it = l_part + ip * (kTBufs * 128);
            // inputs fetched while the item's steps run: this row's gates and (cube layout) the
            // coarse output of the warp's query cube; and the next item's records, towards L1
            int cube;
            const int64_t tok = row_token(item, cube);
            const bool store = tok >= 0;
            const int64_t grow = (static_cast<int64_t>(item.b) * p.N + (store ? tok : 0)) * p.H + item.h;
            float gc = 0.f, gf = 1.f;
            if (store) {
                if (p.g_coarse) gc = __uint_as_float(static_cast<uint32_t>(__ldg(p.g_coarse + grow)) << 16);
                if (p.g_fine) gf = __uint_as_float(static_cast<uint32_t>(__ldg(p.g_fine + grow)) << 16);
            }
            const float* ocr = nullptr;
            if (p.o_coarse != nullptr) {
                if (LM == kLoadTokens) {
                    ocr = p.o_coarse + (item.bh * p.C + cube) * D;
                } else {
                    const int cb = item.blk[slot];
                    if (lane < D / 4) {
                        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (cb >= 0) v = __ldg(reinterpret_cast<const float4*>(p.o_coarse + (item.bh * p.C + cb) * D) + lane);
                        reinterpret_cast<float4*>(oc_w)[lane] = v;
                    }
                    __syncwarp();
                    ocr = oc_w;
                }
            }
            // the next item, when it is already published (a look at its slot, no wait)
            int64_t nxt = -1;
            {
                const int ns = (n_item + 1) % kTItemRing;
                if (mbar_try_wait(bar(kTBarItemFull + ns), static_cast<uint32_t>((n_item + 1) / kTItemRing) & 1u))
                    nxt = item_ring[ns];
            }
            if (nxt >= 0 && nxt < p.items && q == 0 && lane < 3) {
                if (lane < 2 && p.steps != nullptr && 128 * lane < 8 * p.steps_stride)
                    prefetch_l1(reinterpret_cast<const uint8_t*>(p.steps + nxt * p.steps_stride) + 128 * lane);
                if (lane == 2 && p.order != nullptr) {
                    const int64_t nbh = nxt / p.ngroups, pos = p.group * (nxt - nbh * p.ngroups);
                    if (pos < p.nblk) prefetch_l1(p.order + nbh * p.C + pos);
                }
            }
            // the item's output accumulator is complete and the three groups' row sums are in
            if (!(ok = wait_all(bar(kTBarODone), static_cast<uint32_t>(n_item) & 1u))) break;
            if (!(ok = wait_all(bar(kTBarEpi + ip), ipar))) break;
            tc_fence_after();
            const float l_tot = (l_it[row] + l_it[128 + row]) + l_it[256 + row];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kTBarSetFree + ip));   // this item's set may be reused
            const float inv_l = l_tot > 0.f ? 1.0f / l_tot : 0.f;
            const float sf = gf * inv_l;
            // 32-column chunk ch of O (in registers) -> gated merge -> bf16 row segment
            auto emit = [&](int ch, const uint32_t* o) {
                float v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(o[j]) * sf;
                if (ocr != nullptr) {
                    const float4* oc4 = reinterpret_cast<const float4*>(ocr + 32 * ch);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 cv = oc4[j];
                        v[4 * j] = fmaf(gc, cv.x, v[4 * j]);
                        v[4 * j + 1] = fmaf(gc, cv.y, v[4 * j + 1]);
                        v[4 * j + 2] = fmaf(gc, cv.z, v[4 * j + 2]);
                        v[4 * j + 3] = fmaf(gc, cv.w, v[4 * j + 3]);
                    }
                }
                uint32_t w16[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) w16[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                uint4* dst = reinterpret_cast<uint4*>(p.o + grow * D + 32 * ch);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4)
                    dst[v4] = make_uint4(w16[4 * v4], w16[4 * v4 + 1], w16[4 * v4 + 2], w16[4 * v4 + 3]);
            };
            // O in two halves of 64 columns (D = 128) or one (D = 64); O is released after the
            // last read, so the next item's first PV does not wait for the last stores
            uint32_t o[64];
            if constexpr (D == 128) {
                tmem_ld64_wait(tO, o);
                if (store) {
                    emit(0, o);
                    emit(1, o + 32);
                }
                tmem_ld64_wait(tO + 64u, o);
            } else {
                tmem_ld64_wait(tO, o);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kTBarOFree));   // O may be overwritten by the next item
            if (store) {
                emit(D / 32 - 2, o);
                emit(D / 32 - 1, o + 32);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax groups
        const int g = warp >> 2;                 // group: score buffer g, steps s with s % 3 == g
        const int q = warp & 3;                  // TMEM lane quarter
        const int row = q * 32 + lane;           // query row of the tile, 0..127
        const int slot = q >> 1;                 // query block of the row
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t tS = tmem + 128u * g + lane_addr;
        const float c = p.c_log2;
        uint32_t n_s = 0;                         // S-full phases consumed (buffer g)
        bool ok = true;
        auto wait_all = [&](uint32_t b, uint32_t par) -> bool {
            const bool mine = bw.wait(b, par);
            return __all_sync(0xffffffffu, mine);
        };
        for (int n_item = 0; ok; ++n_item) {
            int64_t it;
            if (!(ok = take_item(n_item, 0xffffffffu, it)) || it < 0) break;
            const Item item = decode_item(it, p);
            // The groups go on to the next item while the epilogue warps write this one, so the
            // maxima, the row sums and their barriers alternate between two sets by item parity.
            const int ip = n_item & 1;
            const uint32_t ipar = static_cast<uint32_t>(n_item >> 1) & 1u;
            float* m_it = m_row + ip * 128;
            float* l_it = l_part + ip * (kTBufs * 128);
            const uint32_t mready = bar(kTBarMReady + 2 * ip + slot);
            // The set was last used by item n - 2: its row sums must have been read.  A group with no
            // step in an item depends on nothing else, so without this wait it could run two items
            // ahead and arrive on a barrier phase that belongs to the earlier item.
            if (n_item >= 2 && !(ok = wait_all(bar(kTBarSetFree + ip), static_cast<uint32_t>((n_item - 2) >> 1) & 1u)))
                break;
            float m = 0.f, l = 0.f;
            bool have_m = false;
            int sfirst = -1;     // first step that selects this row's query block (the same in every warp)
            for (int s = 0;; ++s) {
                const StepRec r = tile_step(p, it, s, item.present);
                const bool sel_a = ((r.flags >> slot) & 1u) != 0u, sel_b = ((r.flags >> (4 + slot)) & 1u) != 0u;
                if (sfirst < 0 && (sel_a || sel_b)) sfirst = s;
                const int b = s % kTBufs;
                if (b == g) {
                    if (!(ok = wait_all(bar(kTBarSFull + g), n_s & 1u))) break;
                    ++n_s;
                    tc_fence_after();
                    if (sel_a || sel_b) {
                        // warp-uniform: this warp's rows belong to one query block
                        const uint64_t vm_a = sel_a ? key_mask<LM>(r.ca, p) : 0ull;
                        const uint64_t vm_b = sel_b ? key_mask<LM>(r.cb, p) : 0ull;
                        if (s == sfirst) {
                            // the row's first selected scores fix its maximum for the item
                            float mx = -INFINITY;
#pragma unroll 1
                            for (int ch = 0; ch < 4; ++ch) {
                                const uint64_t vm = ch < 2 ? vm_a : vm_b;
                                const uint32_t w = static_cast<uint32_t>(vm >> (32 * (ch & 1)));
                                if (LM == kLoadCubes && w == 0u) continue;   // warp-uniform: no key counts
                                uint32_t sc[32];
                                tmem_ld32_wait(tS + 32u * ch, sc);
                                mask32(sc, w);
                                mx = fmaxf(mx, max32(sc));
                            }
                            m = mx == -INFINITY ? 0.f : mx * c;
                            m_it[row] = m;
                            have_m = true;
                            __syncwarp();
                            if (lane == 0) mbar_arrive(mready);   // release: the maximum is visible
                        } else if (!have_m) {
                            if (!(ok = wait_all(mready, ipar))) break;
                            m = m_it[row];
                            have_m = true;
                        }
                        float sum = 0.f;
#pragma unroll 1
                        for (int ch = 0; ch < 4; ++ch) {
                            const uint64_t vm = ch < 2 ? vm_a : vm_b;
                            const uint32_t w = static_cast<uint32_t>(vm >> (32 * (ch & 1)));
                            uint32_t pk[16];
                            if (LM == kLoadCubes && w == 0u) {
                                // warp-uniform: the chunk's 32 keys are outside this row's selection (a key
                                // cube only the other query cube of the tile selected): P = 0, no exponentials.
                                // (Dense blocks are selected by every row: the dense kernel keeps no such test.)
#pragma unroll
                                for (int j = 0; j < 16; ++j) pk[j] = 0u;
                            } else {
                                uint32_t sc[32];
                                tmem_ld32_wait(tS + 32u * ch, sc);
                                mask32(sc, w);
                                sum += probs32(sc, c, m, pk);
                            }
                            // P of keys 32ch.. over columns 16ch..: scores there were already read (or,
                            // for a skipped chunk 0, are not needed)
                            tmem_st16(tS + 16u * ch, pk);
                        }
                        if (!(sum <= kSumLimit) && p.overflow != nullptr) *p.overflow = 1;
                        l += sum;
                    } else {
                        // neither key block is selected by this row's query block: P = 0
                        uint32_t z[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) z[j] = 0u;
                        tmem_st32(tS, z);
                        tmem_st32(tS + 32u, z);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(kTBarPFull + g));
                }
                if (r.last) break;
            }
            if (!ok) break;
            // one arrival per item and query block on its max-ready barrier: when no step selects
            // the block, group 0's two warps of the block make it
            if (sfirst < 0 && g == 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(mready);
            }
            // hand the row sums to the epilogue warps and go on
            l_it[g * 128 + row] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kTBarEpi + ip));   // release: the sums are visible
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kTSWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Steps of one work item by the serial three-pass walk (TileWalk), written by
// one thread: the general case, which also visits repeated entries of a list
// as often as they appear.
__device__ void schedule_serial(const Item& item, const FineParams& p, uint2* out) {
    TileWalk tw;
    tw.w0 = make_walk(item, p);
    tw.w = tw.w0;
    tw.pass = 0;
    int blk = -1;
    uint32_t fl = 0;
    bool more = tw.next_entry(blk, fl);
    if (!more) {   // no query block in the group (order entries out of range): one empty step
        out[0] = encode_step(StepRec{-1, -1, 0u, 1u});
        return;
    }
    for (int s = 0; more; ++s) {
        StepRec r;
        r.ca = blk;
        r.flags = fl;
        more = tw.next_entry(blk, fl);
        r.cb = -1;
        if (more) {
            r.cb = blk;
            r.flags |= fl << 4;
            more = tw.next_entry(blk, fl);
        }
        r.last = more ? 0u : 1u;
        out[s] = encode_step(r);
    }
}

// Entries of a nibble word (cube 8w + n in nibble n, bit j set when query
// slot j selected it), one bit per nibble: selected by slot 0 or 1 (tile A),
// by slot 2 or 3 (tile B).
__device__ __forceinline__ uint32_t nib_tile_a(uint32_t v) { return (v | (v >> 1)) & 0x11111111u; }
__device__ __forceinline__ uint32_t nib_tile_b(uint32_t v) { return ((v >> 2) | (v >> 3)) & 0x11111111u; }

// Steps of every work item of a sparse selection, precomputed so the fine
// kernel's producer only reads them: the union of the group's four lists in
// three classes (key cubes only tile A's query blocks selected, only tile B's,
// both tiles'), ascending within a class, paired two per step.
//
// One warp per item.  The warp marks each list entry as a bit in a nibble per
// cube (cubes 0..C, C standing for every out-of-range entry) in shared memory,
// then scans the nibbles in cube order twice: once to count each class, once
// to place each cube at its class's offset plus its rank, with warp prefix
// sums over packed per-lane counts.  A list that holds a cube twice (never the
// case for a top-k selection) sends the item to the serial walk.
constexpr int kScheduleWarps = 4;

__host__ __device__ __forceinline__ int schedule_words(int C) { return (C + 8) >> 3; }

__global__ void __launch_bounds__(kScheduleWarps * 32) schedule_kernel(const FineParams p, uint2* __restrict__ steps) {
    extern __shared__ uint32_t sched_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = schedule_words(p.C), E = p.group * p.k;
    uint32_t* nib = sched_smem + static_cast<int64_t>(warp) * (W + E);
    uint32_t* ent = nib + W;
    const int64_t it = static_cast<int64_t>(blockIdx.x) * kScheduleWarps + warp;
    if (it >= p.items) return;   // warp-uniform
    for (int i = lane; i < W; i += 32) nib[i] = 0u;
    __syncwarp();
    const Item item = decode_item(it, p);
    uint2* out = steps + it * p.steps_stride;
    if (item.present == 0u) {   // no query block in the group: one empty step
        if (lane == 0) out[0] = encode_step(StepRec{-1, -1, 0u, 1u});
        return;
    }
    bool dup = false;
    for (int e = lane; e < E; e += 32) {
        const int j = e / p.k, i = e - j * p.k;
        if (!((item.present >> j) & 1u)) continue;
        int x = __ldg(p.idx + (item.bh * p.C + item.blk[j]) * static_cast<int64_t>(p.k) + i);
        if (x < 0 || x >= p.C) x = p.C;
        const uint32_t bit = 1u << (j + 4 * (x & 7));
        dup |= (atomicOr(nib + (x >> 3), bit) & bit) != 0u;
    }
    __syncwarp();
    if (__any_sync(0xFFFFFFFFu, dup)) {
        if (lane == 0) schedule_serial(item, p, out);
        return;
    }
    // class totals
    uint32_t t1 = 0, t2 = 0, t3 = 0;
    for (int w0 = 0; w0 < W; w0 += 32) {
        const uint32_t v = w0 + lane < W ? nib[w0 + lane] : 0u;
        const uint32_t a = nib_tile_a(v), b = nib_tile_b(v);
        t1 += __popc(a & ~b);
        t2 += __popc(b & ~a);
        t3 += __popc(a & b);
    }
    t1 = __reduce_add_sync(0xFFFFFFFFu, t1);
    t2 = __reduce_add_sync(0xFFFFFFFFu, t2);
    t3 = __reduce_add_sync(0xFFFFFFFFu, t3);
    // placement: class base + cubes of the class in earlier words
    uint32_t base[3] = {0u, t1, t1 + t2};
    for (int w0 = 0; w0 < W; w0 += 32) {
        const int wi = w0 + lane;
        const uint32_t v = wi < W ? nib[wi] : 0u;
        const uint32_t a = nib_tile_a(v), b = nib_tile_b(v);
        // per-lane counts of the three classes in 10-bit fields (at most 8 each)
        const uint32_t mine = __popc(a & ~b) | (__popc(b & ~a) << 10) | (__popc(a & b) << 20);
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - mine;
        uint32_t pa = base[0] + (excl & 1023u), pb = base[1] + ((excl >> 10) & 1023u), pab = base[2] + (excl >> 20);
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const uint32_t f = (v >> (4 * n)) & 15u;
            if (f == 0u) continue;
            const bool in_a = (f & 3u) != 0u, in_b = (f & 12u) != 0u;
            const uint32_t at = in_a ? (in_b ? pab++ : pa++) : pb++;
            ent[at] = static_cast<uint32_t>(8 * wi + n) | (f << 16);
        }
        const uint32_t tot = __shfl_sync(0xFFFFFFFFu, incl, 31);
        base[0] += tot & 1023u;
        base[1] += (tot >> 10) & 1023u;
        base[2] += tot >> 20;
    }
    __syncwarp();
    const int U = static_cast<int>(t1 + t2 + t3);
    const int nsteps = (U + 1) >> 1;
    for (int st = lane; st < nsteps; st += 32) {
        const uint32_t ea = ent[2 * st];
        const bool has_b = 2 * st + 1 < U;
        const uint32_t eb = has_b ? ent[2 * st + 1] : 0u;
        StepRec r;
        r.ca = static_cast<int32_t>(ea & 0xFFFFu);
        r.cb = has_b ? static_cast<int32_t>(eb & 0xFFFFu) : -1;
        r.flags = (ea >> 16) | (has_b ? (eb >> 16) << 4 : 0u);
        r.last = st == nsteps - 1 ? 1u : 0u;
        out[st] = encode_step(r);
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

// bf16 tensor map with a 64-channel (128-byte, swizzled) innermost box edge.
bool encode_map(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                const cuuint32_t* box) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void*>(ptr), dims,
              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tiled [rows, D]: box 64 channels x 64 rows.
bool encode_tiled(CUtensorMap* m, const void* ptr, const Dims& d) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d.D), static_cast<cuuint64_t>(d.rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d.D) * 2u};
    const cuuint32_t box[2] = {64u, 64u};
    return encode_map(m, ptr, 2, dims, strides, box);
}

// Projection layout [B, N, H, D] seen as (H*D channels, Y, X, T, B): box
// 64 channels x 4 x 4 x 4 tokens = one cube in cube-major offset order.
bool encode_cubes(CUtensorMap* m, const void* ptr, const Dims& d) {
    const cuuint64_t hd = static_cast<cuuint64_t>(d.H) * d.D;
    const cuuint64_t dims[5] = {hd, static_cast<cuuint64_t>(d.Y), static_cast<cuuint64_t>(d.X),
                                static_cast<cuuint64_t>(d.T), static_cast<cuuint64_t>(d.B)};
    const cuuint64_t row = hd * 2u;
    const cuuint64_t strides[4] = {row, row * d.Y, row * d.Y * d.X, row * static_cast<cuuint64_t>(d.N)};
    const cuuint32_t box[5] = {64u, 4u, 4u, 4u, 1u};
    return encode_map(m, ptr, 5, dims, strides, box);
}

// Projection layout [B, N, H, D] seen as (H*D channels, N, B): box
// 64 channels x 64 consecutive tokens.
bool encode_tokens(CUtensorMap* m, const void* ptr, const Dims& d) {
    const cuuint64_t hd = static_cast<cuuint64_t>(d.H) * d.D;
    const cuuint64_t dims[3] = {hd, static_cast<cuuint64_t>(d.N), static_cast<cuuint64_t>(d.B)};
    const cuuint64_t strides[2] = {hd * 2u, hd * 2u * static_cast<cuuint64_t>(d.N)};
    const cuuint32_t box[3] = {64u, 64u, 1u};
    return encode_map(m, ptr, 3, dims, strides, box);
}

template <int D, int LM, bool FUSED>
cudaError_t launch_instance(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FineParams& p, int grid, cudaStream_t s) {
    static int done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!(dev >= 0 && dev < 64 && done[dev])) {
        cudaError_t e = cudaFuncSetAttribute(fine_kernel<D, LM, FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemBytes));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) done[dev] = 1;
    }
    fine_kernel<D, LM, FUSED><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

template <int D, int LM>
cudaError_t launch_tile_instance(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                 const FineParams& p, int grid, cudaStream_t s) {
    static int done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!(dev >= 0 && dev < 64 && done[dev])) {
        cudaError_t e = cudaFuncSetAttribute(fine_tile_kernel<D, LM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kTSmemBytes));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) done[dev] = 1;
    }
    fine_tile_kernel<D, LM><<<grid, kTThreads, kTSmemBytes, s>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

uint64_t magic48(uint32_t d) { return ((uint64_t{1} << 48) / d) + 1; }

// Real offsets o = (t%4)*16 + (x%4)*4 + y%4 of a cube whose extent along one
// axis is n (< 4 only in the last cube layer of that axis).
uint64_t axis_mask(int axis, int n) {
    uint64_t m = 0;
    for (int o = 0; o < 64; ++o) {
        const int e = axis == 0 ? (o >> 4) : axis == 1 ? ((o >> 2) & 3) : (o & 3);
        if (e < n) m |= 1ull << o;
    }
    return m;
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

namespace {

FineParams make_params(const Dims& d, const FineArgs& a, int group) {
    const int mode = a.mode;
    FineParams p{};
    p.idx = a.idx;
    p.order = a.order;
    p.steps = reinterpret_cast<const uint2*>(a.steps);
    p.o = a.out;
    p.lse = a.lse;
    p.o_coarse = a.o_coarse;
    p.g_coarse = a.g_coarse;
    p.g_fine = a.g_fine;
    p.B = d.B;
    p.H = d.H;
    p.nblk = mode == kFineTokensFused ? static_cast<int>((d.N + 63) / 64) : d.C;
    p.k = a.idx ? a.k_sel : p.nblk;
    p.steps_stride = schedule_stride(p.k);
    p.C = d.C;
    p.Ct = d.Ct;
    p.Cx = d.Cx;
    p.Cy = d.Cy;
    p.T = d.T;
    p.X = d.X;
    p.Y = d.Y;
    p.N = d.N;
    p.group = group;
    p.ngroups = (p.nblk + group - 1) / group;
    p.magic_cxcy = magic48(static_cast<uint32_t>(d.Cx * d.Cy));
    p.magic_cy = magic48(static_cast<uint32_t>(d.Cy));
    p.magic_cx = magic48(static_cast<uint32_t>(d.Cx));
    p.mask_t = axis_mask(0, d.T - 4 * (d.Ct - 1));
    p.mask_x = axis_mask(1, d.X - 4 * (d.Cx - 1));
    p.mask_y = axis_mask(2, d.Y - 4 * (d.Cy - 1));
    p.Npad = d.Npad;
    p.items = static_cast<int64_t>(d.B) * d.H * p.ngroups;
    p.oob_row = static_cast<int32_t>(d.rows);
    p.c_log2 = a.scale * 1.4426950408889634f;
    p.status = status_word();
    p.limit_ns = kWaitLimitNs;
    return p;
}

}  // namespace

size_t schedule_bytes(const Dims& d, int k) {
    const int64_t items = static_cast<int64_t>(d.B) * d.H * ((d.C + kTileGroup - 1) / kTileGroup);
    return static_cast<size_t>(items) * static_cast<size_t>(schedule_stride(k)) * sizeof(uint2);
}

namespace {
size_t schedule_smem(const Dims& d, int k) {
    return static_cast<size_t>(kScheduleWarps) * (static_cast<size_t>(schedule_words(d.C)) + kTileGroup * k) * 4u;
}
}  // namespace

bool schedule_supported(const Dims& d, int k) {
    return d.C <= kScheduleMaxC && k >= 1 && k <= d.C && schedule_smem(d, k) <= 48u * 1024u;
}

cudaError_t launch_schedule(const Dims& d, const int32_t* idx, int k, const int32_t* order, void* steps,
                            cudaStream_t s) {
    if (!schedule_supported(d, k)) return cudaErrorInvalidValue;
    FineArgs a{};
    a.mode = kFineCubesFused;
    a.idx = idx;
    a.k_sel = k;
    a.order = order;
    const FineParams p = make_params(d, a, kTileGroup);
    if (p.items > 0x7FFFFFFFll) return cudaErrorInvalidValue;   // decode_item's 32-bit arithmetic
    const int64_t blocks = (p.items + kScheduleWarps - 1) / kScheduleWarps;
    if (blocks == 0) return cudaSuccess;
    schedule_kernel<<<static_cast<unsigned>(blocks), kScheduleWarps * 32, schedule_smem(d, k), s>>>(
        p, static_cast<uint2*>(steps));
    return cudaGetLastError();
}

cudaError_t launch_fine(const Dims& d, const FineArgs& a, cudaStream_t s, const char** why) {
    CUtensorMap tq, tk, tv;
    bool enc = false;
    const int mode = a.mode;
    if (mode == kFineTiled) {
        enc = encode_tiled(&tq, a.q, d) && encode_tiled(&tk, a.k, d) && encode_tiled(&tv, a.v, d);
    } else if (mode == kFineCubesFused) {
        enc = encode_cubes(&tq, a.q, d) && encode_cubes(&tk, a.k, d) && encode_cubes(&tv, a.v, d);
    } else if (mode == kFineTokensFused) {
        enc = encode_tokens(&tq, a.q, d) && encode_tokens(&tk, a.k, d) && encode_tokens(&tv, a.v, d);
    } else {
        if (why) *why = "unknown fine-stage mode";
        return cudaErrorInvalidValue;
    }
    if (!enc) {
        if (why) *why = "cuTensorMapEncodeTiled failed for a Q/K/V tensor";
        return cudaErrorInvalidValue;
    }
    // sparse selections with precomputed steps and dense attention on the token layout run on the
    // one-tile kernel (shorter items, no four-list union, three steps in flight).  For dense attention
    // it takes about 15% fewer cycles than fine_kernel, whose two tiles share each K/V step, and about
    // 6% less time at the lower clock its power draw leaves (Wan 480p, each kernel in its own run).
    const bool tile = (mode == kFineCubesFused && a.steps != nullptr) || mode == kFineTokensFused;
    if (tile) {
        // the one-tile kernel, then fine_kernel over the whole stage only if its fixed maxima overflowed
        int* ovf = a.overflow;   // the caller's word: calls on other streams never share it
        if (!ovf) {
            if (why) *why = "the fixed-maximum kernel needs an overflow word";
            return cudaErrorInvalidValue;
        }
        FineParams pt = make_params(d, a, kTileGroup);
        if (pt.items > 0x7FFFFFFFll) {   // decode_item's 32-bit arithmetic
            if (why) *why = "too many work items";
            return cudaErrorInvalidValue;
        }
        if (!pt.status) {
            if (why) *why = "watchdog word unavailable";
            return cudaErrorInvalidValue;
        }
        pt.overflow = ovf;
        pt.work = ovf + 1;   // the item counter beside the overflow flag
        cudaError_t e = cudaMemsetAsync(ovf, 0, 2 * sizeof(int), s);
        if (e != cudaSuccess) return e;
        const int gt = static_cast<int>(pt.items < sm_count() ? pt.items : sm_count());
        if (gt > 0) {
            if (mode == kFineTokensFused)
                e = d.D == 128 ? launch_tile_instance<128, kLoadTokens>(tq, tk, tv, pt, gt, s)
                               : launch_tile_instance<64, kLoadTokens>(tq, tk, tv, pt, gt, s);
            else
                e = d.D == 128 ? launch_tile_instance<128, kLoadCubes>(tq, tk, tv, pt, gt, s)
                               : launch_tile_instance<64, kLoadCubes>(tq, tk, tv, pt, gt, s);
            if (e != cudaSuccess) return e;
        }
        FineArgs ar = a;
        ar.steps = nullptr;   // the re-run walks the selection itself
        FineParams pr = make_params(d, ar, 4);
        pr.run_if = ovf;
        const int gr = static_cast<int>(pr.items < sm_count() ? pr.items : sm_count());
        if (gr <= 0) return cudaSuccess;
        if (mode == kFineTokensFused)
            return d.D == 128 ? launch_instance<128, kLoadTokens, true>(tq, tk, tv, pr, gr, s)
                              : launch_instance<64, kLoadTokens, true>(tq, tk, tv, pr, gr, s);
        return d.D == 128 ? launch_instance<128, kLoadCubes, true>(tq, tk, tv, pr, gr, s)
                          : launch_instance<64, kLoadCubes, true>(tq, tk, tv, pr, gr, s);
    }
    FineParams p = make_params(d, a, 4);
    if (p.items > 0x7FFFFFFFll) {   // decode_item's 32-bit arithmetic
        if (why) *why = "too many work items";
        return cudaErrorInvalidValue;
    }
    if (!p.status) {
        if (why) *why = "watchdog word unavailable";
        return cudaErrorInvalidValue;
    }
    const int grid = static_cast<int>(p.items < sm_count() ? p.items : sm_count());
    if (d.D == 128) {
        if (mode == kFineTiled) return launch_instance<128, kLoadTiled, false>(tq, tk, tv, p, grid, s);
        if (mode == kFineCubesFused) return launch_instance<128, kLoadCubes, true>(tq, tk, tv, p, grid, s);
        return launch_instance<128, kLoadTokens, true>(tq, tk, tv, p, grid, s);
    }
    if (mode == kFineTiled) return launch_instance<64, kLoadTiled, false>(tq, tk, tv, p, grid, s);
    if (mode == kFineCubesFused) return launch_instance<64, kLoadCubes, true>(tq, tk, tv, p, grid, s);
    return launch_instance<64, kLoadTokens, true>(tq, tk, tv, p, grid, s);
}

cudaError_t launch_wait_probe(uint64_t limit_ns, cudaStream_t s) {
    int* st = status_word();
    if (!st) return cudaErrorInvalidValue;
    wait_probe_kernel<<<1, 32, 0, s>>>(st, limit_ns);
    return cudaGetLastError();
}

}  // namespace vsa
