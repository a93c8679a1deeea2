// Coarse stage and cube selection (Wan2.2 teardown, zharfai.com, section
// "Video sparse attention selects cubes", part 1: cheap block-level attention
// over the mean-pooled cubes that ranks the candidate key cubes, of which
// each query cube keeps the top-k).
//
// The coarse scores decide the selection, so they are computed in float32 on
// the CUDA cores (a deterministic sequential sum over the channels), not on
// the bf16/tf32 tensor paths whose rounding would reorder near-equal cubes.
#include <cfloat>

#include "vsa_internal.h"

namespace vsa {
namespace {

constexpr int kBK = 16;     // reduction slice
constexpr int kThreads = 256;
constexpr int kSTI = 128;   // score tile rows (query cubes)
constexpr int kSTJ = 64;    // score tile columns (key cubes)
constexpr int kSRI = 8;     // rows per thread
constexpr int kSRJ = 4;     // columns per thread
static_assert((kSTI / kSRI) * (kSTJ / kSRJ) == kThreads, "one output block per thread");

// scores[bh][i][j] = scale * sum_d qbar[bh][i][d] * kbar[bh][j][d]
// A 128x64 output tile per block; thread (ty, tx) owns rows 8ty..8ty+7 and
// columns 4tx..4tx+3 (32 accumulators, 12 operands read from shared memory
// per 32 fma); the next 16-channel slice is loaded into registers while the
// current one is multiplied.  Each output is one sequential float32 fma chain
// over the channels, so the tiling does not change a single bit of the result.
__global__ void __launch_bounds__(kThreads) coarse_scores_kernel(int C, int D, const float* __restrict__ qbar,
                                                                 const float* __restrict__ kbar, float scale,
                                                                 float* __restrict__ scores) {
    __shared__ __align__(16) float As[kBK][kSTI + 4];
    __shared__ __align__(16) float Bs[kBK][kSTJ + 4];
    const int bh = blockIdx.z;
    const int i0 = blockIdx.y * kSTI, j0 = blockIdx.x * kSTJ;
    constexpr int NTX = kSTJ / kSRJ;
    const int tx = threadIdx.x % NTX, ty = threadIdx.x / NTX;
    const float* Q = qbar + static_cast<int64_t>(bh) * C * D;
    const float* K = kbar + static_cast<int64_t>(bh) * C * D;
    float acc[kSRI][kSRJ] = {};
    // the tile's rows x 16 channels of each operand: this thread's share, loaded one slice ahead
    constexpr int kLA = kSTI * kBK / kThreads, kLB = kSTJ * kBK / kThreads;
    float ra[kLA], rb[kLB];
    auto load_slice = [&](int d0) {
#pragma unroll
        for (int e = 0; e < kLA; ++e) {
            const int idx = threadIdx.x + e * kThreads;
            const int gi = i0 + idx / kBK;
            ra[e] = gi < C ? __ldg(Q + static_cast<int64_t>(gi) * D + d0 + idx % kBK) : 0.f;
        }
#pragma unroll
        for (int e = 0; e < kLB; ++e) {
            const int idx = threadIdx.x + e * kThreads;
            const int gj = j0 + idx / kBK;
            rb[e] = gj < C ? __ldg(K + static_cast<int64_t>(gj) * D + d0 + idx % kBK) : 0.f;
        }
    };
    load_slice(0);
    for (int d0 = 0; d0 < D; d0 += kBK) {
        // stored channel-major; the next slice's loads are in flight while this one is multiplied
#pragma unroll
        for (int e = 0; e < kLA; ++e) {
            const int idx = threadIdx.x + e * kThreads;
            As[idx % kBK][idx / kBK] = ra[e];
        }
#pragma unroll
        for (int e = 0; e < kLB; ++e) {
            const int idx = threadIdx.x + e * kThreads;
            Bs[idx % kBK][idx / kBK] = rb[e];
        }
        __syncthreads();
        if (d0 + kBK < D) load_slice(d0 + kBK);
#pragma unroll
        for (int kk = 0; kk < kBK; ++kk) {
            float av[kSRI], bv[kSRJ];
#pragma unroll
            for (int q4 = 0; q4 < kSRI / 4; ++q4) {
                const float4 a = *reinterpret_cast<const float4*>(&As[kk][kSRI * ty + 4 * q4]);
                av[4 * q4] = a.x;
                av[4 * q4 + 1] = a.y;
                av[4 * q4 + 2] = a.z;
                av[4 * q4 + 3] = a.w;
            }
            const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][kSRJ * tx]);
            bv[0] = b.x;
            bv[1] = b.y;
            bv[2] = b.z;
            bv[3] = b.w;
#pragma unroll
            for (int r = 0; r < kSRI; ++r)
#pragma unroll
                for (int c = 0; c < kSRJ; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
        }
        __syncthreads();
    }
    float* S = scores + static_cast<int64_t>(bh) * C * C;
#pragma unroll
    for (int r = 0; r < kSRI; ++r) {
        const int gi = i0 + kSRI * ty + r;
        if (gi >= C) continue;
#pragma unroll
        for (int c = 0; c < kSRJ; ++c) {
            const int gj = j0 + kSRJ * tx + c;
            if (gj < C) S[static_cast<int64_t>(gi) * C + gj] = scale * acc[r][c];
        }
    }
}

// o_coarse[bh][i] = sum_j softmax(scores[bh][i][:])_j * vbar[bh][j]
// One pass over each score row (online maximum): a block owns kPvRows query
// rows and walks the keys in slices of 16.  Half a warp holds a row's 16
// scores of the slice: it takes their maximum by shuffles, raises the row's
// running maximum m, and writes p = exp(s - m) to shared memory together with
// the factor exp(m_old - m) by which the row's accumulators are rescaled; each
// lane keeps a partial denominator, summed over the half warp at the end.
// Thread (ty, tx) owns RPT rows and 4 output channels.  The next slice's
// scores and V rows are loaded into registers while this slice accumulates.
constexpr int kPvRows = 32;

// n consecutive floats of shared memory (16-byte aligned for n % 4 == 0, else 8-byte) into registers
template <int n>
__device__ __forceinline__ void read_rows(const float* src, float* dst) {
    if constexpr (n % 4 == 0) {
#pragma unroll
        for (int i = 0; i < n / 4; ++i) {
            const float4 a = reinterpret_cast<const float4*>(src)[i];
            dst[4 * i] = a.x;
            dst[4 * i + 1] = a.y;
            dst[4 * i + 2] = a.z;
            dst[4 * i + 3] = a.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float2 a = reinterpret_cast<const float2*>(src)[i];
            dst[2 * i] = a.x;
            dst[2 * i + 1] = a.y;
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads) coarse_pv_kernel(int C, const float* __restrict__ scores,
                                                             const float* __restrict__ vbar,
                                                             float* __restrict__ o_coarse) {
    constexpr int TX = D / 4;                     // threads across the channels
    constexpr int RPT = kPvRows * TX / kThreads;  // rows per thread
    constexpr int SPT = kPvRows * kBK / kThreads; // scores per thread per slice
    constexpr int VPT = kBK * D / 4 / kThreads;   // V float4 per thread per slice
    static_assert(RPT % 2 == 0 && SPT >= 1 && VPT >= 1, "tile shape");
    __shared__ __align__(16) float Ps[kBK][kPvRows + 4];
    __shared__ __align__(16) float Vs[kBK][D];
    __shared__ __align__(16) float alpha_s[kPvRows];
    __shared__ float row_inv[kPvRows];
    const int bh = blockIdx.y;
    const int i0 = blockIdx.x * kPvRows;
    const float* S = scores + static_cast<int64_t>(bh) * C * C;
    const float* V = vbar + static_cast<int64_t>(bh) * C * D;
    const int cc = threadIdx.x % kBK, rbase = threadIdx.x / kBK;   // score role: key cc of rows rbase + 16e
    const int tx = threadIdx.x % TX, ty = threadIdx.x / TX;        // accumulate role
    float m[SPT], l[SPT], s_next[SPT];
    float4 v_next[VPT];
    auto load_slice = [&](int j0) {
        const int gj = j0 + cc;
#pragma unroll
        for (int e = 0; e < SPT; ++e) {
            const int gi = i0 + rbase + e * (kThreads / kBK);
            s_next[e] = gi >= C ? 0.f : gj < C ? __ldg(S + static_cast<int64_t>(gi) * C + gj) : -FLT_MAX;
        }
#pragma unroll
        for (int e = 0; e < VPT; ++e) {
            const int idx = threadIdx.x + e * kThreads;
            const int kk = idx / (D / 4), c4 = idx % (D / 4);
            v_next[e] = j0 + kk < C ? __ldg(reinterpret_cast<const float4*>(V + static_cast<int64_t>(j0 + kk) * D) + c4)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
#pragma unroll
    for (int e = 0; e < SPT; ++e) {
        m[e] = -FLT_MAX;
        l[e] = 0.f;
    }
    float acc[RPT][4] = {};
    load_slice(0);
    for (int j0 = 0; j0 < C; j0 += kBK) {
#pragma unroll
        for (int e = 0; e < SPT; ++e) {
            const int r = rbase + e * (kThreads / kBK);
            float mx = s_next[e];
#pragma unroll
            for (int off = kBK / 2; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float mn = fmaxf(m[e], mx);
            const float a = expf(m[e] - mn);
            const float pv = expf(s_next[e] - mn);
            m[e] = mn;
            l[e] = l[e] * a + pv;
            Ps[cc][r] = pv;
            if (cc == 0) alpha_s[r] = a;
        }
#pragma unroll
        for (int e = 0; e < VPT; ++e) {
            const int idx = threadIdx.x + e * kThreads;
            *reinterpret_cast<float4*>(&Vs[idx / (D / 4)][4 * (idx % (D / 4))]) = v_next[e];
        }
        __syncthreads();
        if (j0 + kBK < C) load_slice(j0 + kBK);
        {
            float av[RPT];
            read_rows<RPT>(&alpha_s[RPT * ty], av);
#pragma unroll
            for (int r = 0; r < RPT; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] *= av[r];
        }
#pragma unroll
        for (int kk = 0; kk < kBK; ++kk) {
            float pr[RPT];
            read_rows<RPT>(&Ps[kk][RPT * ty], pr);
            const float4 b = *reinterpret_cast<const float4*>(&Vs[kk][4 * tx]);
            const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int r = 0; r < RPT; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(pr[r], bv[c], acc[r][c]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int e = 0; e < SPT; ++e) {
        float t = l[e];
#pragma unroll
        for (int off = kBK / 2; off; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
        if (cc == 0) row_inv[rbase + e * (kThreads / kBK)] = t > 0.f ? 1.0f / t : 0.f;
    }
    __syncthreads();
    float* O = o_coarse + static_cast<int64_t>(bh) * C * D;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int li = RPT * ty + r, gi = i0 + li;
        if (gi >= C) continue;
        const float inv = row_inv[li];
        *reinterpret_cast<float4*>(O + static_cast<int64_t>(gi) * D + 4 * tx) =
            make_float4(acc[r][0] * inv, acc[r][1] * inv, acc[r][2] * inv, acc[r][3] * inv);
    }
}

// Order-preserving map float -> uint32 (larger float, larger key); -0 is
// folded onto +0 so that equal scores compare equal.
__device__ __forceinline__ uint32_t order_key(float f) {
    if (f == 0.0f) f = 0.0f;
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void top3_insert(uint64_t (&t)[3], uint64_t v) {
    if (v > t[2]) {
        if (v > t[1]) {
            t[2] = t[1];
            if (v > t[0]) {
                t[1] = t[0];
                t[0] = v;
            } else {
                t[1] = v;
            }
        } else {
            t[2] = v;
        }
    }
}

// Work-order key of query cube i from its three best key cubes t[0..2]
// (score order, lower index first; 0xFFFF for an absent entry): the three
// cube indices, then i, so sorting the keys groups cubes with similar
// selections and is a permutation.
__device__ __forceinline__ uint64_t group_signature(const uint64_t (&t)[3], uint32_t i) {
    uint64_t sg = static_cast<uint64_t>(i);
#pragma unroll
    for (int e = 0; e < 3; ++e) {
        const uint64_t c = t[e] ? (0xFFFFFFFFu - static_cast<uint32_t>(t[e] & 0xFFFFFFFFu)) : 0xFFFFu;
        sg |= (c & 0xFFFFu) << (48 - 16 * e);
    }
    return sg;
}

// One warp per (b, h, query cube) row.  The k-th largest key T is built bit
// by bit from the top (largest T with at least k keys >= T); the row is then
// scanned in index order, keeping every key > T and the lowest-index keys
// equal to T until k are kept, so the output is ascending by construction.
__global__ void __launch_bounds__(kThreads) topk_kernel(int64_t rows, int C, int k, const float* __restrict__ scores,
                                                        int32_t* __restrict__ idx) {
    extern __shared__ uint32_t keys_all[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* keys = keys_all + static_cast<int64_t>(warp) * C;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + warp; row < rows; row += warps) {
        const float* s = scores + row * C;
        for (int j = lane; j < C; j += 32) keys[j] = order_key(__ldcs(s + j));
        __syncwarp();
        uint32_t T = 0u;
        for (int bit = 31; bit >= 0; --bit) {
            const uint32_t cand = T | (1u << bit);
            int cnt = 0;
            for (int j0 = 0; j0 < C; j0 += 32) {
                const int j = j0 + lane;
                cnt += __popc(__ballot_sync(0xffffffffu, j < C && keys[j] >= cand));
            }
            if (cnt >= k) T = cand;
        }
        int gt = 0;
        for (int j0 = 0; j0 < C; j0 += 32) {
            const int j = j0 + lane;
            gt += __popc(__ballot_sync(0xffffffffu, j < C && keys[j] > T));
        }
        const int need_eq = k - gt;
        int out = 0, eq_seen = 0;
        int32_t* dst = idx + row * k;
        for (int j0 = 0; j0 < C && out < k; j0 += 32) {
            const int j = j0 + lane;
            const uint32_t key = j < C ? keys[j] : 0u;
            const bool is_gt = j < C && key > T;
            const bool is_eq = j < C && key == T;
            const uint32_t eq_mask = __ballot_sync(0xffffffffu, is_eq);
            const int eq_rank = eq_seen + __popc(eq_mask & lt_mask);
            const bool take = is_gt || (is_eq && eq_rank < need_eq);
            const uint32_t take_mask = __ballot_sync(0xffffffffu, take);
            if (take) dst[out + __popc(take_mask & lt_mask)] = j;
            out += __popc(take_mask);
            eq_seen += __popc(eq_mask);
        }
        __syncwarp();
    }
}

// Top-k with the row held in registers (KPL keys per lane, key j in lane
// j % 32, slot j / 32), for C <= 32 * KPL.  The k-th largest key T is built
// bit by bit from the top with warp sums (redux) of per-lane counts; the row
// is then scanned in index order exactly as topk_kernel does, so both give
// the same selection.  When `sig` is non-null the row's work-order key is
// written as well: its four smallest selected cubes (12 bits each, C <= 4096)
// above the cube's own index, so that sorting the keys puts query cubes whose
// selections start alike next to each other (the fine stage's tiles are pairs
// of consecutive cubes, and a tile's steps are the union of its two
// selections).
template <int KPL>
__global__ void __launch_bounds__(kThreads) topk_reg_kernel(int64_t rows, int C, int k, const float* __restrict__ scores,
                                                            int32_t* __restrict__ idx, uint64_t* __restrict__ sig) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + warp; row < rows; row += warps) {
        const float* s = scores + row * C;
        uint32_t key[KPL];
#pragma unroll
        for (int i = 0; i < KPL; ++i) {
            const int j = lane + 32 * i;
            key[i] = j < C ? order_key(__ldcs(s + j)) : 0u;   // 0 ranks below every real score
        }
        // T lies between a lower bound and the largest key, so it shares their
        // leading bits: only the bits below the highest differing one are searched.
        // Lower bound: the smallest lane maximum when k <= 32 (at least 32 keys
        // reach it), else the smallest key.
        uint32_t lane_max = 0u, lane_min = 0xFFFFFFFFu;
#pragma unroll
        for (int i = 0; i < KPL; ++i) {
            lane_max = max(lane_max, key[i]);
            if (lane + 32 * i < C) lane_min = min(lane_min, key[i]);
        }
        const uint32_t hi = __reduce_max_sync(0xffffffffu, lane_max);
        const uint32_t lo = k <= 32 ? __reduce_min_sync(0xffffffffu, lane_max) : __reduce_min_sync(0xffffffffu, lane_min);
        const uint32_t diff = hi ^ lo;
        const int top = diff ? 31 - __clz(diff) : -1;          // highest differing bit
        uint32_t T = top < 0 ? hi : (top >= 31 ? 0u : (hi & ~((2u << top) - 1u)));
#pragma unroll 1
        for (int bit = top; bit >= 0; --bit) {
            const uint32_t cand = T | (1u << bit);
            uint32_t cnt = 0;
#pragma unroll
            for (int i = 0; i < KPL; ++i) cnt += key[i] >= cand ? 1u : 0u;
            if (static_cast<int>(__reduce_add_sync(0xffffffffu, cnt)) >= k) T = cand;
        }
        uint32_t gt = 0;
#pragma unroll
        for (int i = 0; i < KPL; ++i) gt += key[i] > T ? 1u : 0u;
        const int need_eq = k - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
        int out = 0, eq_seen = 0;
        int32_t* dst = idx + row * k;
        uint64_t lex = 0ull;   // the row's four smallest selected cubes, 12 bits each from bit 52 down
        int nlex = 0;
#pragma unroll
        for (int i = 0; i < KPL; ++i) {
            const int j = lane + 32 * i;
            const bool valid = j < C;
            const bool is_gt = valid && key[i] > T;
            const bool is_eq = valid && key[i] == T;
            const uint32_t eq_mask = __ballot_sync(0xffffffffu, is_eq);
            const int eq_rank = eq_seen + __popc(eq_mask & lt_mask);
            const bool take = is_gt || (is_eq && eq_rank < need_eq);
            const uint32_t take_mask = __ballot_sync(0xffffffffu, take);
            if (take) dst[out + __popc(take_mask & lt_mask)] = j;
            out += __popc(take_mask);
            eq_seen += __popc(eq_mask);
            // warp-uniform: the selection is written in ascending order, so its first entries are these
            for (uint32_t mk = take_mask; nlex < 4 && mk != 0u; mk &= mk - 1u, ++nlex)
                lex |= static_cast<uint64_t>(32 * i + __ffs(mk) - 1) << (52 - 12 * nlex);
        }
        if (sig != nullptr && lane == 0) sig[row] = lex | static_cast<uint64_t>(row % C);
    }
}

// Work-order for the fine stage: per (b, h), the query cubes sorted by the
// indices of their three highest-scoring key cubes (ties to the lower index),
// so that consecutive cubes, which the fine kernel processes as a group of
// four sharing one key/value stream, tend to select the same key cubes.  The
// result is a permutation of [0, C); it changes the schedule only, never the
// output.  One block per (b, h); C <= kGroupMaxC.
constexpr int kGroupThreads = 512;

// Sorts keys[0, C) ascending (keys[C, cpow2) are padding set here) with a
// bitonic network over the block and writes each key's low 16 bits (the
// query cube) to order[0, C).
__device__ __forceinline__ void sort_and_write(uint64_t* keys, int C, int cpow2, int32_t* __restrict__ order) {
    for (int i = C + threadIdx.x; i < cpow2; i += kGroupThreads) keys[i] = ~0ull;
    __syncthreads();
    for (int k2 = 2; k2 <= cpow2; k2 <<= 1) {
        for (int j = k2 >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < cpow2; i += kGroupThreads) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const uint64_t a = keys[i], b = keys[ixj];
                    const bool up = (i & k2) == 0;
                    if ((a > b) == up) {
                        keys[i] = b;
                        keys[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int r = threadIdx.x; r < C; r += kGroupThreads) order[r] = static_cast<int32_t>(keys[r] & 0xFFFFu);
}

__global__ void __launch_bounds__(kGroupThreads) group_kernel(int C, int cpow2, const float* __restrict__ scores,
                                                              int32_t* __restrict__ order) {
    __shared__ uint64_t keys[kGroupMaxC];
    const int bh = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float* S = scores + static_cast<int64_t>(bh) * C * C;
    for (int i = warp; i < C; i += kGroupThreads / 32) {
        const float* row = S + static_cast<int64_t>(i) * C;
        uint64_t t[3] = {0ull, 0ull, 0ull};
        for (int j = lane; j < C; j += 32)   // key: score order, then lower index first
            top3_insert(t, (static_cast<uint64_t>(order_key(row[j])) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(j)));
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            uint64_t o[3];
#pragma unroll
            for (int e = 0; e < 3; ++e) o[e] = __shfl_xor_sync(0xffffffffu, t[e], off);
#pragma unroll
            for (int e = 0; e < 3; ++e) top3_insert(t, o[e]);
        }
        if (lane == 0) keys[i] = group_signature(t, static_cast<uint32_t>(i));
    }
    sort_and_write(keys, C, cpow2, order + static_cast<int64_t>(bh) * C);
}

// The work order from signatures already computed (topk_reg_kernel): one
// block per (b, h) sorts them.
__global__ void __launch_bounds__(kGroupThreads) group_sort_kernel(int C, int cpow2, const uint64_t* __restrict__ sig,
                                                                   int32_t* __restrict__ order) {
    __shared__ uint64_t keys[kGroupMaxC];
    const int bh = blockIdx.x;
    for (int i = threadIdx.x; i < C; i += kGroupThreads) keys[i] = sig[static_cast<int64_t>(bh) * C + i];
    sort_and_write(keys, C, cpow2, order + static_cast<int64_t>(bh) * C);
}

}  // namespace

cudaError_t launch_group(const Dims& d, const float* scores, int32_t* order, cudaStream_t s) {
    if (d.C > kGroupMaxC) return cudaErrorInvalidValue;
    int cpow2 = 1;
    while (cpow2 < d.C) cpow2 <<= 1;
    group_kernel<<<d.B * d.H, kGroupThreads, 0, s>>>(d.C, cpow2, scores, order);
    return cudaGetLastError();
}

cudaError_t launch_coarse_scores(const Dims& d, const float* qbar, const float* kbar, float scale, float* scores,
                                 cudaStream_t s) {
    const int bh = d.B * d.H;
    const dim3 grid((d.C + kSTJ - 1) / kSTJ, (d.C + kSTI - 1) / kSTI, bh);
    coarse_scores_kernel<<<grid, kThreads, 0, s>>>(d.C, d.D, qbar, kbar, scale, scores);
    return cudaGetLastError();
}

cudaError_t launch_coarse_pv(const Dims& d, const float* scores, const float* vbar, float* o_coarse, cudaStream_t s) {
    const int bh = d.B * d.H;
    const int pv_blocks = (d.C + kPvRows - 1) / kPvRows;
    if (d.D == 128) coarse_pv_kernel<128><<<dim3(pv_blocks, bh), kThreads, 0, s>>>(d.C, scores, vbar, o_coarse);
    else coarse_pv_kernel<64><<<dim3(pv_blocks, bh), kThreads, 0, s>>>(d.C, scores, vbar, o_coarse);
    return cudaGetLastError();
}

cudaError_t launch_coarse(const Dims& d, const float* qbar, const float* kbar, const float* vbar, float scale,
                          float* scores, float* o_coarse, cudaStream_t s) {
    const cudaError_t e = launch_coarse_scores(d, qbar, kbar, scale, scores, s);
    if (e != cudaSuccess) return e;
    return launch_coarse_pv(d, scores, vbar, o_coarse, s);
}

// Largest C the selection kernel keeps in shared memory (one row per warp).
constexpr int kTopkMaxC = 49152;

int topk_warps_per_block(int C) {
    int w = 8;
    while (w > 1 && static_cast<int64_t>(w) * C * 4 > 200 * 1024) w >>= 1;
    return w;
}

namespace {

// Register-resident selection for C <= 2048 (a warp holds the row, KPL keys per lane).
template <int KPL>
cudaError_t launch_topk_reg(int64_t rows, int C, int k, const float* scores, int32_t* idx, uint64_t* sig,
                            cudaStream_t s) {
    const int64_t blocks_needed = (rows + kThreads / 32 - 1) / (kThreads / 32);
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
    topk_reg_kernel<KPL><<<grid, kThreads, 0, s>>>(rows, C, k, scores, idx, sig);
    return cudaGetLastError();
}

cudaError_t topk_reg_dispatch(const Dims& d, const float* scores, int k, int32_t* idx, uint64_t* sig,
                              cudaStream_t s) {
    const int64_t rows = static_cast<int64_t>(d.B) * d.H * d.C;
    const int kpl = (d.C + 31) / 32;
    if (kpl <= 4) return launch_topk_reg<4>(rows, d.C, k, scores, idx, sig, s);
    if (kpl <= 8) return launch_topk_reg<8>(rows, d.C, k, scores, idx, sig, s);
    if (kpl <= 12) return launch_topk_reg<12>(rows, d.C, k, scores, idx, sig, s);
    if (kpl <= 16) return launch_topk_reg<16>(rows, d.C, k, scores, idx, sig, s);
    if (kpl <= 20) return launch_topk_reg<20>(rows, d.C, k, scores, idx, sig, s);
    if (kpl <= 24) return launch_topk_reg<24>(rows, d.C, k, scores, idx, sig, s);
    if (kpl <= 32) return launch_topk_reg<32>(rows, d.C, k, scores, idx, sig, s);
    if (kpl <= 40) return launch_topk_reg<40>(rows, d.C, k, scores, idx, sig, s);
    if (kpl <= 48) return launch_topk_reg<48>(rows, d.C, k, scores, idx, sig, s);
    return launch_topk_reg<64>(rows, d.C, k, scores, idx, sig, s);
}

}  // namespace

cudaError_t launch_topk(const Dims& d, const float* scores, int k, int32_t* idx, cudaStream_t s) {
    if (d.C > kTopkMaxC) return cudaErrorInvalidValue;
    if (d.C <= kTopkRegMaxC) return topk_reg_dispatch(d, scores, k, idx, nullptr, s);
    const int64_t rows = static_cast<int64_t>(d.B) * d.H * d.C;
    const int wpb = topk_warps_per_block(d.C);
    const size_t smem = static_cast<size_t>(wpb) * d.C * 4;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int64_t blocks_needed = (rows + wpb - 1) / wpb;
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
    topk_kernel<<<grid, wpb * 32, smem, s>>>(rows, d.C, k, scores, idx);
    return cudaGetLastError();
}

cudaError_t launch_topk_sig(const Dims& d, const float* scores, int k, int32_t* idx, uint64_t* sig, cudaStream_t s) {
    if (d.C > kTopkRegMaxC) return cudaErrorInvalidValue;
    return topk_reg_dispatch(d, scores, k, idx, sig, s);
}

cudaError_t launch_group_sort(const Dims& d, const uint64_t* sig, int32_t* order, cudaStream_t s) {
    if (d.C > kGroupMaxC) return cudaErrorInvalidValue;
    int cpow2 = 1;
    while (cpow2 < d.C) cpow2 <<= 1;
    group_sort_kernel<<<d.B * d.H, kGroupThreads, 0, s>>>(d.C, cpow2, sig, order);
    return cudaGetLastError();
}


}  // namespace vsa
