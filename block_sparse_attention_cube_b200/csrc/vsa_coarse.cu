// Cube selection (Wan2.2 teardown, zharfai.com, section "Video sparse
// attention selects cubes", part 1: the coarse scores rank the candidate key
// cubes, of which each query cube keeps the top-k) and the fine stage's work
// order.  The scores themselves come from vsa_coarse_mma.cu.
#include <cfloat>

#include "vsa_internal.h"

namespace vsa {
namespace {

constexpr int kThreads = 256;

// Order-preserving map float -> uint32 (larger float, larger key); -0 is
// folded onto +0 (-0 + 0 = +0) so that equal scores compare equal.  Every
// score's key is at least 0x007FFFFF (that of -inf), so 0 ranks below all.
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);
    return u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
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

// T = the k-th largest key of a row, built bit by bit from the top, searching only the bits below the
// highest one in which hi and lo differ (lo <= T <= hi); keys are counted over n[] (N per lane).
template <int N>
__device__ __forceinline__ uint32_t kth_key(const uint32_t (&n)[N], uint32_t hi, uint32_t lo, int k) {
    const uint32_t diff = hi ^ lo;
    const int top = diff ? 31 - __clz(diff) : -1;
    uint32_t T = top < 0 ? hi : (top >= 31 ? 0u : (hi & ~((2u << top) - 1u)));
#pragma unroll 1
    for (int bit = top; bit >= 0; --bit) {
        const uint32_t cand = T | (1u << bit);
        uint32_t cnt = 0;
#pragma unroll
        for (int i = 0; i < N; ++i) cnt += n[i] >= cand ? 1u : 0u;
        if (static_cast<int>(__reduce_add_sync(0xffffffffu, cnt)) >= k) T = cand;
    }
    return T;
}

__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

constexpr int kTopM = 4;      // k <= 32 * kTopM: the k-th largest is searched in a compacted candidate list
constexpr int kTopCand = 8;   // candidates per lane in that list (256 per row)

// Writes a row's selection (every key above T, then the lowest-index keys equal to T, ascending
// index) from keys held key j in lane j % 32, slot j / 32 of n[] (idx_of gives j), and returns the
// row's work-order key bits (its four smallest selected cubes, 12 bits each from bit 52 down).
template <int N, typename IndexOf>
__device__ __forceinline__ uint64_t write_selection(const uint32_t (&n)[N], int count, uint32_t T, int need_eq,
                                                    int32_t* dst, IndexOf idx_of) {
    const int lane = threadIdx.x & 31;
    const uint32_t lt_mask = (1u << lane) - 1u;
    int out = 0, eq_seen = 0, nlex = 0;
    uint64_t lex = 0ull;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        if (32 * i >= count) break;                      // warp-uniform
        const bool valid = lane + 32 * i < count;
        const bool is_gt = valid && n[i] > T;
        const bool is_eq = valid && n[i] == T;
        const uint32_t eq_mask = __ballot_sync(0xffffffffu, is_eq);
        const int eq_rank = eq_seen + __popc(eq_mask & lt_mask);
        const bool take = is_gt || (is_eq && eq_rank < need_eq);
        const uint32_t take_mask = __ballot_sync(0xffffffffu, take);
        const int j = idx_of(i);
        if (take) dst[out + __popc(take_mask & lt_mask)] = j;
        for (uint32_t mk = take_mask; nlex < 4 && mk != 0u; mk &= mk - 1u, ++nlex)   // warp-uniform
            lex |= static_cast<uint64_t>(__shfl_sync(0xffffffffu, j, __ffs(mk) - 1)) << (52 - 12 * nlex);
        out += __popc(take_mask);
        eq_seen += __popc(eq_mask);
    }
    return lex;
}

// Top-k with the row held in registers (KPL keys per lane, key j in lane j % 32, slot j / 32), for
// C <= 32 * KPL.  For k <= 32 the smallest lane maximum, for k <= 128 the k-th largest among the lanes'
// m + 1 largest keys (m = ceil(k / 32)), bounds the row's k-th largest from below (lo: at least k real
// keys reach it); when at most 256 keys reach lo
// they are compacted, with their cube indices and in index order, into a list whose count of keys
// >= t equals the row's for every t > lo (and both reach k for t <= lo), so the k-th largest key T
// is built bit by bit from the top over that short list, and the selection (every key above T, then
// the lowest-index keys equal to T, ascending) is read off the same list; otherwise both run over the
// whole row.  Either way the selection is topk_kernel's.  When `sig` is non-null the row's work-order
// key is written as well: its four smallest selected cubes (12 bits each, C <= 4096) above the
// cube's own index, so that sorting the keys puts query cubes whose selections start alike next to
// each other (the fine stage's tiles are pairs of consecutive cubes, and a tile's steps are the
// union of its two selections).
// 16 bytes global -> shared, asynchronous (cp.async, L2 only); groups committed and awaited per thread.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(reinterpret_cast<uint64_t>(src))
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// STAGED (C a multiple of 4, 16-byte aligned scores): each warp copies the next row it will take into
// the other half of its shared-memory row buffer (cp.async) while it works on the current one, so a
// row's loads are in flight during the previous row's selection.
template <int KPL, bool STAGED>
__global__ void __launch_bounds__(kThreads) topk_reg_kernel(int64_t rows, int C, int k, const float* __restrict__ scores,
                                                            int32_t* __restrict__ idx, uint64_t* __restrict__ sig) {
    __shared__ uint32_t cand_key_all[kThreads / 32][32 * kTopCand];
    __shared__ uint16_t cand_idx_all[kThreads / 32][32 * kTopCand];
    extern __shared__ __align__(16) float row_buf_all[];   // STAGED: [warp][2][C] floats
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t* cand_key = cand_key_all[warp];
    uint16_t* cand_idx = cand_idx_all[warp];
    float* row_buf = row_buf_all + static_cast<int64_t>(warp) * 2 * C;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
    const int m = (k + 31) / 32;
    auto stage = [&](int64_t r, int b) {   // row r's C floats into half b, one 16-byte chunk per lane per step
        const float* src = scores + r * C;
        float* dst = row_buf + b * C;
        for (int q = lane; q < C / 4; q += 32) cp_async16(dst + 4 * q, src + 4 * q);
        cp_async_commit();
    };
    const int64_t first = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + warp;
    if (STAGED && first < rows) stage(first, 0);
    int b = 0;
    for (int64_t row = first; row < rows; row += warps, b ^= 1) {
        const float* s = scores + row * C;
        uint32_t key[KPL];
        if constexpr (STAGED) {
            if (row + warps < rows) {
                stage(row + warps, b ^ 1);
                cp_async_wait<1>();   // this lane's copies of the current row have landed
            } else {
                cp_async_wait<0>();
            }
            __syncwarp();             // ... and every lane's
            const float* rb = row_buf + b * C;
#pragma unroll
            for (int i = 0; i < KPL; ++i) {
                const int j = lane + 32 * i;
                key[i] = j < C ? order_key(rb[j]) : 0u;   // 0 ranks below every real score
            }
            __syncwarp();             // the buffer is free for the copy two rows ahead
        } else {
#pragma unroll
            for (int i = 0; i < KPL; ++i) {
                const int j = lane + 32 * i;
                key[i] = j < C ? order_key(__ldcs(s + j)) : 0u;   // 0 ranks below every real score
            }
        }
        // lo: a lower bound of the k-th largest key.  For k <= 32: the smallest lane maximum (32 keys reach
        // it); for k <= 32 kTopM: the k-th largest among the lanes' m + 1 largest keys (k real keys reach
        // it); otherwise the row's smallest key.
        uint32_t hi, lo;
        int ncand = 0x7FFFFFFF;
        if (m <= kTopM) {
            uint32_t top[kTopM + 1] = {0u, 0u, 0u, 0u, 0u};   // the lane's m + 1 largest keys, descending
            if (m == 1) {
#pragma unroll
                for (int i = 0; i < KPL; ++i) top[0] = max(top[0], key[i]);
            } else if (m == 2) {
#pragma unroll
                for (int i = 0; i < KPL; ++i) {
                    uint32_t v = key[i];
#pragma unroll
                    for (int e = 0; e < 3; ++e) {
                        const uint32_t hv = max(top[e], v);
                        v = min(top[e], v);
                        top[e] = hv;
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < KPL; ++i) {
                    uint32_t v = key[i];
#pragma unroll
                    for (int e = 0; e < kTopM + 1; ++e) {
                        const uint32_t hv = max(top[e], v);
                        v = min(top[e], v);
                        top[e] = hv;
                    }
                }
            }
            hi = __reduce_max_sync(0xffffffffu, top[0]);
            if (m == 1) {
                // k <= 32: the smallest lane maximum already leaves few candidates (a search for a tighter
                // bound costs more than it saves)
                lo = __reduce_min_sync(0xffffffffu, top[0]);
            } else {
                const uint32_t lane_last = m == 2 ? top[2] : m == 3 ? top[3] : top[4];
                const uint32_t lo0 = __reduce_min_sync(0xffffffffu, lane_last);   // <= the bound sought
                if (m == 2) {
                    const uint32_t t3[3] = {top[0], top[1], top[2]};
                    lo = kth_key<3>(t3, hi, lo0, k);
                } else {
                    lo = kth_key<kTopM + 1>(top, hi, lo0, k);
                }
            }
            // a lane holding only padding (C < 32) has maximum 0; lo >= 1 keeps padding keys out of every
            // count below (real keys are all >= 1, and at least k of them reach lo)
            lo = max(lo, 1u);
            // the keys >= lo, with their cube indices and in index order, into the candidate list while it
            // has room; ncand counts them all
            ncand = 0;
#pragma unroll
            for (int i = 0; i < KPL; ++i) {
                const bool f = key[i] >= lo;
                const uint32_t bal = __ballot_sync(0xffffffffu, f);
                const int pos = ncand + __popc(bal & lt_mask);
                if (f && pos < 32 * kTopCand) {
                    cand_key[pos] = key[i];
                    cand_idx[pos] = static_cast<uint16_t>(lane + 32 * i);
                }
                ncand += __popc(bal);
            }
        } else {
            uint32_t lane_max = 0u, lane_min = 0xFFFFFFFFu;
#pragma unroll
            for (int i = 0; i < KPL; ++i) {
                lane_max = max(lane_max, key[i]);
                if (lane + 32 * i < C) lane_min = min(lane_min, key[i]);
            }
            hi = __reduce_max_sync(0xffffffffu, lane_max);
            lo = __reduce_min_sync(0xffffffffu, lane_min);
        }
        int32_t* dst = idx + row * k;
        uint64_t lex;
        if (ncand <= 32 * kTopCand) {
            __syncwarp();
            uint32_t ck[kTopCand];
#pragma unroll
            for (int e = 0; e < kTopCand; ++e) ck[e] = lane + 32 * e < ncand ? cand_key[lane + 32 * e] : 0u;
            const uint32_t T = ncand <= 64    ? kth_key<2>(reinterpret_cast<const uint32_t(&)[2]>(ck), hi, lo, k)
                               : ncand <= 128 ? kth_key<4>(reinterpret_cast<const uint32_t(&)[4]>(ck), hi, lo, k)
                                              : kth_key<kTopCand>(ck, hi, lo, k);
            uint32_t gt = 0;
#pragma unroll
            for (int e = 0; e < kTopCand; ++e) gt += ck[e] > T ? 1u : 0u;
            const int need_eq = k - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
            lex = write_selection<kTopCand>(ck, ncand, T, need_eq, dst,
                                            [&](int e) { return lane + 32 * e < ncand ? int(cand_idx[lane + 32 * e]) : 0; });
            __syncwarp();
        } else {
            // (padding keys are 0: below lo, so below T)
            const uint32_t T = kth_key<KPL>(key, hi, lo, k);
            uint32_t gt = 0;
#pragma unroll
            for (int i = 0; i < KPL; ++i) gt += key[i] > T ? 1u : 0u;
            const int need_eq = k - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
            lex = write_selection<KPL>(key, C, T, need_eq, dst, [&](int i) { return lane + 32 * i; });
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
    const bool staged = (C & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0;
    if (!staged) {
        topk_reg_kernel<KPL, false><<<grid, kThreads, 0, s>>>(rows, C, k, scores, idx, sig);
        return cudaGetLastError();
    }
    const size_t smem = static_cast<size_t>(kThreads / 32) * 2 * C * 4;   // <= 128 KB for C <= 2048
    static int configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (!(dev >= 0 && dev < 64 && configured[dev])) {
        e = cudaFuncSetAttribute(topk_reg_kernel<KPL, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(static_cast<size_t>(kThreads / 32) * 2 * (32 * KPL) * 4));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = 1;
    }
    topk_reg_kernel<KPL, true><<<grid, kThreads, smem, s>>>(rows, C, k, scores, idx, sig);
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
