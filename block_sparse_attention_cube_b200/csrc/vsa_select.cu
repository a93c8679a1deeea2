// The coarse stage and the cube selection in one kernel (Wan2.2 teardown,
// zharfai.com, section "Video sparse attention selects cubes", part 1: cheap
// block-level attention over the mean-pooled cubes ranks the candidate key
// cubes, and each query cube keeps the top-k; section "Fusion targets launch
// overhead and memory": work that would round-trip HBM between two launches
// stays on chip).
//
// One block owns 32 query cubes of one (b, h).  It computes their rows of the
// coarse scores into shared memory (each score the same sequential float32
// fma chain over the channels as coarse_scores_kernel, so the bits are
// identical), selects each row's top-k key cubes there (the same rule as
// vsa_topk: the k largest, ties to the lower index, ascending output), writes
// each row's work-order key, and, when V-bar is given, turns the rows into
// softmax probabilities in place and multiplies them by V-bar for the coarse
// output.  The [B, H, C, C] score matrix never reaches global memory.
#include <cfloat>

#include "ptx_sm100.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

using ptx::fma_f32x2;
using ptx::f32x2;
using ptx::f32x2_split;

constexpr int kSelRows = 32;      // query cubes per block
constexpr int kSelThreads = 256;  // 8 warps
constexpr int kSelKT = 256;       // key cubes per score tile (4 warp columns of 64)
constexpr int kSelBK = 16;        // channels per staged slice of K-bar
constexpr int kSelVK = 16;        // key cubes per staged slice of V-bar
constexpr int kSelTopM = 4;       // k <= 32 * kSelTopM: the selection searches a compacted candidate list
constexpr int kSelCand = 8;       // candidates per lane in that list (256 per row)
constexpr int kSelMaxC = 1536;    // largest C whose 32 score rows (and the staging) fit in shared memory

struct SelParams {
    int C, k;
    float scale;
    const float* qbar;
    const float* kbar;
    const float* vbar;       // null: no coarse output
    int32_t* idx;
    uint64_t* sig;           // null: no work-order keys
    float* o_coarse;
    float* scores_out;       // null, or a copy of the ranked scores
};

// Order-preserving map float -> uint32 (larger float, larger key); -0 folds onto +0.
__device__ __forceinline__ uint32_t sel_key(float f) {
    if (f == 0.0f) f = 0.0f;
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float sel_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Score row storage: key cube j, query row r (0..31) at j*32 + 4*((r/4) ^ (j%8)) + r%4.  Four
// consecutive rows stay one 16-byte chunk; the XOR spreads a warp's reads of one row over 8 chunks.
__device__ __forceinline__ int st_off(int j, int r) { return j * kSelRows + ((((r >> 2) ^ (j & 7))) << 2) + (r & 3); }
__device__ __forceinline__ int st_chunk(int j, int q) { return j * kSelRows + ((q ^ (j & 7)) << 2); }

size_t sel_smem_bytes(int C, int D) {
    const size_t cpad = static_cast<size_t>((C + 63) / 64) * 64;
    return cpad * kSelRows * 4 + static_cast<size_t>(D) * kSelRows * 4 + static_cast<size_t>(kSelBK) * kSelKT * 4 +
           kSelRows * 4;
}

// T = the k-th largest key of the row, built bit by bit from the top, searching only the bits below
// the highest one in which hi and lo differ (lo <= T <= hi); keys are counted over n[] (N per lane).
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

template <int D, int KPL>
__global__ void __launch_bounds__(kSelThreads, 2) coarse_select_kernel(SelParams p) {
    extern __shared__ __align__(16) float sm[];
    const int C = p.C;
    const int cpad = (C + 63) / 64 * 64;
    float* St = sm;                               // [cpad][32] score rows (swizzled), then probabilities
    float* As = St + cpad * kSelRows;             // [D][32] the block's query cubes, channel-major
    float* Bs = As + D * kSelRows;                // [16][256] K-bar slice; later candidates and V-bar slices
    float* row_inv = Bs + kSelBK * kSelKT;        // [32] 1 / softmax denominator
    const int bh = blockIdx.y;
    const int i0 = blockIdx.x * kSelRows;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const float* Q = p.qbar + static_cast<int64_t>(bh) * C * D;
    const float* K = p.kbar + static_cast<int64_t>(bh) * C * D;

    // ---- the block's query cubes, transposed: lanes take consecutive rows of one channel group
    for (int e = t; e < kSelRows * (D / 4); e += kSelThreads) {
        const int r = e % kSelRows, d4 = e / kSelRows;
        const float4 v = i0 + r < C ? __ldg(reinterpret_cast<const float4*>(Q + static_cast<int64_t>(i0 + r) * D) + d4)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        As[(4 * d4 + 0) * kSelRows + r] = v.x;
        As[(4 * d4 + 1) * kSelRows + r] = v.y;
        As[(4 * d4 + 2) * kSelRows + r] = v.z;
        As[(4 * d4 + 3) * kSelRows + r] = v.w;
    }

    // ---- scores: tiles of 256 key cubes; warp (wr, wc) owns rows 16wr..16wr+15 and keys 64wc..64wc+63
    // of the tile, lane (ty, tx) rows 8ty..8ty+7 of those and keys 4tx..4tx+3
    const int wr = warp & 1, wc = warp >> 1;
    const int ty = lane >> 4, tx = lane & 15;
    const int row0 = 16 * wr + 8 * ty;
    constexpr int kSlices = D / kSelBK;
    const int tiles = (C + kSelKT - 1) / kSelKT;
    float4 pre[kSelBK / 4];   // thread t stages key (tile + t), 16 channels
    auto load_slice = [&](int tile, int s) {
        const int j = tile * kSelKT + t;
#pragma unroll
        for (int u = 0; u < kSelBK / 4; ++u)
            pre[u] = j < C ? __ldg(reinterpret_cast<const float4*>(K + static_cast<int64_t>(j) * D + s * kSelBK) + u)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    load_slice(0, 0);
    for (int tile = 0; tile < tiles; ++tile) {
        const int kt0 = tile * kSelKT;
        const bool active = kt0 + 64 * wc < C;   // warp-uniform
        // acc[c][rp]: key c, rows (2rp, 2rp+1) of the thread's eight, as one packed float32 pair
        uint64_t acc[4][4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int rp = 0; rp < 4; ++rp) acc[c][rp] = 0ull;
        for (int s = 0; s < kSlices; ++s) {
#pragma unroll
            for (int u = 0; u < kSelBK / 4; ++u) {
                Bs[(4 * u + 0) * kSelKT + t] = pre[u].x;
                Bs[(4 * u + 1) * kSelKT + t] = pre[u].y;
                Bs[(4 * u + 2) * kSelKT + t] = pre[u].z;
                Bs[(4 * u + 3) * kSelKT + t] = pre[u].w;
            }
            __syncthreads();
            if (s + 1 < kSlices) load_slice(tile, s + 1);
            else if (tile + 1 < tiles) load_slice(tile + 1, 0);
            if (active) {
                const float* a_base = As + (s * kSelBK) * kSelRows + row0;
                const float* b_base = Bs + 64 * wc + 4 * tx;
                // operands of step kk + 1 are read while step kk multiplies
                ulonglong2 a_lo = *reinterpret_cast<const ulonglong2*>(a_base);
                ulonglong2 a_hi = *reinterpret_cast<const ulonglong2*>(a_base + 4);
                float4 b = *reinterpret_cast<const float4*>(b_base);
#pragma unroll
                for (int kk = 0; kk < kSelBK; ++kk) {
                    const uint64_t ap[4] = {a_lo.x, a_lo.y, a_hi.x, a_hi.y};
                    const float bv[4] = {b.x, b.y, b.z, b.w};
                    if (kk + 1 < kSelBK) {
                        a_lo = *reinterpret_cast<const ulonglong2*>(a_base + (kk + 1) * kSelRows);
                        a_hi = *reinterpret_cast<const ulonglong2*>(a_base + (kk + 1) * kSelRows + 4);
                        b = *reinterpret_cast<const float4*>(b_base + (kk + 1) * kSelKT);
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint64_t bb = f32x2(bv[c], bv[c]);
#pragma unroll
                        for (int rp = 0; rp < 4; ++rp) acc[c][rp] = fma_f32x2(ap[rp], bb, acc[c][rp]);
                    }
                }
            }
            __syncthreads();
        }
        if (active) {
            // scale * acc, the same single rounding as coarse_scores_kernel; rows of the block past C and
            // keys past C hold scores of zero vectors, which nothing reads as real
            float sc[8][4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int rp = 0; rp < 4; ++rp) {
                    f32x2_split(acc[c][rp], sc[2 * rp][c], sc[2 * rp + 1][c]);
                    sc[2 * rp][c] = p.scale * sc[2 * rp][c];
                    sc[2 * rp + 1][c] = p.scale * sc[2 * rp + 1][c];
                }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int j = kt0 + 64 * wc + 4 * tx + c;   // < cpad: active warps start below C
                const int q0 = row0 >> 2;
                *reinterpret_cast<float4*>(St + st_chunk(j, q0)) = make_float4(sc[0][c], sc[1][c], sc[2][c], sc[3][c]);
                *reinterpret_cast<float4*>(St + st_chunk(j, q0 + 1)) =
                    make_float4(sc[4][c], sc[5][c], sc[6][c], sc[7][c]);
                if (p.scores_out != nullptr && j < C) {
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const int gi = i0 + row0 + r;
                        if (gi < C) p.scores_out[(static_cast<int64_t>(bh) * C + gi) * C + j] = sc[r][c];
                    }
                }
            }
        }
    }
    __syncthreads();

    // ---- selection: warp w takes rows w, w+8, w+16, w+24; the row sits in registers, key j in lane j%32
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t* cand = reinterpret_cast<uint32_t*>(Bs) + warp * (32 * kSelCand);
    const int k = p.k;
    const int m = (k + 31) / 32;   // per-lane rank that bounds the k-th largest from below
    for (int r = warp; r < kSelRows; r += kSelThreads / 32) {
        const int i = i0 + r;
        if (i >= C) break;
        uint32_t key[KPL];
#pragma unroll
        for (int u = 0; u < KPL; ++u) {
            const int j = lane + 32 * u;
            key[u] = j < C ? sel_key(St[st_off(j, r)]) : 0u;   // 0 ranks below every real score
        }
        uint32_t lane_max = 0u, lane_m = 0u;   // the lane's largest and m-th largest keys
        if (m == 1) {
#pragma unroll
            for (int u = 0; u < KPL; ++u) lane_max = max(lane_max, key[u]);
            lane_m = lane_max;
        } else if (m <= kSelTopM) {
            uint32_t top[kSelTopM] = {0u, 0u, 0u, 0u};   // descending
#pragma unroll
            for (int u = 0; u < KPL; ++u) {
                uint32_t v = key[u];
#pragma unroll
                for (int e = 0; e < kSelTopM; ++e) {
                    const uint32_t hi_v = max(top[e], v);
                    v = min(top[e], v);
                    top[e] = hi_v;
                }
            }
            lane_max = top[0];
            lane_m = m == 2 ? top[1] : m == 3 ? top[2] : top[3];
        } else {
#pragma unroll
            for (int u = 0; u < KPL; ++u) lane_max = max(lane_max, key[u]);
        }
        const uint32_t hi = __reduce_max_sync(0xffffffffu, lane_max);
        uint32_t T;
        if (m <= kSelTopM) {
            // at least 32*m >= k keys reach lo (each lane holds m of them), so the k-th largest is >= lo
            const uint32_t lo = __reduce_min_sync(0xffffffffu, lane_m);
            uint32_t mine = 0;
#pragma unroll
            for (int u = 0; u < KPL; ++u) mine += (lane + 32 * u < C && key[u] >= lo) ? 1u : 0u;
            const int ncand = static_cast<int>(__reduce_add_sync(0xffffffffu, mine));
            if (ncand <= 32 * kSelCand) {
                // every key >= lo to a compact list; counting over it equals counting over the row
                // for every threshold above lo, and both accept every threshold at or below it
                int base = 0;
#pragma unroll
                for (int u = 0; u < KPL; ++u) {
                    const bool f = lane + 32 * u < C && key[u] >= lo;
                    const uint32_t bal = __ballot_sync(0xffffffffu, f);
                    if (f) cand[base + __popc(bal & lt_mask)] = key[u];
                    base += __popc(bal);
                }
                __syncwarp();
                uint32_t ck[kSelCand];
#pragma unroll
                for (int e = 0; e < kSelCand; ++e) ck[e] = lane + 32 * e < ncand ? cand[lane + 32 * e] : 0u;
                __syncwarp();
                T = ncand <= 32 * (kSelCand / 2) ? kth_key<kSelCand / 2>(reinterpret_cast<const uint32_t(&)[kSelCand / 2]>(ck), hi, lo, k)
                                                 : kth_key<kSelCand>(ck, hi, lo, k);
            } else {
                T = kth_key<KPL>(key, hi, lo, k);
            }
        } else {
            uint32_t lane_min = 0xFFFFFFFFu;
#pragma unroll
            for (int u = 0; u < KPL; ++u)
                if (lane + 32 * u < C) lane_min = min(lane_min, key[u]);
            T = kth_key<KPL>(key, hi, __reduce_min_sync(0xffffffffu, lane_min), k);
        }
        // every key above T, then the lowest-index keys equal to T, in index order
        uint32_t gt = 0;
#pragma unroll
        for (int u = 0; u < KPL; ++u) gt += key[u] > T ? 1u : 0u;
        const int need_eq = k - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
        int out = 0, eq_seen = 0;
        int32_t* dst = p.idx + (static_cast<int64_t>(bh) * C + i) * k;
        uint64_t lex = 0ull;   // the row's four smallest selected cubes, 12 bits each from bit 52 down
        int nlex = 0;
#pragma unroll
        for (int u = 0; u < KPL; ++u) {
            const int j = lane + 32 * u;
            const bool valid = j < C;
            const bool is_gt = valid && key[u] > T;
            const bool is_eq = valid && key[u] == T;
            const uint32_t eq_mask = __ballot_sync(0xffffffffu, is_eq);
            const int eq_rank = eq_seen + __popc(eq_mask & lt_mask);
            const bool take = is_gt || (is_eq && eq_rank < need_eq);
            const uint32_t take_mask = __ballot_sync(0xffffffffu, take);
            if (take) dst[out + __popc(take_mask & lt_mask)] = j;
            out += __popc(take_mask);
            eq_seen += __popc(eq_mask);
            for (uint32_t mk = take_mask; nlex < 4 && mk != 0u; mk &= mk - 1u, ++nlex)
                lex |= static_cast<uint64_t>(32 * u + __ffs(mk) - 1) << (52 - 12 * nlex);
        }
        if (p.sig != nullptr && lane == 0) p.sig[static_cast<int64_t>(bh) * C + i] = lex | static_cast<uint64_t>(i);
        if (p.vbar != nullptr) {
            // probabilities in place: exp(s - max), the maximum being the largest key (the keys decode
            // back to the scores exactly, -0 as +0); keys past C up to cpad get 0
            const float mx = sel_value(hi);
            float l = 0.f;
#pragma unroll
            for (int u = 0; u < KPL; ++u) {
                const int j = lane + 32 * u;
                if (j >= cpad) break;
                const float e = j < C ? expf(sel_value(key[u]) - mx) : 0.f;
                St[st_off(j, r)] = e;
                l += e;
            }
#pragma unroll
            for (int off = 16; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
            if (lane == 0) row_inv[r] = 1.0f / l;
        }
    }
    if (p.vbar == nullptr) return;
    __syncthreads();

    // ---- coarse output: O = P V-bar / l.  Thread (h, py, px): rows 8py..8py+7, channels CPT*px.., and
    // keys 8h..8h+7 of every 16-key slice; the two halves h = 0, 1 add their sums at the end.
    constexpr int CPT = D / 32;                          // channels per thread: 4 (D = 128) or 2 (D = 64)
    const int h = t / 128, py = (t / 32) % 4, px = t % 32;
    const float* V = p.vbar + static_cast<int64_t>(bh) * C * D;
    float* Vs = Bs;                                      // [16][D]
    constexpr int VF4 = kSelVK * D / 4 / kSelThreads;    // float4 of a V-bar slice per thread
    float4 vpre[VF4];
    auto load_v = [&](int j0) {
#pragma unroll
        for (int u = 0; u < VF4; ++u) {
            const int e = t + u * kSelThreads;
            const int kk = e / (D / 4), c4 = e % (D / 4);
            vpre[u] = j0 + kk < C ? __ldg(reinterpret_cast<const float4*>(V + static_cast<int64_t>(j0 + kk) * D) + c4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    // oacc[c][rp]: channel c, rows (2rp, 2rp+1), packed
    uint64_t oacc[CPT][4];
#pragma unroll
    for (int c = 0; c < CPT; ++c)
#pragma unroll
        for (int rp = 0; rp < 4; ++rp) oacc[c][rp] = 0ull;
    load_v(0);
    for (int j0 = 0; j0 < C; j0 += kSelVK) {
#pragma unroll
        for (int u = 0; u < VF4; ++u) {
            const int e = t + u * kSelThreads;
            *reinterpret_cast<float4*>(Vs + (e / (D / 4)) * D + 4 * (e % (D / 4))) = vpre[u];
        }
        __syncthreads();
        if (j0 + kSelVK < C) load_v(j0 + kSelVK);
#pragma unroll
        for (int kk = 8 * h; kk < 8 * h + 8; ++kk) {
            const int j = j0 + kk;
            const ulonglong2 p0 = *reinterpret_cast<const ulonglong2*>(St + st_chunk(j, 2 * py));
            const ulonglong2 p1 = *reinterpret_cast<const ulonglong2*>(St + st_chunk(j, 2 * py + 1));
            const uint64_t pp[4] = {p0.x, p0.y, p1.x, p1.y};
            float vv[CPT];
            if constexpr (CPT == 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(Vs + kk * D + 4 * px);
                vv[0] = v4.x;
                vv[1] = v4.y;
                vv[2] = v4.z;
                vv[3] = v4.w;
            } else {
                const float2 v2 = *reinterpret_cast<const float2*>(Vs + kk * D + 2 * px);
                vv[0] = v2.x;
                vv[1] = v2.y;
            }
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                const uint64_t vb = f32x2(vv[c], vv[c]);
#pragma unroll
                for (int rp = 0; rp < 4; ++rp) oacc[c][rp] = fma_f32x2(pp[rp], vb, oacc[c][rp]);
            }
        }
        __syncthreads();
    }
    // half 1 hands its sums to half 0 through the (now idle) staging buffer: [32 rows][D]
    float* part = Bs;
    float o[8][CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c)
#pragma unroll
        for (int rp = 0; rp < 4; ++rp) f32x2_split(oacc[c][rp], o[2 * rp][c], o[2 * rp + 1][c]);
    if (h == 1) {
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int c = 0; c < CPT; ++c) part[(8 * py + r) * D + CPT * px + c] = o[r][c];
    }
    __syncthreads();
    if (h == 1) return;
    float* O = p.o_coarse + static_cast<int64_t>(bh) * C * D;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int li = 8 * py + r, gi = i0 + li;
        if (gi >= C) continue;
        const float inv = row_inv[li];
        float v[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c) v[c] = (o[r][c] + part[li * D + CPT * px + c]) * inv;
        if constexpr (CPT == 4) {
            *reinterpret_cast<float4*>(O + static_cast<int64_t>(gi) * D + 4 * px) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
            *reinterpret_cast<float2*>(O + static_cast<int64_t>(gi) * D + 2 * px) = make_float2(v[0], v[1]);
        }
    }
}

template <int D, int KPL>
cudaError_t launch_select_instance(const Dims& d, const SelParams& p, size_t smem, cudaStream_t s) {
    static int configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (!(dev >= 0 && dev < 64 && configured[dev])) {
        e = cudaFuncSetAttribute(coarse_select_kernel<D, KPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(sel_smem_bytes(kSelMaxC, D)));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = 1;
    }
    const dim3 grid((d.C + kSelRows - 1) / kSelRows, d.B * d.H);
    coarse_select_kernel<D, KPL><<<grid, kSelThreads, smem, s>>>(p);
    return cudaGetLastError();
}

template <int D>
cudaError_t select_dispatch(const Dims& d, const SelParams& p, size_t smem, cudaStream_t s) {
    const int kpl = (d.C + 31) / 32;
    if (kpl <= 4) return launch_select_instance<D, 4>(d, p, smem, s);
    if (kpl <= 8) return launch_select_instance<D, 8>(d, p, smem, s);
    if (kpl <= 12) return launch_select_instance<D, 12>(d, p, smem, s);
    if (kpl <= 16) return launch_select_instance<D, 16>(d, p, smem, s);
    if (kpl <= 20) return launch_select_instance<D, 20>(d, p, smem, s);
    if (kpl <= 24) return launch_select_instance<D, 24>(d, p, smem, s);
    if (kpl <= 32) return launch_select_instance<D, 32>(d, p, smem, s);
    if (kpl <= 40) return launch_select_instance<D, 40>(d, p, smem, s);
    return launch_select_instance<D, 48>(d, p, smem, s);
}

}  // namespace

bool coarse_select_supported(const Dims& d) {
    return d.C <= kSelMaxC && sel_smem_bytes(d.C, d.D) <= 227u * 1024u;
}

cudaError_t launch_coarse_select(const Dims& d, const float* qbar, const float* kbar, const float* vbar, float scale,
                                 int k, int32_t* idx, uint64_t* sig, float* o_coarse, float* scores_out,
                                 cudaStream_t s) {
    if (!coarse_select_supported(d) || k < 1 || k > d.C) return cudaErrorInvalidValue;
    SelParams p{};
    p.C = d.C;
    p.k = k;
    p.scale = scale;
    p.qbar = qbar;
    p.kbar = kbar;
    p.vbar = o_coarse ? vbar : nullptr;
    p.idx = idx;
    p.sig = sig;
    p.o_coarse = o_coarse;
    p.scores_out = scores_out;
    const size_t smem = sel_smem_bytes(d.C, d.D);
    return d.D == 128 ? select_dispatch<128>(d, p, smem, s) : select_dispatch<64>(d, p, smem, s);
}

}  // namespace vsa
