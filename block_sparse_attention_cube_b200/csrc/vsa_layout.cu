// Memory-bound steps of the path: cube-major tiling with zero padding, its
// inverse, the cube mean-pool and the gated merge.
//
// All four kernels work on "cube tasks" (tensor, b, h, cube) with a
// grid-stride loop over a grid sized as a multiple of the SM count; a block
// of 256 threads moves one cube (64 rows of D bf16) per task with 16-byte
// vector accesses.  The cube-major order is the one of the Wan2.2 teardown
// (zharfai.com), section "Video sparse attention selects cubes": 4x4x4 cubes
// of 64 tokens on a grid padded per axis to a multiple of 4.
#include <cuda_bf16.h>

#include "vsa_internal.h"

namespace vsa {
namespace {

constexpr int kBlock = 256;
// Resident blocks per SM that the copy kernels' register bounds guarantee; their
// grids are sized to exactly that many per SM.
constexpr int kLayoutPerSm = 8;

struct CubeTask {
    int tensor;
    int64_t bh;   // b * H + h
    int b, h, c;
    int ct, cx, cy;
};

__device__ __forceinline__ CubeTask decode_task(int64_t task, const Dims& d) {
    const int64_t per_tensor = static_cast<int64_t>(d.B) * d.H * d.C;
    CubeTask t;
    t.tensor = static_cast<int>(task / per_tensor);
    const int64_t r = task - t.tensor * per_tensor;
    t.c = static_cast<int>(r % d.C);
    t.bh = r / d.C;
    t.h = static_cast<int>(t.bh % d.H);
    t.b = static_cast<int>(t.bh / d.H);
    t.ct = t.c / (d.Cx * d.Cy);
    t.cx = (t.c / d.Cy) % d.Cx;
    t.cy = t.c % d.Cy;
    return t;
}

// Source token of offset o inside the cube, or -1 for a padded position.
__device__ __forceinline__ int64_t token_of(const Dims& d, const CubeTask& t, int o) {
    const int tt = t.ct * kCube + (o >> 4);
    const int xx = t.cx * kCube + ((o >> 2) & 3);
    const int yy = t.cy * kCube + (o & 3);
    if (tt >= d.T || xx >= d.X || yy >= d.Y) return -1;
    return (static_cast<int64_t>(tt) * d.X + xx) * d.Y + yy;
}

// A thread's PER row loads are all issued before its first store.
template <int D>
__global__ void __launch_bounds__(kBlock, kLayoutPerSm) tile_kernel(Dims d, Bf16Triple io) {
    constexpr int CH = D / 8;                   // 16-byte chunks per row
    constexpr int PER = kCubeTokens * CH / kBlock;
    constexpr int ROWS = kBlock / CH;           // rows covered by one pass of the block
    static_assert(kBlock % CH == 0, "a thread's column chunk must stay fixed across its rows");
    const int64_t total = static_cast<int64_t>(d.B) * d.H * d.C * io.count;
    const int j = threadIdx.x % CH, o0 = threadIdx.x / CH;
    for (int64_t task = blockIdx.x; task < total; task += gridDim.x) {
        const CubeTask t = decode_task(task, d);
        // pointers chosen by value: a runtime index into the parameter arrays would go through local memory
        const uint16_t* src_t = t.tensor == 0 ? io.src[0] : t.tensor == 1 ? io.src[1] : io.src[2];
        uint16_t* dst_t = t.tensor == 0 ? io.dst[0] : t.tensor == 1 ? io.dst[1] : io.dst[2];
        const uint4* src = reinterpret_cast<const uint4*>(src_t);
        uint4* dst = reinterpret_cast<uint4*>(dst_t);
        const int64_t out_row0 = t.bh * d.Npad + static_cast<int64_t>(t.c) * kCubeTokens;
        uint4 v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int64_t n = token_of(d, t, o0 + i * ROWS);
            v[i] = n >= 0 ? __ldcs(src + ((static_cast<int64_t>(t.b) * d.N + n) * d.H + t.h) * CH + j)
                          : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) dst[(out_row0 + o0 + i * ROWS) * CH + j] = v[i];
    }
}

template <int D>
__global__ void __launch_bounds__(kBlock, kLayoutPerSm) untile_kernel(Dims d, const uint16_t* __restrict__ xt,
                                                                      uint16_t* __restrict__ x) {
    constexpr int CH = D / 8;
    constexpr int PER = kCubeTokens * CH / kBlock;
    const int64_t total = static_cast<int64_t>(d.B) * d.H * d.C;
    const uint4* src = reinterpret_cast<const uint4*>(xt);
    uint4* dst = reinterpret_cast<uint4*>(x);
    for (int64_t task = blockIdx.x; task < total; task += gridDim.x) {
        const CubeTask t = decode_task(task, d);
        const int64_t in_row0 = t.bh * d.Npad + static_cast<int64_t>(t.c) * kCubeTokens;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int q = threadIdx.x + i * kBlock;
            const int o = q / CH, j = q % CH;
            const int64_t n = token_of(d, t, o);
            if (n < 0) continue;
            const uint4 v = __ldcs(src + (in_row0 + o) * CH + j);
            __stcs(dst + ((static_cast<int64_t>(t.b) * d.N + n) * d.H + t.h) * CH + j, v);
        }
    }
}

// One warp per cube: lanes split a row into 16-byte chunks, rows are spread
// over the warp's lane groups, partial sums are combined with shuffles.
struct PoolIO {
    const uint16_t* src[3];
    float* dst[3];          // float32 means [B, H, C, D], or null
    uint16_t* parts[3];     // the means as three bf16 parts [3][B*H][C][D], or null
    int count;
};

// x = hi + mid + lo with each part the bf16 nearest to what the larger parts leave (the residuals are
// exact in float32); the three parts hold x to within 2^-24 |x| (bits: bf16 patterns).
__device__ __forceinline__ void split3(float x, uint16_t& hi, uint16_t& mid, uint16_t& lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(m);
    const __nv_bfloat16 l = __float2bfloat16_rn(r2);
    hi = __bfloat16_as_ushort(h);
    mid = __bfloat16_as_ushort(m);
    lo = __bfloat16_as_ushort(l);
}

// Eight consecutive float32 values to their three bf16 parts: 16 bytes into each part plane.
__device__ __forceinline__ void store_parts8(const float (&v)[8], uint16_t* parts, int64_t plane, int64_t off) {
    uint32_t h[4], m[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        uint16_t h0, m0, l0, h1, m1, l1;
        split3(v[2 * e], h0, m0, l0);
        split3(v[2 * e + 1], h1, m1, l1);
        h[e] = h0 | (uint32_t{h1} << 16);
        m[e] = m0 | (uint32_t{m1} << 16);
        l[e] = l0 | (uint32_t{l1} << 16);
    }
    *reinterpret_cast<uint4*>(parts + off) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(parts + plane + off) = make_uint4(m[0], m[1], m[2], m[3]);
    *reinterpret_cast<uint4*>(parts + 2 * plane + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

template <int D>
__global__ void __launch_bounds__(kBlock) pool_kernel(Dims d, PoolIO io) {
    constexpr int LPR = D / 8;          // lanes per row
    constexpr int RPI = 32 / LPR;       // rows per warp iteration
    const int lane = threadIdx.x & 31;
    const int sub = lane / LPR, j = lane % LPR;
    const int64_t total = static_cast<int64_t>(d.B) * d.H * d.C * io.count;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (kBlock / 32);
    for (int64_t task = static_cast<int64_t>(blockIdx.x) * (kBlock / 32) + threadIdx.x / 32; task < total;
         task += warps) {
        const CubeTask t = decode_task(task, d);
        const uint4* src = reinterpret_cast<const uint4*>(io.src[t.tensor]);
        const int64_t row0 = t.bh * d.Npad + static_cast<int64_t>(t.c) * kCubeTokens;
        const int nt = min(kCube, d.T - t.ct * kCube);
        const int nx = min(kCube, d.X - t.cx * kCube);
        const int ny = min(kCube, d.Y - t.cy * kCube);
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 4
        for (int o = sub; o < kCubeTokens; o += RPI) {
            if ((o >> 4) >= nt || ((o >> 2) & 3) >= nx || (o & 3) >= ny) continue;
            const uint4 v = __ldcs(src + (row0 + o) * LPR + j);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[2 * e] += __uint_as_float(w[e] << 16);
                acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
#pragma unroll
        for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
        }
        if (sub == 0) {
            const float inv = 1.0f / static_cast<float>(nt * nx * ny);
            float4* out = reinterpret_cast<float4*>(io.dst[t.tensor] + (t.bh * d.C + t.c) * D + j * 8);
            out[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
            out[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
        }
    }
}

// The same pool read straight from the projection layout [B, N, H, D], so a
// forward call needs no tiled copy.  A token's H*D channels are contiguous,
// so a block of kPoolThreads threads owns one (tensor, b, cube) and a range
// of 16-byte channel chunks, one chunk per thread, and walks the cube's real
// tokens: every token row it reads is kPoolThreads * 16 contiguous bytes.
// Each channel is summed in the order of pool_kernel: R = 256 / D partial
// sums over the offsets o with o % R == r, each in offset order, combined as
// pool_kernel's shuffle tree does; both kernels give identical float32 means.
constexpr int kPoolThreads = 128;

template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_tokens_kernel(Dims d, PoolIO io) {
    constexpr int CH = D / 8;            // 16-byte chunks per head
    constexpr int R = 256 / D;           // partial sums per channel (lane groups of pool_kernel)
    const int q = blockIdx.y * kPoolThreads + threadIdx.x;   // chunk of the token row
    if (q >= d.H * CH) return;
    const int64_t bc = blockIdx.x;       // (tensor * B + b) * C + c
    const int c = static_cast<int>(bc % d.C);
    const int tb = static_cast<int>(bc / d.C);
    const int tensor = tb / d.B, b = tb - tensor * d.B;
    const int h = q / CH, j = q - h * CH;
    const int ct = c / (d.Cx * d.Cy), cx = (c / d.Cy) % d.Cx, cy = c % d.Cy;
    const int nt = min(kCube, d.T - ct * kCube);
    const int nx = min(kCube, d.X - cx * kCube);
    const int ny = min(kCube, d.Y - cy * kCube);
    const int64_t row = static_cast<int64_t>(d.H) * CH;   // 16-byte chunks per token
    // pick the tensor's pointers by value: indexing the parameter arrays with a runtime index would copy them
    // to the stack
    const uint16_t* src_t = tensor == 0 ? io.src[0] : tensor == 1 ? io.src[1] : io.src[2];
    float* dst_t = tensor == 0 ? io.dst[0] : tensor == 1 ? io.dst[1] : io.dst[2];
    uint16_t* parts_t = tensor == 0 ? io.parts[0] : tensor == 1 ? io.parts[1] : io.parts[2];
    const uint4* src = reinterpret_cast<const uint4*>(src_t) + static_cast<int64_t>(b) * d.N * row + q;
    const int64_t base_n = (static_cast<int64_t>(ct) * kCube * d.X + cx * kCube) * d.Y + cy * kCube;
    float acc[R][8];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[r][e] = 0.f;
#pragma unroll
    for (int o = 0; o < kCubeTokens; ++o) {
        const int ot = o >> 4, ox = (o >> 2) & 3, oy = o & 3;
        if (ot >= nt || ox >= nx || oy >= ny) continue;
        const int64_t n = base_n + (static_cast<int64_t>(ot) * d.X + ox) * d.Y + oy;
        const uint4 v = __ldcs(src + n * row);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc[o % R][2 * e] += __uint_as_float(w[e] << 16);
            acc[o % R][2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
    float m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        if (R == 1) m[e] = acc[0][e];
        else if (R == 2) m[e] = acc[0][e] + acc[R - 1][e];
        else m[e] = (acc[0][e] + acc[1 % R][e]) + (acc[2 % R][e] + acc[3 % R][e]);
    }
    const float inv = 1.0f / static_cast<float>(nt * nx * ny);
    const int64_t bh = static_cast<int64_t>(b) * d.H + h;
    float mean[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) mean[e] = m[e] * inv;
    if (dst_t != nullptr) {
        float4* out = reinterpret_cast<float4*>(dst_t + (bh * d.C + c) * D + j * 8);
        out[0] = make_float4(mean[0], mean[1], mean[2], mean[3]);
        out[1] = make_float4(mean[4], mean[5], mean[6], mean[7]);
    }
    if (parts_t != nullptr)
        store_parts8(mean, parts_t, static_cast<int64_t>(d.B) * d.H * d.C * D, (bh * d.C + c) * D + j * 8);
}

// Up to three tensors in one launch: float32 [rows, D] -> three bf16 parts [3][rows][D] each (the
// split of pool_tokens_kernel's means).
struct SplitIO {
    const float* x[3];
    uint16_t* parts[3];
    int count;
};

__global__ void __launch_bounds__(kBlock) split_parts_kernel(int64_t groups, const SplitIO io) {
    const int64_t total = groups * io.count;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kBlock + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * kBlock) {
        const int t = static_cast<int>(i / groups);
        const int64_t g = i - t * groups;
        // pointers chosen by value: a runtime index into the parameter arrays would go through local memory
        const float* x = t == 0 ? io.x[0] : t == 1 ? io.x[1] : io.x[2];
        uint16_t* parts = t == 0 ? io.parts[0] : t == 1 ? io.parts[1] : io.parts[2];
        const float4 a = __ldg(reinterpret_cast<const float4*>(x) + 2 * g);
        const float4 b = __ldg(reinterpret_cast<const float4*>(x) + 2 * g + 1);
        const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        store_parts8(v, parts, groups * 8, g * 8);
    }
}

// Each thread keeps one 16-byte column chunk j of the cube's rows (kBlock is a
// multiple of the chunks per row), so its eight coarse values are loaded once
// per cube.  All of a cube's loads (O_f rows, gates) are issued before any
// arithmetic: the gate loads are scattered (one 2-byte value per 80-byte row of
// the [B, N, H] layout), and issuing them one row at a time behind each O_f
// load left too few bytes in flight to cover HBM latency.  The registers that
// hold them allow kCombinePerSm resident blocks per SM, and the grid is sized to
// exactly that many: a grid-stride grid larger than the resident blocks would
// leave its last blocks to run alone after the first wave.
constexpr int kCombinePerSm = 5;

template <int D>
__global__ void __launch_bounds__(kBlock, kCombinePerSm) combine_kernel(Dims d, const float* __restrict__ o_coarse,
                                                                        const uint16_t* __restrict__ o_fine,
                                                                        const uint16_t* __restrict__ g_coarse,
                                                                        const uint16_t* __restrict__ g_fine,
                                                                        uint16_t* __restrict__ o_tiled) {
    constexpr int CH = D / 8;
    constexpr int PER = kCubeTokens * CH / kBlock;
    constexpr int ROWS = kBlock / CH;   // rows covered by one pass of the block
    static_assert(kBlock % CH == 0, "a thread's column chunk must stay fixed across its rows");
    const int64_t total = static_cast<int64_t>(d.B) * d.H * d.C;
    const uint4* of = reinterpret_cast<const uint4*>(o_fine);
    uint4* out = reinterpret_cast<uint4*>(o_tiled);
    const int j = threadIdx.x % CH, o0 = threadIdx.x / CH;
    for (int64_t task = blockIdx.x; task < total; task += gridDim.x) {
        const CubeTask t = decode_task(task, d);
        const int64_t row0 = t.bh * d.Npad + static_cast<int64_t>(t.c) * kCubeTokens;
        const float4* oc = reinterpret_cast<const float4*>(o_coarse + (t.bh * d.C + t.c) * D);
        int n[PER];   // token of each row, -1 for padding (below 2^30: at most 2^24 cubes)
        uint4 f[PER];
        float gc[PER], gf[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) n[i] = static_cast<int>(token_of(d, t, o0 + i * ROWS));
#pragma unroll
        for (int i = 0; i < PER; ++i)
            f[i] = n[i] >= 0 ? __ldcs(of + (row0 + o0 + i * ROWS) * CH + j) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int64_t g = (static_cast<int64_t>(t.b) * d.N + (n[i] >= 0 ? n[i] : 0)) * d.H + t.h;
            gc[i] = g_coarse && n[i] >= 0 ? __uint_as_float(static_cast<uint32_t>(g_coarse[g]) << 16) : 0.f;
            gf[i] = g_fine && n[i] >= 0 ? __uint_as_float(static_cast<uint32_t>(g_fine[g]) << 16) : 1.f;
        }
        const float4 c0 = __ldg(oc + 2 * j), c1 = __ldg(oc + 2 * j + 1);
        const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            uint4 r = make_uint4(0u, 0u, 0u, 0u);
            if (n[i] >= 0) {
                const uint32_t fw[4] = {f[i].x, f[i].y, f[i].z, f[i].w};
                uint32_t ow[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float lo = fmaf(gc[i], cv[2 * e], gf[i] * __uint_as_float(fw[e] << 16));
                    const float hi = fmaf(gc[i], cv[2 * e + 1], gf[i] * __uint_as_float(fw[e] & 0xFFFF0000u));
                    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
                    ow[e] = *reinterpret_cast<const uint32_t*>(&p);
                }
                r = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
            out[(row0 + o0 + i * ROWS) * CH + j] = r;
        }
    }
}

int grid_for(int64_t tasks, int per_sm) {
    const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
    return static_cast<int>(tasks < cap ? (tasks > 0 ? tasks : 1) : cap);
}

}  // namespace

cudaError_t launch_tile(const Dims& d, const Bf16Triple& t, cudaStream_t s) {
    const int grid = grid_for(static_cast<int64_t>(d.B) * d.H * d.C * t.count, kLayoutPerSm);
    if (d.D == 128) tile_kernel<128><<<grid, kBlock, 0, s>>>(d, t);
    else tile_kernel<64><<<grid, kBlock, 0, s>>>(d, t);
    return cudaGetLastError();
}

cudaError_t launch_untile(const Dims& d, const uint16_t* xt, uint16_t* x, cudaStream_t s) {
    const int grid = grid_for(static_cast<int64_t>(d.B) * d.H * d.C, kLayoutPerSm);
    if (d.D == 128) untile_kernel<128><<<grid, kBlock, 0, s>>>(d, xt, x);
    else untile_kernel<64><<<grid, kBlock, 0, s>>>(d, xt, x);
    return cudaGetLastError();
}

cudaError_t launch_pool(const Dims& d, const uint16_t* const* xt, float* const* xbar, int count, cudaStream_t s) {
    PoolIO io{};
    for (int i = 0; i < count; ++i) {
        io.src[i] = xt[i];
        io.dst[i] = xbar[i];
    }
    io.count = count;
    const int64_t warps = static_cast<int64_t>(d.B) * d.H * d.C * count;
    const int grid = grid_for((warps + 7) / 8, 8);
    if (d.D == 128) pool_kernel<128><<<grid, kBlock, 0, s>>>(d, io);
    else pool_kernel<64><<<grid, kBlock, 0, s>>>(d, io);
    return cudaGetLastError();
}

cudaError_t launch_split_parts(const Dims& d, const float* const* x, uint16_t* const* parts, int count,
                               cudaStream_t s) {
    if (count < 1 || count > 3) return cudaErrorInvalidValue;
    SplitIO io{};
    for (int t = 0; t < count; ++t) {
        io.x[t] = x[t];
        io.parts[t] = parts[t];
    }
    io.count = count;
    const int64_t groups = static_cast<int64_t>(d.B) * d.H * d.C * d.D / 8;
    const int grid = grid_for((groups * count + kBlock - 1) / kBlock, 8);
    split_parts_kernel<<<grid, kBlock, 0, s>>>(groups, io);
    return cudaGetLastError();
}

cudaError_t launch_pool_tokens(const Dims& d, const uint16_t* const* x, float* const* xbar, int count,
                               cudaStream_t s, uint16_t* const* parts) {
    PoolIO io{};
    for (int i = 0; i < count; ++i) {
        io.src[i] = x[i];
        io.dst[i] = xbar ? xbar[i] : nullptr;
        io.parts[i] = parts ? parts[i] : nullptr;
    }
    io.count = count;
    const int64_t cubes = static_cast<int64_t>(count) * d.B * d.C;
    const int slots = (d.H * (d.D / 8) + kPoolThreads - 1) / kPoolThreads;
    if (cubes > 0x7FFFFFFFll || slots > 65535) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>(cubes), static_cast<unsigned>(slots));
    if (d.D == 128) pool_tokens_kernel<128><<<grid, kPoolThreads, 0, s>>>(d, io);
    else pool_tokens_kernel<64><<<grid, kPoolThreads, 0, s>>>(d, io);
    return cudaGetLastError();
}

namespace {
__global__ void gather_heads_kernel(const uint16_t* __restrict__ src, int64_t rows, int H, int h0, int hg,
                                    uint16_t* __restrict__ dst) {
    const int64_t total = rows * hg;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / hg;
        dst[i] = src[r * H + h0 + (i - r * hg)];
    }
}
}  // namespace

cudaError_t launch_gather_heads(const uint16_t* src, int64_t rows, int H, int h0, int hg, uint16_t* dst,
                                cudaStream_t s) {
    if (rows <= 0 || hg <= 0) return cudaSuccess;
    const int grid = grid_for((rows * hg + kBlock - 1) / kBlock, 8);
    gather_heads_kernel<<<grid, kBlock, 0, s>>>(src, rows, H, h0, hg, dst);
    return cudaGetLastError();
}

cudaError_t launch_combine(const Dims& d, const float* o_coarse, const uint16_t* o_fine, const uint16_t* g_coarse,
                           const uint16_t* g_fine, uint16_t* o_tiled, cudaStream_t s) {
    const int grid = grid_for(static_cast<int64_t>(d.B) * d.H * d.C, kCombinePerSm);
    if (d.D == 128) combine_kernel<128><<<grid, kBlock, 0, s>>>(d, o_coarse, o_fine, g_coarse, g_fine, o_tiled);
    else combine_kernel<64><<<grid, kBlock, 0, s>>>(d, o_coarse, o_fine, g_coarse, g_fine, o_tiled);
    return cudaGetLastError();
}

}  // namespace vsa
