// Pre-attention pass: RMSNorm of each token's Q and K over all H*D channels,
// then the 3D rotary position embedding, in one read and one write of Q and K.
//
// Sources: WorldFoundry inference-optimisation guide (openenvision.org,
// "推理优化"), table of exact Wan kernels, row "fused_rope" (3D RoPE as one
// kernel; under sequence parallelism the kernel takes the rank's token offset
// and the padding; fp32 or fp64 rotation); Wan2.2 real-time inference teardown
// (zharfai.com), section "Fusion targets launch overhead and memory" (the Q/K
// normalisation read once, reduced and scaled in registers, written once).
//
// Layout [B, n_tokens, H, D] bf16; row r = b * n_tokens + i is global token
// token_offset + i, whose coordinates follow n = (t*X + x)*Y + y.  The D/2
// channel pairs (2i, 2i+1) of each head form three bands for t, x and y (x and
// y floor(D/6) pairs each, t the rest); pair j of a band of P pairs turns by
// pos * theta^(-j/P).  Rows past the N real tokens (shard padding) are zeros.
//
// One warp per token, Q then K: lane L handles the 16-byte chunks L + 32c
// of the row.  A first pass sums the squares (warp reduction in fp32); the
// second reads the row again, from L1 or L2, and writes the result, so HBM
// sees one read and one write.  Each turn angle is formed and reduced to
// [-pi, pi] in fp64 (the frequencies come from the host, in fp64); its sine
// and cosine are taken in fp32 and applied in fp32; the result is rounded to
// bf16 once.  Because 32 is a multiple of D/8, a lane's chunks all sit at the
// same channel offset of their heads, so a lane needs the same four pairs'
// angles for every chunk.
#include <cmath>

#include <cuda_bf16.h>

#include "vsa_internal.h"

namespace vsa {
namespace {

constexpr int kWarps = 8;

struct NormRopeParams {
    const uint16_t* in[2];    // q, k
    uint16_t* out[2];         // q_out, k_out (may equal in[])
    const uint16_t* w[2];     // RMSNorm weights [H*D] or null
    int64_t rows;             // B * n_tokens
    int64_t n_tokens;
    int64_t token_offset;
    int64_t N;
    int X, Y;
    int HD;                   // H * D
    int chunks;               // HD / 8
    float eps;
    double freq[64];          // turn per position step of each rotation pair (D/2 <= 64)
    int axis[64];             // 0: t, 1: x, 2: y
};

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_rn(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

template <int D, int CPL>
__global__ void __launch_bounds__(kWarps * 32) norm_rope_kernel(const NormRopeParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t warp_global = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * kWarps;
    // this lane's four rotation pairs (the same for every chunk)
    const int pair0 = 4 * (lane % (D / 8));
    const float inv_hd = 1.0f / static_cast<float>(p.HD);
    for (int64_t r = warp_global; r < p.rows; r += warp_stride) {
        const int64_t i = r % p.n_tokens;
        const int64_t g = p.token_offset + i;
        const bool real = g < p.N;
        float cs[4], sn[4];
        if (real) {
            const int64_t xy = static_cast<int64_t>(p.X) * p.Y;
            const double pt = static_cast<double>(g / xy), px = static_cast<double>((g / p.Y) % p.X),
                         py = static_cast<double>(g % p.Y);
            constexpr double kTwoPi = 6.283185307179586476925286766559;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int ax = p.axis[pair0 + e];
                double ang = (ax == 0 ? pt : ax == 1 ? px : py) * p.freq[pair0 + e];
                ang -= kTwoPi * rint(ang / kTwoPi);
                __sincosf(static_cast<float>(ang), &sn[e], &cs[e]);
            }
        }
#pragma unroll 1
        for (int tsr = 0; tsr < 2; ++tsr) {
            const uint4* src = reinterpret_cast<const uint4*>(p.in[tsr]) + r * p.chunks;
            uint4* dst = reinterpret_cast<uint4*>(p.out[tsr]) + r * p.chunks;
            if (!real) {
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    const int j = lane + 32 * c;
                    if (j < p.chunks) dst[j] = make_uint4(0u, 0u, 0u, 0u);
                }
                continue;
            }
            // pass 1: the row's sum of squares (the row stays in L1 / L2 for pass 2)
            float ss = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const int j = lane + 32 * c;
                const uint4 v = j < p.chunks ? __ldg(src + j) : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t x4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float a = bf16_lo(x4[e]), b = bf16_hi(x4[e]);
                    ss = fmaf(a, a, ss);
                    ss = fmaf(b, b, ss);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
            const float inv = 1.0f / sqrtf(ss * inv_hd + p.eps);
            const uint4* wv = reinterpret_cast<const uint4*>(p.w[tsr]);
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                const int j = lane + 32 * c;
                if (j >= p.chunks) continue;
                const uint4 v = __ldg(src + j);   // pass 2: normalise, weight, rotate
                const uint32_t x4[4] = {v.x, v.y, v.z, v.w};
                uint32_t w4[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};   // bf16 1.0 pairs
                if (wv != nullptr) {
                    const uint4 ww = __ldg(wv + j);
                    w4[0] = ww.x; w4[1] = ww.y; w4[2] = ww.z; w4[3] = ww.w;
                }
                uint32_t o4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float a = bf16_lo(x4[e]) * inv * bf16_lo(w4[e]);
                    const float b = bf16_hi(x4[e]) * inv * bf16_hi(w4[e]);
                    o4[e] = pack_rn(a * cs[e] - b * sn[e], a * sn[e] + b * cs[e]);
                }
                dst[j] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
    }
}

template <int D, int CPL>
cudaError_t launch_cpl(const NormRopeParams& p, cudaStream_t s) {
    const int64_t blocks_needed = (p.rows + kWarps - 1) / kWarps;
    const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
    const int blocks = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
    norm_rope_kernel<D, CPL><<<blocks, kWarps * 32, 0, s>>>(p);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const NormRopeParams& p, cudaStream_t s) {
    const int cpl = (p.chunks + 31) / 32;
    if (cpl <= 2) return launch_cpl<D, 2>(p, s);
    if (cpl <= 4) return launch_cpl<D, 4>(p, s);
    if (cpl <= 8) return launch_cpl<D, 8>(p, s);
    if (cpl <= 12) return launch_cpl<D, 12>(p, s);
    if (cpl <= 16) return launch_cpl<D, 16>(p, s);
    if (cpl <= 20) return launch_cpl<D, 20>(p, s);
    if (cpl <= 24) return launch_cpl<D, 24>(p, s);
    return launch_cpl<D, 32>(p, s);
}

}  // namespace

cudaError_t launch_norm_rope(const Dims& d, const NormRopeArgs& a, cudaStream_t s) {
    if (a.n_tokens == 0 || d.B == 0) return cudaSuccess;
    if (static_cast<int64_t>(d.H) * d.D > kNormRopeMaxHD) return cudaErrorInvalidValue;
    NormRopeParams p{};
    p.in[0] = a.q;
    p.in[1] = a.k;
    p.out[0] = a.q_out;
    p.out[1] = a.k_out;
    p.w[0] = a.w_q;
    p.w[1] = a.w_k;
    p.rows = static_cast<int64_t>(d.B) * a.n_tokens;
    p.n_tokens = a.n_tokens;
    p.token_offset = a.token_offset;
    p.N = d.N;
    p.X = d.X;
    p.Y = d.Y;
    p.HD = d.H * d.D;
    p.chunks = p.HD / 8;
    p.eps = a.eps;
    const int pxy = d.D / 6, pt = d.D / 2 - 2 * pxy;
    for (int pr = 0; pr < d.D / 2; ++pr) {
        int j, P;
        if (pr < pt) {
            p.axis[pr] = 0; j = pr; P = pt;
        } else if (pr < pt + pxy) {
            p.axis[pr] = 1; j = pr - pt; P = pxy;
        } else {
            p.axis[pr] = 2; j = pr - pt - pxy; P = pxy;
        }
        p.freq[pr] = std::pow(static_cast<double>(a.theta), -static_cast<double>(j) / static_cast<double>(P));
    }
    return d.D == 128 ? launch_d<128>(p, s) : launch_d<64>(p, s);
}

}  // namespace vsa
