// Host-side declarations shared by the library's translation units.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "vsa.h"

namespace vsa {

constexpr int kCube = 4;
constexpr int kCubeTokens = 64;

// Sizes derived from a vsa_shape (see include/vsa.h for the layouts).
struct Dims {
    int B, H, D;
    int T, X, Y;        // token grid
    int Ct, Cx, Cy;     // cubes per axis
    int C;              // cubes
    int64_t N;          // real tokens per batch element
    int64_t Npad;       // padded tokens per batch element = C * 64
    int64_t rows;       // B * H * Npad rows of the tiled layout
};

// Records `message` as this thread's vsa_last_error() text and returns `st`.
vsa_status set_last_error(vsa_status st, const char* message);

// Number of SMs of the current device (cached per device).
int sm_count();

// Watchdog word of the current device (device address, cached per device).
int* status_word();

// Upper bound on any device-side wait, in nanoseconds.
constexpr uint64_t kWaitLimitNs = 4000000000ull;

// ---- launches; each returns the launch error (cudaSuccess when enqueued)
struct Bf16Triple {
    const uint16_t* src[3];
    uint16_t* dst[3];
    int count;
};

cudaError_t launch_tile(const Dims& d, const Bf16Triple& t, cudaStream_t s);
cudaError_t launch_untile(const Dims& d, const uint16_t* xt, uint16_t* x, cudaStream_t s);
cudaError_t launch_pool(const Dims& d, const uint16_t* const* xt, float* const* xbar, int count, cudaStream_t s);
cudaError_t launch_combine(const Dims& d, const float* o_coarse, const uint16_t* o_fine, const uint16_t* g_coarse,
                           const uint16_t* g_fine, uint16_t* o_tiled, cudaStream_t s);
cudaError_t launch_topk(const Dims& d, const float* scores, int k, int32_t* idx, cudaStream_t s);

// Largest C whose rows the selection holds in registers; up to it, top-k can
// also emit each row's work-order signature (uint64 [B, H, C]) in the same
// pass, and launch_group_sort turns those into the order launch_group gives.
constexpr int kTopkRegMaxC = 2048;
cudaError_t launch_topk_sig(const Dims& d, const float* scores, int k, int32_t* idx, uint64_t* sig, cudaStream_t s);

// Work order of the fine stage from the coarse scores (C <= kGroupMaxC).
constexpr int kGroupMaxC = 4096;
cudaError_t launch_group(const Dims& d, const float* scores, int32_t* order, cudaStream_t s);
cudaError_t launch_group_sort(const Dims& d, const uint64_t* sig, int32_t* order, cudaStream_t s);

// Fine stage.  Modes:
//  kFineTiled       - q/k/v tiled [B, H, Npad, D]; out = tiled O_f (+ lse when non-null);
//  kFineCubesFused  - q/k/v in the projection layout [B, N, H, D], cubes gathered by TMA;
//                     out = g_c * O_c[cube] + g_f * O_f in [B, N, H, D] (o_coarse/g_coarse/g_fine
//                     may be null: no coarse term / gate 1);
//  kFineTokensFused - as kFineCubesFused but attending over blocks of 64 consecutive real
//                     tokens (dense attention only: idx must be null).
// `order` (may be null) is a per-head permutation of the query cubes; groups
// of four consecutive entries share one key/value stream.  Returns
// cudaErrorInvalidValue (with *why set) when a tensor map cannot be encoded.
enum FineMode : int { kFineTiled = 0, kFineCubesFused = 1, kFineTokensFused = 2 };

struct FineArgs {
    int mode;
    const uint16_t *q, *k, *v;
    const int32_t* idx;     // [B, H, C, k] or null (every block)
    int k_sel;
    const int32_t* order;   // [B, H, C] or null
    const void* steps;      // precomputed steps (launch_schedule) or null: the kernel walks the selection
    int* overflow;          // caller's device word: cleared, raised by the one-tile kernel on overflow,
                            // read by the re-run (required with steps)
    float scale;
    uint16_t* out;
    float* lse;             // kFineTiled only
    const float* o_coarse;  // fused modes only
    const uint16_t* g_coarse;
    const uint16_t* g_fine;
};

cudaError_t launch_fine(const Dims& d, const FineArgs& a, cudaStream_t s, const char** why);

// Precomputed steps of the fine stage's work items for a sparse selection
// (idx [B, H, C, k], order [B, H, C] or null): a work item is a pair of query
// cubes (consecutive entries of the order), one 128-row tile; 8 bytes per
// step, at most k steps per item.  Cube indices travel in 16 bits, so the
// fine kernel takes steps for C <= kScheduleMaxC; launch_schedule also needs
// its shared memory (four warps x (C/8 + 1 + 2k) words) within 48 KB.
constexpr int kTileGroup = 2;
constexpr int kScheduleMaxC = 65534;
inline int64_t schedule_stride(int k) { return k; }
size_t schedule_bytes(const Dims& d, int k);
bool schedule_supported(const Dims& d, int k);
cudaError_t launch_schedule(const Dims& d, const int32_t* idx, int k, const int32_t* order, void* steps,
                            cudaStream_t s);

// Pre-attention pass: Q/K RMSNorm over H*D channels, then 3D RoPE, on the
// [B, n_tokens, H, D] rows of global tokens [token_offset, token_offset + n_tokens).
struct NormRopeArgs {
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* w_q;   // [H*D] or null (1)
    const uint16_t* w_k;
    uint16_t* q_out;       // may equal q
    uint16_t* k_out;       // may equal k
    float eps, theta;
    int64_t token_offset, n_tokens;
};
constexpr int kNormRopeMaxHD = 8192;   // a lane holds at most 32 16-byte chunks of a row
cudaError_t launch_norm_rope(const Dims& d, const NormRopeArgs& a, cudaStream_t s);

// Cube mean-pool read straight from the projection layout [B, N, H, D]
// (same fp32 summation order as launch_pool on the tiled tensor).
// dst[r][j] = src[r][h0 + j] for r < rows, j < hg: a head range of per-(token, head) values [rows, H]
// (the gates) gathered into [rows, hg].
cudaError_t launch_gather_heads(const uint16_t* src, int64_t rows, int H, int h0, int hg, uint16_t* dst,
                                cudaStream_t s);

// xbar (float32 means) and parts (the means split into three bf16 parts, [3][B*H][C][D] per tensor) may
// each be null.
cudaError_t launch_pool_tokens(const Dims& d, const uint16_t* const* x, float* const* xbar, int count,
                               cudaStream_t s, uint16_t* const* parts = nullptr);

// The coarse stage on the tensor cores: float32 pooled vectors carried as three bf16 parts.
// launch_split_parts: count (1-3) tensors, float32 [B, H, C, D] -> parts [3][B*H][C][D]
// (split_parts_elems(d) uint16 each), in one launch.
size_t split_parts_elems(const Dims& d);
cudaError_t launch_split_parts(const Dims& d, const float* const* x, uint16_t* const* parts, int count,
                               cudaStream_t s);
// scores [B, H, C, C] = scale * qbar kbar^T from the parts of qbar and kbar (six partial products per
// channel step), and, when stats is non-null, stats [B, H, C] float2: each score row's maximum m and
// 1 / sum(exp(s - m)); *why set when a tensor map cannot be encoded.
cudaError_t launch_coarse_scores_mma(const Dims& d, const uint16_t* q_parts, const uint16_t* k_parts, float scale,
                                     float* scores, float* stats, cudaStream_t s, const char** why);
// o_coarse [B, H, C, D] = softmax(scores) vbar from the row statistics and the parts of vbar.
cudaError_t launch_coarse_pv_mma(const Dims& d, const float* scores, const float* stats, const uint16_t* v_parts,
                                 float* o_coarse, cudaStream_t s, const char** why);

cudaError_t launch_wait_probe(uint64_t limit_ns, cudaStream_t s);

}  // namespace vsa
