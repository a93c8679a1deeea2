// C ABI of the library (declared in include/vsa.h): argument checks, error
// reporting and the orchestration of the kernels of one attention call.
// Every argument check runs on the host before anything is enqueued.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "vsa_internal.h"

namespace vsa {
namespace {

thread_local char g_last_error[256] = "";

vsa_status fail(vsa_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

vsa_status cuda_fail(cudaError_t e, const char* where) {
    return fail(VSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr int64_t kMaxRows = (int64_t{1} << 31) - 1;

vsa_status make_dims(const vsa_shape* s, Dims* d) {
    if (!s) return fail(VSA_ERR_INVALID_ARGUMENT, "shape is NULL");
    if (s->batch < 1 || s->heads < 1 || s->grid_t < 1 || s->grid_h < 1 || s->grid_w < 1)
        return fail(VSA_ERR_INVALID_ARGUMENT, "batch, heads and grid dims must be >= 1 (got B=%d H=%d grid=%dx%dx%d)",
                    s->batch, s->heads, s->grid_t, s->grid_h, s->grid_w);
    if (s->head_dim < 1) return fail(VSA_ERR_INVALID_ARGUMENT, "head_dim must be >= 1 (got %d)", s->head_dim);
    if (s->head_dim != 64 && s->head_dim != 128)
        return fail(VSA_ERR_UNSUPPORTED, "head_dim %d is not supported (64 or 128)", s->head_dim);
    d->B = s->batch;
    d->H = s->heads;
    d->D = s->head_dim;
    d->T = s->grid_t;
    d->X = s->grid_h;
    d->Y = s->grid_w;
    d->Ct = (d->T + kCube - 1) / kCube;
    d->Cx = (d->X + kCube - 1) / kCube;
    d->Cy = (d->Y + kCube - 1) / kCube;
    const int64_t C = static_cast<int64_t>(d->Ct) * d->Cx * d->Cy;
    if (C > (int64_t{1} << 24)) return fail(VSA_ERR_INVALID_ARGUMENT, "grid too large (%lld cubes)", (long long)C);
    d->C = static_cast<int>(C);
    d->N = static_cast<int64_t>(d->T) * d->X * d->Y;
    d->Npad = C * kCubeTokens;
    d->rows = static_cast<int64_t>(d->B) * d->H * d->Npad;
    if (static_cast<int64_t>(d->B) * d->H > 65535)
        return fail(VSA_ERR_UNSUPPORTED, "batch*heads = %lld exceeds 65535", (long long)d->B * d->H);
    if (d->rows > kMaxRows)
        return fail(VSA_ERR_INVALID_ARGUMENT, "B*H*Npad = %lld rows exceeds 2^31-1", (long long)d->rows);
    return VSA_OK;
}

vsa_status need_ptr(const void* p, const char* name) {
    if (!p) return fail(VSA_ERR_INVALID_ARGUMENT, "%s is NULL", name);
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return fail(VSA_ERR_MISALIGNED, "%s is not 16-byte aligned", name);
    return VSA_OK;
}

vsa_status opt_ptr(const void* p, const char* name) { return p ? need_ptr(p, name) : VSA_OK; }

struct Range {
    const void* p;
    size_t bytes;
    const char* name;
};

bool overlap(const Range& a, const Range& b) {
    if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
    return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

vsa_status check_disjoint(std::initializer_list<Range> ins, std::initializer_list<Range> outs) {
    for (const Range& o : outs) {
        for (const Range& i : ins)
            if (overlap(o, i)) return fail(VSA_ERR_INVALID_ARGUMENT, "output %s overlaps input %s", o.name, i.name);
        for (const Range& o2 : outs)
            if (&o2 != &o && overlap(o, o2)) return fail(VSA_ERR_INVALID_ARGUMENT, "outputs %s and %s overlap", o.name, o2.name);
    }
    return VSA_OK;
}

// The kernels are built for sm_100a only.
vsa_status check_device() {
    static int checked[64] = {};   // 0 unknown, 1 ok, 2 unsupported
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev >= 0 && dev < 64 && checked[dev] == 1) return VSA_OK;
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute");
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute");
    if (major != 10 || minor != 0) {
        if (dev >= 0 && dev < 64) checked[dev] = 2;
        return fail(VSA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library runs on sm_100a only", dev, major, minor);
    }
    if (dev >= 0 && dev < 64) checked[dev] = 1;
    return VSA_OK;
}

cudaStream_t as_stream(vsa_stream_t s) { return static_cast<cudaStream_t>(s); }

// vsa_forward_host's copy streams on the current device (0: host->device, 1: device->host), created
// on first use and kept for the life of the process.
vsa_status lib_stream(int which, cudaStream_t* out) {
    static std::mutex mu;
    static cudaStream_t streams[64][2] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(VSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (streams[dev][which] == nullptr) {
        if ((e = cudaStreamCreateWithFlags(&streams[dev][which], cudaStreamNonBlocking)) != cudaSuccess) {
            streams[dev][which] = nullptr;
            return cuda_fail(e, "cudaStreamCreateWithFlags");
        }
    }
    *out = streams[dev][which];
    return VSA_OK;
}

// vsa_forward_host: head groups per call (the copies of one overlap the compute of another)
constexpr int kHostGroups = 8;

// The head ranges [h0, h0 + hn) of one vsa_forward_host call.  Every upload but the first overlaps
// compute, so the call takes about all its uploads plus the last group's compute and download: with 27 or
// more heads the last three groups hold 4, 2 and 1 heads and the others split the rest evenly, largest
// first (Wan's 40 heads: 7 7 7 6 6 4 2 1); with fewer heads, groups of ceil(H / kHostGroups).  Copies of
// 256-byte rows (one head) still run at about 52 GB/s against 55 for whole rows, measured on B200.
struct HostPlan {
    int n = 0, largest = 0;
    int h0[kHostGroups] = {}, hn[kHostGroups] = {};
};

HostPlan host_plan(int H) {
    HostPlan pl;
    if (H >= 27) {
        const int rest = H - 7, nr = kHostGroups - 3;
        for (int i = 0; i < nr; ++i) pl.hn[pl.n++] = rest / nr + (i < rest % nr ? 1 : 0);
        pl.hn[pl.n++] = 4;
        pl.hn[pl.n++] = 2;
        pl.hn[pl.n++] = 1;
    } else {
        const int hg = (H + kHostGroups - 1) / kHostGroups;
        for (int h = 0; h < H; h += hg) pl.hn[pl.n++] = H - h < hg ? H - h : hg;
    }
    for (int i = 0, h = 0; i < pl.n; h += pl.hn[i], ++i) {
        pl.h0[i] = h;
        if (pl.hn[i] > pl.largest) pl.largest = pl.hn[i];
    }
    return pl;
}

// Events of one vsa_forward_host call, destroyed when it returns (CUDA keeps a recorded event
// alive until the work it marks is done).
struct EventSet {
    cudaEvent_t e[2 * kHostGroups + 2] = {};
    int n = 0;
    cudaError_t create(int count) {
        for (; n < count; ++n) {
            const cudaError_t r = cudaEventCreateWithFlags(&e[n], cudaEventDisableTiming);
            if (r != cudaSuccess) return r;
        }
        return cudaSuccess;
    }
    cudaEvent_t operator[](int i) const { return e[i]; }
    ~EventSet() {
        for (int i = 0; i < n; ++i) cudaEventDestroy(e[i]);
    }
};

size_t tiled_bytes(const Dims& d) { return static_cast<size_t>(d.rows) * d.D * 2; }
size_t token_bytes(const Dims& d) { return static_cast<size_t>(d.B) * d.N * d.H * d.D * 2; }
size_t gate_bytes(const Dims& d) { return static_cast<size_t>(d.B) * d.N * d.H * 2; }
size_t pooled_bytes(const Dims& d) { return static_cast<size_t>(d.B) * d.H * d.C * d.D * 4; }
size_t score_bytes(const Dims& d) { return static_cast<size_t>(d.B) * d.H * d.C * d.C * 4; }
size_t idx_bytes(const Dims& d, int k) { return static_cast<size_t>(d.B) * d.H * d.C * k * 4; }
size_t order_bytes(const Dims& d) { return static_cast<size_t>(d.B) * d.H * d.C * 4; }

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Workspace of vsa_forward: q/k/v parts | row stats | o_coarse | scores | idx | order | sig | steps |
// overflow.  Q, K and V are read in the caller's [B, N, H, D] layout (the fine stage gathers cubes with
// TMA), so no tiled copies are kept; the pooled vectors are kept only as their three bf16 parts (the
// coarse stage's tensor-core operands).  With every cube selected the fine stage is dense attention
// and needs none of it; the coarse buffers are then used only when a coarse gate is given.
struct Carve {
    uint16_t *qp, *kp, *vp;   // the pooled q, k, v as three bf16 parts each
    float* stats;             // per score row: maximum and 1 / sum of exp
    float *oc, *scores;
    int32_t* idx;
    int32_t* order;
    uint64_t* sig;   // work-order signatures, when top-k computes them (C <= kTopkRegMaxC)
    void* steps;     // the fine stage's precomputed steps (when schedule_supported)
    int* overflow;   // the fine stage's overflow word
    size_t bytes;
};

size_t parts_bytes(const Dims& d) { return split_parts_elems(d) * 2u; }
size_t stats_bytes(const Dims& d) { return static_cast<size_t>(d.B) * d.H * d.C * 8u; }

Carve carve(const Dims& d, int k, bool coarse_gate, void* ws) {
    Carve c{};
    uint8_t* b = static_cast<uint8_t*>(ws);
    size_t off = 0;
    auto take = [&](size_t n) {
        uint8_t* p = b ? b + off : nullptr;
        off += up(n);
        return p;
    };
    const bool sparse = k < d.C;
    if (sparse || coarse_gate) {
        c.qp = reinterpret_cast<uint16_t*>(take(parts_bytes(d)));
        c.kp = reinterpret_cast<uint16_t*>(take(parts_bytes(d)));
        c.vp = reinterpret_cast<uint16_t*>(take(parts_bytes(d)));
        c.stats = reinterpret_cast<float*>(take(stats_bytes(d)));
        c.oc = reinterpret_cast<float*>(take(pooled_bytes(d)));
        c.scores = reinterpret_cast<float*>(take(score_bytes(d)));
    }
    if (sparse) {
        c.idx = reinterpret_cast<int32_t*>(take(idx_bytes(d, k)));
        c.order = reinterpret_cast<int32_t*>(take(order_bytes(d)));
        if (d.C <= kTopkRegMaxC) c.sig = reinterpret_cast<uint64_t*>(take(2 * order_bytes(d)));
        if (schedule_supported(d, k)) c.steps = take(schedule_bytes(d, k));
    }
    c.overflow = reinterpret_cast<int*>(take(2 * sizeof(int)));
    c.bytes = off > kAlign ? off : kAlign;
    return c;
}

vsa_status check_scale(float scale) {
    if (!(scale > 0.f) || !std::isfinite(scale))
        return fail(VSA_ERR_INVALID_ARGUMENT, "scale must be finite and > 0 (got %g)", static_cast<double>(scale));
    return VSA_OK;
}

vsa_status check_k(const Dims& d, int32_t k) {
    if (k < 1 || k > d.C) return fail(VSA_ERR_INVALID_ARGUMENT, "top-k %d outside [1, C=%d]", k, d.C);
    return VSA_OK;
}

#define VSA_TRY(expr)                      \
    do {                                   \
        const vsa_status st_ = (expr);     \
        if (st_ != VSA_OK) return st_;     \
    } while (0)

#define VSA_CUDA(expr, where)                               \
    do {                                                    \
        const cudaError_t e_ = (expr);                      \
        if (e_ != cudaSuccess) return cuda_fail(e_, where); \
    } while (0)

// The fused fine stage once the arguments are checked: cube gathers when a
// selection is given, blocks of consecutive real tokens for dense attention.
vsa_status run_fine_fused(const Dims& d, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          const int32_t* idx, int topk, const int32_t* order, const void* steps, float scale,
                          const float* o_coarse, const uint16_t* gc, const uint16_t* gf, uint16_t* out,
                          int* overflow, cudaStream_t s) {
    FineArgs a{};
    a.overflow = overflow;
    a.mode = idx ? kFineCubesFused : kFineTokensFused;
    a.q = q;
    a.k = k;
    a.v = v;
    a.idx = idx;
    a.k_sel = topk;
    a.order = idx ? order : nullptr;
    a.steps = idx ? steps : nullptr;
    a.scale = scale;
    a.out = out;
    a.o_coarse = o_coarse;
    a.g_coarse = o_coarse ? gc : nullptr;
    a.g_fine = gf;
    const char* why = nullptr;
    cudaError_t e = launch_fine(d, a, s, &why);
    if (e != cudaSuccess) return why ? fail(VSA_ERR_CUDA, "%s", why) : cuda_fail(e, "fine launch");
    return VSA_OK;
}

// Body of vsa_forward once the arguments are checked.
//  * top-k < C:  pool (Q, K, V read in place) -> coarse -> top-k -> work order
//                -> fine with cube gathers and the merge + untiling in its epilogue;
//  * top-k == C: every cube is selected, so the fine stage is dense attention
//                over the real tokens (blocks of 64 consecutive tokens, no
//                padding); pool -> coarse run only when a coarse gate is given.
vsa_status run_forward(const Dims& d, const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* gc,
                       const uint16_t* gf, int topk, float scale, void* ws, uint16_t* out, cudaStream_t s) {
    const bool sparse = topk < d.C;
    const Carve c = carve(d, topk, gc != nullptr, ws);
    const char* why = nullptr;
    if (sparse || gc != nullptr) {
        // pooled q, k, v straight into their bf16 parts, then the scores on the tensor cores
        const uint16_t* pin[3] = {q, k, v};
        uint16_t* parts[3] = {c.qp, c.kp, c.vp};
        // v-bar feeds only the coarse output, which only the coarse gate uses: without it v is not pooled
        VSA_CUDA(launch_pool_tokens(d, pin, nullptr, gc != nullptr ? 3 : 2, s, parts), "pool launch");
        // the softmax statistics of the score rows are needed only for the coarse output
        const cudaError_t e =
            launch_coarse_scores_mma(d, c.qp, c.kp, scale, c.scores, gc != nullptr ? c.stats : nullptr, s, &why);
        if (e != cudaSuccess) return why ? fail(VSA_ERR_CUDA, "%s", why) : cuda_fail(e, "coarse launch");
    }
    const int32_t* order = nullptr;
    if (sparse) {
        if (d.C <= kTopkRegMaxC && d.C <= kGroupMaxC) {
            // one pass over the scores gives the selection and the work-order keys
            VSA_CUDA(launch_topk_sig(d, c.scores, topk, c.idx, c.sig, s), "topk launch");
            VSA_CUDA(launch_group_sort(d, c.sig, c.order, s), "group launch");
            order = c.order;
        } else {
            VSA_CUDA(launch_topk(d, c.scores, topk, c.idx, s), "topk launch");
            if (d.C <= kGroupMaxC) {
                VSA_CUDA(launch_group(d, c.scores, c.order, s), "group launch");
                order = c.order;
            }
        }
    }
    // the coarse output (softmax(scores) x V-bar) is used only by the merge, and only with a coarse gate
    if (gc != nullptr) {
        const cudaError_t e = launch_coarse_pv_mma(d, c.scores, c.stats, c.vp, c.oc, s, &why);
        if (e != cudaSuccess) return why ? fail(VSA_ERR_CUDA, "%s", why) : cuda_fail(e, "coarse launch");
    }
    const void* steps = nullptr;
    if (sparse && c.steps != nullptr) {
        VSA_CUDA(launch_schedule(d, c.idx, topk, order, c.steps, s), "schedule launch");
        steps = c.steps;
    }
    return run_fine_fused(d, q, k, v, sparse ? c.idx : nullptr, topk, order, steps, scale, gc ? c.oc : nullptr, gc,
                          gf, out, c.overflow, s);
}

// vsa_forward_host's pipeline over the head groups of `pl` (see vsa_forward_host): uploads on up_s,
// compute on s, downloads on down_s, ordered by events; `stream` waits for the last download.
vsa_status forward_host_groups(const Dims& d, const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k,
                               const vsa_bf16* v, const vsa_bf16* g_coarse, const vsa_bf16* g_fine, int32_t topk,
                               float scale, void* workspace, const HostPlan& pl, size_t fwd_g, size_t gate_g,
                               uint16_t* dq, uint16_t* dk, uint16_t* dv, uint16_t* dout, uint16_t* dgc,
                               uint16_t* dgf, vsa_bf16* out, cudaStream_t s, cudaStream_t up_s,
                               cudaStream_t down_s) {
    uint8_t* w = static_cast<uint8_t*>(workspace);
    const int64_t rows = static_cast<int64_t>(d.B) * d.N;
    const size_t gb = gate_bytes(d);
    vsa_shape sg = *shape;
    const int groups = pl.n;
    EventSet ev;
    VSA_CUDA(ev.create(2 * groups + 2), "create events");
    uint16_t* cgc = dgc ? reinterpret_cast<uint16_t*>(w + fwd_g) : nullptr;
    uint16_t* cgf = dgf ? reinterpret_cast<uint16_t*>(w + fwd_g + gate_g) : nullptr;
    // everything already on `stream` (earlier users of the workspace) comes first
    VSA_CUDA(cudaEventRecord(ev[0], s), "record start");
    VSA_CUDA(cudaStreamWaitEvent(up_s, ev[0], 0), "order copies");
    VSA_CUDA(cudaStreamWaitEvent(down_s, ev[0], 0), "order copies");
    if (dgc) VSA_CUDA(cudaMemcpyAsync(dgc, g_coarse, gb, cudaMemcpyHostToDevice, up_s), "copy g_coarse to device");
    if (dgf) VSA_CUDA(cudaMemcpyAsync(dgf, g_fine, gb, cudaMemcpyHostToDevice, up_s), "copy g_fine to device");
    const size_t row_all = static_cast<size_t>(d.H) * d.D * 2;
    for (int gi = 0; gi < groups; ++gi) {
        const int h0 = pl.h0[gi], hn = pl.hn[gi];
        const size_t off = static_cast<size_t>(rows) * h0 * d.D;   // elements before this group's block
        const size_t row_g = static_cast<size_t>(hn) * d.D * 2;
        const size_t src_off = static_cast<size_t>(h0) * d.D;
        VSA_CUDA(cudaMemcpy2DAsync(dq + off, row_g, q + src_off, row_all, row_g, rows, cudaMemcpyHostToDevice, up_s),
                 "copy q to device");
        VSA_CUDA(cudaMemcpy2DAsync(dk + off, row_g, k + src_off, row_all, row_g, rows, cudaMemcpyHostToDevice, up_s),
                 "copy k to device");
        VSA_CUDA(cudaMemcpy2DAsync(dv + off, row_g, v + src_off, row_all, row_g, rows, cudaMemcpyHostToDevice, up_s),
                 "copy v to device");
        VSA_CUDA(cudaEventRecord(ev[1 + gi], up_s), "record upload");
        VSA_CUDA(cudaStreamWaitEvent(s, ev[1 + gi], 0), "wait upload");
        sg.heads = hn;
        Dims dh{};
        VSA_TRY(make_dims(&sg, &dh));
        if (cgc) VSA_CUDA(launch_gather_heads(dgc, rows, d.H, h0, hn, cgc, s), "gate gather launch");
        if (cgf) VSA_CUDA(launch_gather_heads(dgf, rows, d.H, h0, hn, cgf, s), "gate gather launch");
        VSA_TRY(run_forward(dh, dq + off, dk + off, dv + off, cgc, cgf, topk, scale, workspace, dout + off, s));
        VSA_CUDA(cudaEventRecord(ev[1 + groups + gi], s), "record compute");
        VSA_CUDA(cudaStreamWaitEvent(down_s, ev[1 + groups + gi], 0), "wait compute");
        VSA_CUDA(cudaMemcpy2DAsync(out + src_off, row_all, dout + off, row_g, row_g, rows, cudaMemcpyDeviceToHost,
                                   down_s),
                 "copy out to host");
    }
    // the call is complete on `stream` once the last output copy is
    VSA_CUDA(cudaEventRecord(ev[1 + 2 * groups], down_s), "record end");
    VSA_CUDA(cudaStreamWaitEvent(s, ev[1 + 2 * groups], 0), "wait end");
    return VSA_OK;
}

}  // namespace

int sm_count() {
    static int counts[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!counts[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        counts[dev] = n;
    }
    return counts[dev];
}

vsa_status set_last_error(vsa_status st, const char* message) { return fail(st, "%s", message); }

}  // namespace vsa

using namespace vsa;

extern "C" {

int32_t vsa_abi_version(void) { return VSA_ABI_VERSION; }

const char* vsa_status_string(vsa_status st) {
    switch (st) {
        case VSA_OK: return "VSA_OK";
        case VSA_ERR_INVALID_ARGUMENT: return "VSA_ERR_INVALID_ARGUMENT";
        case VSA_ERR_UNSUPPORTED: return "VSA_ERR_UNSUPPORTED";
        case VSA_ERR_MISALIGNED: return "VSA_ERR_MISALIGNED";
        case VSA_ERR_WORKSPACE: return "VSA_ERR_WORKSPACE";
        case VSA_ERR_CUDA: return "VSA_ERR_CUDA";
        case VSA_ERR_TIMEOUT: return "VSA_ERR_TIMEOUT";
    }
    return "VSA_ERR_UNKNOWN";
}

const char* vsa_last_error(void) { return g_last_error; }

vsa_status vsa_shape_info(const vsa_shape* shape, int64_t* npad, int32_t* num_cubes) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    if (npad) *npad = d.Npad;
    if (num_cubes) *num_cubes = d.C;
    return VSA_OK;
}

vsa_status vsa_tile(const vsa_shape* shape, const vsa_bf16* x, vsa_bf16* xt, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(need_ptr(x, "x"));
    VSA_TRY(need_ptr(xt, "xt"));
    VSA_TRY(check_disjoint({{x, token_bytes(d), "x"}}, {{xt, tiled_bytes(d), "xt"}}));
    VSA_TRY(check_device());
    Bf16Triple t{{x, nullptr, nullptr}, {xt, nullptr, nullptr}, 1};
    VSA_CUDA(launch_tile(d, t, as_stream(stream)), "tile launch");
    return VSA_OK;
}

vsa_status vsa_untile(const vsa_shape* shape, const vsa_bf16* xt, vsa_bf16* x, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(need_ptr(xt, "xt"));
    VSA_TRY(need_ptr(x, "x"));
    VSA_TRY(check_disjoint({{xt, tiled_bytes(d), "xt"}}, {{x, token_bytes(d), "x"}}));
    VSA_TRY(check_device());
    VSA_CUDA(launch_untile(d, xt, x, as_stream(stream)), "untile launch");
    return VSA_OK;
}

vsa_status vsa_pool(const vsa_shape* shape, const vsa_bf16* xt, float* xbar, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(need_ptr(xt, "xt"));
    VSA_TRY(need_ptr(xbar, "xbar"));
    VSA_TRY(check_disjoint({{xt, tiled_bytes(d), "xt"}}, {{xbar, pooled_bytes(d), "xbar"}}));
    VSA_TRY(check_device());
    const uint16_t* in[1] = {xt};
    float* out[1] = {xbar};
    VSA_CUDA(launch_pool(d, in, out, 1, as_stream(stream)), "pool launch");
    return VSA_OK;
}

size_t vsa_coarse_workspace_bytes(const vsa_shape* shape) {
    Dims d{};
    if (make_dims(shape, &d) != VSA_OK) return 0;
    return 3 * up(parts_bytes(d)) + up(stats_bytes(d));
}

vsa_status vsa_coarse(const vsa_shape* shape, const float* qbar, const float* kbar, const float* vbar, float scale,
                      float* scores, float* o_coarse, void* workspace, size_t workspace_bytes, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(need_ptr(qbar, "qbar"));
    VSA_TRY(need_ptr(kbar, "kbar"));
    VSA_TRY(need_ptr(vbar, "vbar"));
    VSA_TRY(need_ptr(scores, "scores"));
    VSA_TRY(need_ptr(o_coarse, "o_coarse"));
    VSA_TRY(check_scale(scale));
    const size_t need = 3 * up(parts_bytes(d)) + up(stats_bytes(d));
    if (!workspace) return fail(VSA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign != 0)
        return fail(VSA_ERR_MISALIGNED, "workspace is not 256-byte aligned");
    if (workspace_bytes < need) return fail(VSA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, need);
    const size_t pb = pooled_bytes(d);
    VSA_TRY(check_disjoint({{qbar, pb, "qbar"}, {kbar, pb, "kbar"}, {vbar, pb, "vbar"}},
                           {{scores, score_bytes(d), "scores"}, {o_coarse, pb, "o_coarse"}, {workspace, need, "workspace"}}));
    VSA_TRY(check_device());
    cudaStream_t s = as_stream(stream);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    uint16_t* qp = reinterpret_cast<uint16_t*>(w);
    uint16_t* kp = reinterpret_cast<uint16_t*>(w + up(parts_bytes(d)));
    uint16_t* vp = reinterpret_cast<uint16_t*>(w + 2 * up(parts_bytes(d)));
    float* stats = reinterpret_cast<float*>(w + 3 * up(parts_bytes(d)));
    const float* xin[3] = {qbar, kbar, vbar};
    uint16_t* pout[3] = {qp, kp, vp};
    VSA_CUDA(launch_split_parts(d, xin, pout, 3, s), "split launch");
    const char* why = nullptr;
    cudaError_t e = launch_coarse_scores_mma(d, qp, kp, scale, scores, stats, s, &why);
    if (e != cudaSuccess) return why ? fail(VSA_ERR_CUDA, "%s", why) : cuda_fail(e, "coarse launch");
    e = launch_coarse_pv_mma(d, scores, stats, vp, o_coarse, s, &why);
    if (e != cudaSuccess) return why ? fail(VSA_ERR_CUDA, "%s", why) : cuda_fail(e, "coarse launch");
    return VSA_OK;
}

vsa_status vsa_topk(const vsa_shape* shape, const float* scores, int32_t k, int32_t* idx, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(check_k(d, k));
    VSA_TRY(need_ptr(scores, "scores"));
    VSA_TRY(need_ptr(idx, "idx"));
    if (d.C > 49152) return fail(VSA_ERR_UNSUPPORTED, "top-k supports at most 49152 cubes (got %d)", d.C);
    VSA_TRY(check_disjoint({{scores, score_bytes(d), "scores"}}, {{idx, idx_bytes(d, k), "idx"}}));
    VSA_TRY(check_device());
    VSA_CUDA(launch_topk(d, scores, k, idx, as_stream(stream)), "topk launch");
    return VSA_OK;
}

vsa_status vsa_group(const vsa_shape* shape, const float* scores, int32_t* order, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(need_ptr(scores, "scores"));
    VSA_TRY(need_ptr(order, "order"));
    if (d.C > kGroupMaxC) return fail(VSA_ERR_UNSUPPORTED, "grouping supports at most %d cubes (got %d)", kGroupMaxC, d.C);
    VSA_TRY(check_disjoint({{scores, score_bytes(d), "scores"}}, {{order, order_bytes(d), "order"}}));
    VSA_TRY(check_device());
    VSA_CUDA(launch_group(d, scores, order, as_stream(stream)), "group launch");
    return VSA_OK;
}

vsa_status vsa_fine(const vsa_shape* shape, const vsa_bf16* qt, const vsa_bf16* kt, const vsa_bf16* vt,
                    const int32_t* idx, int32_t k, const int32_t* order, float scale, vsa_bf16* o_fine, float* lse,
                    vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    if (idx) VSA_TRY(check_k(d, k));
    VSA_TRY(need_ptr(qt, "qt"));
    VSA_TRY(need_ptr(kt, "kt"));
    VSA_TRY(need_ptr(vt, "vt"));
    VSA_TRY(opt_ptr(idx, "idx"));
    VSA_TRY(opt_ptr(order, "order"));
    VSA_TRY(need_ptr(o_fine, "o_fine"));
    VSA_TRY(opt_ptr(lse, "lse"));
    VSA_TRY(check_scale(scale));
    const size_t tb = tiled_bytes(d);
    VSA_TRY(check_disjoint({{qt, tb, "qt"}, {kt, tb, "kt"}, {vt, tb, "vt"}, {idx, idx ? idx_bytes(d, k) : 0, "idx"},
                            {order, order ? order_bytes(d) : 0, "order"}},
                           {{o_fine, tb, "o_fine"}, {lse, lse ? static_cast<size_t>(d.rows) * 4 : 0, "lse"}}));
    VSA_TRY(check_device());
    FineArgs a{};
    a.mode = kFineTiled;
    a.q = qt;
    a.k = kt;
    a.v = vt;
    a.idx = idx;
    a.k_sel = k;
    a.order = order;
    a.scale = scale;
    a.out = o_fine;
    a.lse = lse;
    const char* why = nullptr;
    cudaError_t e = launch_fine(d, a, as_stream(stream), &why);
    if (e != cudaSuccess) return why ? fail(VSA_ERR_CUDA, "%s", why) : cuda_fail(e, "fine launch");
    return VSA_OK;
}

vsa_status vsa_combine(const vsa_shape* shape, const float* o_coarse, const vsa_bf16* o_fine, const vsa_bf16* g_coarse,
                       const vsa_bf16* g_fine, vsa_bf16* o_tiled, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(need_ptr(o_coarse, "o_coarse"));
    VSA_TRY(need_ptr(o_fine, "o_fine"));
    VSA_TRY(opt_ptr(g_coarse, "g_coarse"));
    VSA_TRY(opt_ptr(g_fine, "g_fine"));
    VSA_TRY(need_ptr(o_tiled, "o_tiled"));
    const size_t tb = tiled_bytes(d), gb = gate_bytes(d);
    VSA_TRY(check_disjoint({{o_coarse, pooled_bytes(d), "o_coarse"}, {o_fine, tb, "o_fine"},
                            {g_coarse, g_coarse ? gb : 0, "g_coarse"}, {g_fine, g_fine ? gb : 0, "g_fine"}},
                           {{o_tiled, tb, "o_tiled"}}));
    VSA_TRY(check_device());
    VSA_CUDA(launch_combine(d, o_coarse, o_fine, g_coarse, g_fine, o_tiled, as_stream(stream)), "combine launch");
    return VSA_OK;
}

vsa_status vsa_topk_order(const vsa_shape* shape, const float* scores, int32_t k, int32_t* idx, int32_t* order,
                          uint64_t* sig_scratch, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(check_k(d, k));
    VSA_TRY(need_ptr(scores, "scores"));
    VSA_TRY(need_ptr(idx, "idx"));
    VSA_TRY(need_ptr(order, "order"));
    VSA_TRY(need_ptr(sig_scratch, "sig_scratch"));
    if (d.C > kTopkRegMaxC || d.C > kGroupMaxC)
        return fail(VSA_ERR_UNSUPPORTED, "vsa_topk_order supports at most %d cubes (got %d)", kTopkRegMaxC, d.C);
    VSA_TRY(check_disjoint({{scores, score_bytes(d), "scores"}},
                           {{idx, idx_bytes(d, k), "idx"}, {order, order_bytes(d), "order"},
                            {sig_scratch, 2 * order_bytes(d), "sig_scratch"}}));
    VSA_TRY(check_device());
    VSA_CUDA(launch_topk_sig(d, scores, k, idx, sig_scratch, as_stream(stream)), "topk launch");
    VSA_CUDA(launch_group_sort(d, sig_scratch, order, as_stream(stream)), "group launch");
    return VSA_OK;
}

size_t vsa_schedule_bytes(const vsa_shape* shape, int32_t topk) {
    Dims d{};
    if (make_dims(shape, &d) != VSA_OK || topk < 1 || topk > d.C) return 0;
    return schedule_bytes(d, topk);
}

vsa_status vsa_schedule(const vsa_shape* shape, const int32_t* idx, int32_t topk, const int32_t* order, void* steps,
                        vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(check_k(d, topk));
    VSA_TRY(need_ptr(idx, "idx"));
    VSA_TRY(opt_ptr(order, "order"));
    VSA_TRY(need_ptr(steps, "steps"));
    if (!schedule_supported(d, topk))
        return fail(VSA_ERR_UNSUPPORTED, "vsa_schedule: C = %d, top-k = %d too large for its shared memory", d.C,
                    topk);
    VSA_TRY(check_disjoint({{idx, idx_bytes(d, topk), "idx"}, {order, order ? order_bytes(d) : 0, "order"}},
                           {{steps, schedule_bytes(d, topk), "steps"}}));
    VSA_TRY(check_device());
    VSA_CUDA(launch_schedule(d, idx, topk, order, steps, as_stream(stream)), "schedule launch");
    return VSA_OK;
}

vsa_status vsa_qk_norm_rope(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* w_q,
                            const vsa_bf16* w_k, float eps, float theta, int64_t token_offset, int64_t n_tokens,
                            vsa_bf16* q_out, vsa_bf16* k_out, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    if (!(eps > 0.f) || !std::isfinite(eps)) return fail(VSA_ERR_INVALID_ARGUMENT, "eps must be finite and > 0");
    if (!(theta > 1.f) || !std::isfinite(theta))
        return fail(VSA_ERR_INVALID_ARGUMENT, "theta must be finite and > 1");
    if (token_offset < 0 || n_tokens < 0)
        return fail(VSA_ERR_INVALID_ARGUMENT, "token_offset and n_tokens must be >= 0");
    if (static_cast<int64_t>(d.H) * d.D > kNormRopeMaxHD)
        return fail(VSA_ERR_UNSUPPORTED, "vsa_qk_norm_rope needs H*D <= %d (got %d)", kNormRopeMaxHD, d.H * d.D);
    if (n_tokens == 0) return VSA_OK;   // nothing to read or write
    VSA_TRY(need_ptr(q, "q"));
    VSA_TRY(need_ptr(k, "k"));
    VSA_TRY(opt_ptr(w_q, "w_q"));
    VSA_TRY(opt_ptr(w_k, "w_k"));
    VSA_TRY(need_ptr(q_out, "q_out"));
    VSA_TRY(need_ptr(k_out, "k_out"));
    const size_t tb = static_cast<size_t>(d.B) * static_cast<size_t>(n_tokens) * d.H * d.D * 2;
    const size_t wb = static_cast<size_t>(d.H) * d.D * 2;
    // in place is q_out == q (and k_out == k); any other overlap is refused
    const Range in_q{q, q == q_out ? 0 : tb, "q"}, in_k{k, k == k_out ? 0 : tb, "k"};
    VSA_TRY(check_disjoint({in_q, in_k, {w_q, w_q ? wb : 0, "w_q"}, {w_k, w_k ? wb : 0, "w_k"}},
                           {{q_out, tb, "q_out"}, {k_out, tb, "k_out"}}));
    VSA_TRY(check_disjoint({{q_out, tb, "q_out"}}, {{k_out, tb, "k_out"}}));
    if (q == q_out) VSA_TRY(check_disjoint({{q, tb, "q"}}, {{k_out, tb, "k_out"}}));
    if (k == k_out) VSA_TRY(check_disjoint({{k, tb, "k"}}, {{q_out, tb, "q_out"}}));
    VSA_TRY(check_device());
    NormRopeArgs a{};
    a.q = q;
    a.k = k;
    a.w_q = w_q;
    a.w_k = w_k;
    a.q_out = q_out;
    a.k_out = k_out;
    a.eps = eps;
    a.theta = theta;
    a.token_offset = token_offset;
    a.n_tokens = n_tokens;
    VSA_CUDA(launch_norm_rope(d, a, as_stream(stream)), "norm/rope launch");
    return VSA_OK;
}

vsa_status vsa_pool_qkv(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                        float* qbar, float* kbar, float* vbar, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(need_ptr(q, "q"));
    VSA_TRY(need_ptr(k, "k"));
    VSA_TRY(need_ptr(v, "v"));
    VSA_TRY(need_ptr(qbar, "qbar"));
    VSA_TRY(need_ptr(kbar, "kbar"));
    VSA_TRY(need_ptr(vbar, "vbar"));
    const size_t tb = token_bytes(d), pb = pooled_bytes(d);
    VSA_TRY(check_disjoint({{q, tb, "q"}, {k, tb, "k"}, {v, tb, "v"}},
                           {{qbar, pb, "qbar"}, {kbar, pb, "kbar"}, {vbar, pb, "vbar"}}));
    VSA_TRY(check_device());
    const uint16_t* in[3] = {q, k, v};
    float* out[3] = {qbar, kbar, vbar};
    VSA_CUDA(launch_pool_tokens(d, in, out, 3, as_stream(stream)), "pool launch");
    return VSA_OK;
}

vsa_status vsa_fine_fused(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                          const int32_t* idx, int32_t topk, const int32_t* order, const void* steps, float scale,
                          const float* o_coarse, const vsa_bf16* g_coarse, const vsa_bf16* g_fine, vsa_bf16* out,
                          int32_t* overflow, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    if (idx) VSA_TRY(check_k(d, topk));
    VSA_TRY(need_ptr(q, "q"));
    VSA_TRY(need_ptr(k, "k"));
    VSA_TRY(need_ptr(v, "v"));
    VSA_TRY(opt_ptr(idx, "idx"));
    VSA_TRY(opt_ptr(order, "order"));
    VSA_TRY(opt_ptr(steps, "steps"));
    if (steps && !idx) return fail(VSA_ERR_INVALID_ARGUMENT, "steps given without idx");
    VSA_TRY(opt_ptr(overflow, "overflow"));
    // the fixed-maximum kernel runs with precomputed steps and for dense attention
    const bool fixed_max = steps != nullptr || idx == nullptr;
    if (fixed_max && !overflow)
        return fail(VSA_ERR_INVALID_ARGUMENT, "%s without an overflow word", steps ? "steps given" : "dense attention");
    if (steps && d.C > kScheduleMaxC)
        return fail(VSA_ERR_UNSUPPORTED, "precomputed steps support at most %d cubes (got %d)", kScheduleMaxC, d.C);
    VSA_TRY(opt_ptr(o_coarse, "o_coarse"));
    VSA_TRY(opt_ptr(g_coarse, "g_coarse"));
    VSA_TRY(opt_ptr(g_fine, "g_fine"));
    VSA_TRY(need_ptr(out, "out"));
    VSA_TRY(check_scale(scale));
    const size_t tb = token_bytes(d), gb = gate_bytes(d);
    VSA_TRY(check_disjoint({{q, tb, "q"}, {k, tb, "k"}, {v, tb, "v"}, {idx, idx ? idx_bytes(d, topk) : 0, "idx"},
                            {order, order ? order_bytes(d) : 0, "order"},
                            {steps, steps ? schedule_bytes(d, topk) : 0, "steps"},
                            {o_coarse, o_coarse ? pooled_bytes(d) : 0, "o_coarse"},
                            {g_coarse, g_coarse ? gb : 0, "g_coarse"}, {g_fine, g_fine ? gb : 0, "g_fine"}},
                           {{out, tb, "out"}, {overflow, fixed_max ? 2 * sizeof(int32_t) : 0, "overflow"}}));
    VSA_TRY(check_device());
    return run_fine_fused(d, q, k, v, idx, topk, order, steps, scale, o_coarse, g_coarse, g_fine, out,
                          fixed_max ? overflow : nullptr, as_stream(stream));
}

size_t vsa_workspace_bytes(const vsa_shape* shape, int32_t topk) {
    Dims d{};
    if (make_dims(shape, &d) != VSA_OK || topk < 1 || topk > d.C) return 0;
    return carve(d, topk, true, nullptr).bytes;
}

vsa_status vsa_forward(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                       const vsa_bf16* g_coarse, const vsa_bf16* g_fine, int32_t topk, float scale, void* workspace,
                       size_t workspace_bytes, vsa_bf16* out, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(check_k(d, topk));
    VSA_TRY(check_scale(scale));
    VSA_TRY(need_ptr(q, "q"));
    VSA_TRY(need_ptr(k, "k"));
    VSA_TRY(need_ptr(v, "v"));
    VSA_TRY(opt_ptr(g_coarse, "g_coarse"));
    VSA_TRY(opt_ptr(g_fine, "g_fine"));
    VSA_TRY(need_ptr(out, "out"));
    if (d.C > 49152) return fail(VSA_ERR_UNSUPPORTED, "top-k supports at most 49152 cubes (got %d)", d.C);
    const size_t need = carve(d, topk, g_coarse != nullptr, nullptr).bytes;
    if (!workspace) return fail(VSA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign != 0)
        return fail(VSA_ERR_MISALIGNED, "workspace is not 256-byte aligned");
    if (workspace_bytes < need)
        return fail(VSA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, need);
    const size_t tb = token_bytes(d), gb = gate_bytes(d);
    VSA_TRY(check_disjoint({{q, tb, "q"}, {k, tb, "k"}, {v, tb, "v"}, {g_coarse, g_coarse ? gb : 0, "g_coarse"},
                            {g_fine, g_fine ? gb : 0, "g_fine"}},
                           {{out, tb, "out"}, {workspace, need, "workspace"}}));
    VSA_TRY(check_device());
    return run_forward(d, q, k, v, g_coarse, g_fine, topk, scale, workspace, out, as_stream(stream));
}

vsa_status vsa_forward_rerun(const vsa_shape* shape, int32_t topk, int32_t has_g_coarse, const void* workspace,
                             int32_t* rerun, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(check_k(d, topk));
    if (!rerun) return fail(VSA_ERR_INVALID_ARGUMENT, "rerun is NULL");
    VSA_TRY(need_ptr(workspace, "workspace"));
    *rerun = 0;
    const Carve c = carve(d, topk, has_g_coarse != 0, const_cast<void*>(workspace));
    if (topk < d.C && c.steps == nullptr) return VSA_OK;   // the sparse stage walked the selection: no fixed maximum
    cudaError_t e = cudaStreamSynchronize(as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int value = 0;
    if ((e = cudaMemcpy(&value, c.overflow, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "read overflow word");
    *rerun = value != 0 ? 1 : 0;
    return VSA_OK;
}

size_t vsa_workspace_bytes_host(const vsa_shape* shape, int32_t topk) {
    Dims d{};
    if (make_dims(shape, &d) != VSA_OK || topk < 1 || topk > d.C) return 0;
    return carve(d, topk, true, nullptr).bytes + 4 * up(token_bytes(d)) + 2 * up(gate_bytes(d));
}

vsa_status vsa_forward_host(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                            const vsa_bf16* g_coarse, const vsa_bf16* g_fine, int32_t topk, float scale,
                            void* workspace, size_t workspace_bytes, vsa_bf16* out, vsa_stream_t stream) {
    Dims d{};
    VSA_TRY(make_dims(shape, &d));
    VSA_TRY(check_k(d, topk));
    VSA_TRY(check_scale(scale));
    if (!q || !k || !v || !out) return fail(VSA_ERR_INVALID_ARGUMENT, "q, k, v and out must be non-NULL host pointers");
    if (d.C > 49152) return fail(VSA_ERR_UNSUPPORTED, "top-k supports at most 49152 cubes (got %d)", d.C);
    const size_t fwd = carve(d, topk, true, nullptr).bytes;
    const size_t tb = token_bytes(d), gb = gate_bytes(d);
    const size_t need = fwd + 4 * up(tb) + 2 * up(gb);
    if (!workspace) return fail(VSA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign != 0)
        return fail(VSA_ERR_MISALIGNED, "workspace is not 256-byte aligned");
    if (workspace_bytes < need)
        return fail(VSA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, need);
    VSA_TRY(check_device());
    uint8_t* w = static_cast<uint8_t*>(workspace);
    uint16_t* dq = reinterpret_cast<uint16_t*>(w + fwd);
    uint16_t* dk = reinterpret_cast<uint16_t*>(w + fwd + up(tb));
    uint16_t* dv = reinterpret_cast<uint16_t*>(w + fwd + 2 * up(tb));
    uint16_t* dout = reinterpret_cast<uint16_t*>(w + fwd + 3 * up(tb));
    uint16_t* dgc = g_coarse ? reinterpret_cast<uint16_t*>(w + fwd + 4 * up(tb)) : nullptr;
    uint16_t* dgf = g_fine ? reinterpret_cast<uint16_t*>(w + fwd + 4 * up(tb) + up(gb)) : nullptr;
    cudaStream_t s = as_stream(stream);

    // Head groups: the heads never mix, so the call runs group by group, and the host->device copies of
    // group g+1 and the device->host copy of group g-1 overlap the compute of group g (two copy streams
    // of the library's, ordered against `stream` by events).  A group's q, k, v and output live compact,
    // [B, N, hn, D], one after the other in the staging buffers; its gates are gathered on the device
    // from the whole arrays into the part of the forward workspace that the smaller call leaves free.
    const int64_t rows = static_cast<int64_t>(d.B) * d.N;
    const HostPlan pl = host_plan(d.H);
    int hg = pl.largest;   // the largest group sizes the per-group workspace and gate staging
    Dims dg{};
    vsa_shape sg = *shape;
    sg.heads = hg;
    size_t gate_g = 0, fwd_g = 0;
    if (hg < d.H && make_dims(&sg, &dg) == VSA_OK) {
        fwd_g = carve(dg, topk, true, nullptr).bytes;
        gate_g = up(static_cast<size_t>(rows) * hg * 2);
        if (fwd_g + 2 * gate_g > fwd) hg = d.H;   // no room for the gathered gates: one group
    } else {
        hg = d.H;
    }
    if (hg == d.H) {
        VSA_CUDA(cudaMemcpyAsync(dq, q, tb, cudaMemcpyHostToDevice, s), "copy q to device");
        VSA_CUDA(cudaMemcpyAsync(dk, k, tb, cudaMemcpyHostToDevice, s), "copy k to device");
        VSA_CUDA(cudaMemcpyAsync(dv, v, tb, cudaMemcpyHostToDevice, s), "copy v to device");
        if (dgc) VSA_CUDA(cudaMemcpyAsync(dgc, g_coarse, gb, cudaMemcpyHostToDevice, s), "copy g_coarse to device");
        if (dgf) VSA_CUDA(cudaMemcpyAsync(dgf, g_fine, gb, cudaMemcpyHostToDevice, s), "copy g_fine to device");
        VSA_TRY(run_forward(d, dq, dk, dv, dgc, dgf, topk, scale, workspace, dout, s));
        VSA_CUDA(cudaMemcpyAsync(out, dout, tb, cudaMemcpyDeviceToHost, s), "copy out to host");
        return VSA_OK;
    }
    cudaStream_t up_s = nullptr, down_s = nullptr;
    VSA_TRY(lib_stream(0, &up_s));
    VSA_TRY(lib_stream(1, &down_s));
    const vsa_status st = forward_host_groups(d, shape, q, k, v, g_coarse, g_fine, topk, scale, workspace, pl, fwd_g,
                                              gate_g, dq, dk, dv, dout, dgc, dgf, out, s, up_s, down_s);
    if (st != VSA_OK) {
        // best effort: whatever the copy streams still hold comes before anything later on `stream`
        cudaEvent_t e1 = nullptr, e2 = nullptr;
        if (cudaEventCreateWithFlags(&e1, cudaEventDisableTiming) == cudaSuccess) {
            if (cudaEventRecord(e1, up_s) == cudaSuccess) cudaStreamWaitEvent(s, e1, 0);
            cudaEventDestroy(e1);
        }
        if (cudaEventCreateWithFlags(&e2, cudaEventDisableTiming) == cudaSuccess) {
            if (cudaEventRecord(e2, down_s) == cudaSuccess) cudaStreamWaitEvent(s, e2, 0);
            cudaEventDestroy(e2);
        }
    }
    return st;
}

vsa_status vsa_device_status(vsa_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int* w = status_word();
    if (!w) return fail(VSA_ERR_CUDA, "watchdog word unavailable");
    int value = 0;
    if ((e = cudaMemcpy(&value, w, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "read watchdog word");
    const int zero = 0;
    if ((e = cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice)) != cudaSuccess)
        return cuda_fail(e, "clear watchdog word");
    if (value == VSA_ERR_TIMEOUT) return fail(VSA_ERR_TIMEOUT, "a device-side wait gave up (work incomplete)");
    return VSA_OK;
}

vsa_status vsa_debug_wait_probe(uint64_t limit_ns, vsa_stream_t stream) {
    if (limit_ns < 1000000ull || limit_ns > 10000000000ull)
        return fail(VSA_ERR_INVALID_ARGUMENT, "limit_ns %llu outside [1 ms, 10 s]", (unsigned long long)limit_ns);
    VSA_TRY(check_device());
    VSA_CUDA(launch_wait_probe(limit_ns, as_stream(stream)), "wait probe launch");
    return VSA_OK;
}

}  // extern "C"
