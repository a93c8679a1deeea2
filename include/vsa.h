/*
 * vsa.h — C ABI of the B200 (sm_100a) cube-based Video Sparse Attention library.
 *
 * The library computes self-attention of a video diffusion transformer over a
 * 3D latent token grid, in two forms:
 *
 *   dense:  O = softmax(Q K^T / sqrt(d)) V, bidirectional (no causal mask).
 *           Wan2.1 acceleration article (bafh001.com), section 4.2 "replace
 *           the attention kernel with a fused implementation".
 *   VSA:    the grid is cut into 4x4x4 cubes of 64 tokens (padded per axis to
 *           a multiple of 4); a coarse attention over mean-pooled cubes ranks
 *           key cubes; each query cube keeps its top-k key cubes; a fine
 *           token-level attention runs over those cubes only; the output is
 *           the gated sum of the coarse and fine results.
 *           Wan2.2 real-time inference teardown (zharfai.com), section
 *           "Video sparse attention selects cubes".
 *
 * Conventions shared by every call
 * --------------------------------
 *  * Grid: T x X x Y tokens (frames x height x width); token index
 *    n = (t*X + x)*Y + y.  Padded grid Tp x Xp x Yp with each axis rounded up
 *    to a multiple of 4; Npad = Tp*Xp*Yp; C = Npad/64 cubes.
 *  * Token layout ("BNHD"): element (b, n, h, d) of a [B, N, H, D] array at
 *    ((b*N + n)*H + h)*D + d, as a DiT's q/k/v projections produce it.
 *  * Cube-major layout ("tiled"): [B, H, Npad, D]; position p = c*64 + o with
 *    cube c = ((t/4)*(Xp/4) + x/4)*(Yp/4) + y/4 and offset
 *    o = ((t%4)*4 + x%4)*4 + y%4.  Positions with t >= T, x >= X or y >= Y
 *    are padding.
 *  * bf16 values are passed as uint16_t bit patterns (vsa_bf16).
 *  * Every pointer argument is a DEVICE pointer owned by the caller, except in
 *    vsa_forward_host where the tensors are HOST pointers.  The library never
 *    allocates or frees memory.  Its only device state is one watchdog status
 *    word per device, the static workspace of vsa_forward_noalloc, and, once
 *    vsa_forward_host has run on a device, that function's two copy streams.
 *    The device addresses of the two static words are looked up once per
 *    device and kept for the life of the process, so the library must not be
 *    used across a cudaDeviceReset (or any other teardown of the device's
 *    primary context): the module is then loaded again at other addresses.
 *  * Every device pointer must be 16-byte aligned; input and output ranges of
 *    one call must not overlap.
 *  * `stream` is a cudaStream_t passed as an opaque pointer (NULL = the
 *    legacy default stream).  All work is enqueued asynchronously on it.
 *  * Errors in the arguments are reported synchronously, before anything is
 *    enqueued, by the returned status; vsa_last_error() then gives a one-line
 *    reason (thread-local).  A failed launch returns VSA_ERR_CUDA.  A device
 *    wait that exceeded its limit is reported later by vsa_device_status().
 *  * Supported: head_dim 64 or 128; 1 <= top-k <= C; B*H*Npad < 2^31.
 *    Only sm_100a devices run the kernels; there is no fallback path.
 */
#ifndef VSA_B200_H
#define VSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VSA_ABI_VERSION 3

typedef uint16_t vsa_bf16;
typedef void* vsa_stream_t;

typedef struct vsa_shape {
    int32_t batch;     /* B */
    int32_t heads;     /* H */
    int32_t head_dim;  /* D: 64 or 128 */
    int32_t grid_t;    /* T: latent frames */
    int32_t grid_h;    /* X: token rows per frame */
    int32_t grid_w;    /* Y: token columns per frame */
} vsa_shape;

typedef enum vsa_status {
    VSA_OK = 0,
    VSA_ERR_INVALID_ARGUMENT = 1, /* a size, count or pointer is out of range */
    VSA_ERR_UNSUPPORTED = 2,      /* valid request this build does not run (head_dim, device) */
    VSA_ERR_MISALIGNED = 3,       /* a pointer is not 16-byte aligned */
    VSA_ERR_WORKSPACE = 4,        /* workspace missing or smaller than vsa_workspace_bytes() */
    VSA_ERR_CUDA = 5,             /* a CUDA runtime call or kernel launch failed */
    VSA_ERR_TIMEOUT = 6           /* a device-side wait gave up (see vsa_device_status) */
} vsa_status;

/* ABI version of the loaded library (VSA_ABI_VERSION). */
int32_t vsa_abi_version(void);

/* Static text for a status code. */
const char* vsa_status_string(vsa_status status);

/* One-line reason for the last non-OK status returned on this host thread. */
const char* vsa_last_error(void);

/* Derived sizes of a shape: padded token count Npad and cube count C.
 * Returns VSA_ERR_INVALID_ARGUMENT for a malformed shape. */
vsa_status vsa_shape_info(const vsa_shape* shape, int64_t* npad, int32_t* num_cubes);

/*
 * vsa_tile — cube-major permutation with zero padding (step "pad and cut the
 * grid into 4x4x4 cubes", teardown section "Video sparse attention selects
 * cubes": 21x30x52 is padded to 24x32x52 = 39,936 tokens, 624 cubes).
 *   x   [B, N, H, D] bf16, token layout (read).
 *   xt  [B, H, Npad, D] bf16, tiled layout (written); padded rows are zero.
 */
vsa_status vsa_tile(const vsa_shape* shape, const vsa_bf16* x, vsa_bf16* xt, vsa_stream_t stream);

/*
 * vsa_untile — inverse of vsa_tile on the real tokens; padded rows are dropped.
 *   xt  [B, H, Npad, D] bf16 tiled (read);  x [B, N, H, D] bf16 (written).
 */
vsa_status vsa_untile(const vsa_shape* shape, const vsa_bf16* xt, vsa_bf16* x, vsa_stream_t stream);

/*
 * vsa_pool — one representative vector per cube: the mean of the cube's real
 * tokens (teardown, "Video sparse attention selects cubes", part 1 "coarse
 * attention": each cube's query or key vectors are averaged into one).
 *   xt    [B, H, Npad, D] bf16 tiled (read; padded rows are not read).
 *   xbar  [B, H, C, D] float32 (written).
 */
vsa_status vsa_pool(const vsa_shape* shape, const vsa_bf16* xt, float* xbar, vsa_stream_t stream);

/*
 * vsa_coarse — block-level attention over the pooled cubes (same section,
 * part 1): scores = scale * qbar kbar^T, o_coarse = softmax_rows(scores) vbar,
 * both contractions on the tensor cores.  The scores rank the cubes, so they
 * need float32 accuracy: each float32 input x is carried as three bf16 parts
 * (hi = bf16(x), mid = bf16(x - hi), lo = bf16(x - hi - mid), together within
 * 2^-24 |x|) and each product from its six partial products of size >= 2^-18
 * (hi*hi, hi*mid, mid*hi, hi*lo, lo*hi, mid*mid; the dropped ones are below
 * 2^-26), accumulated in float32.  vsa_forward computes the same bits.
 *   qbar, kbar, vbar  [B, H, C, D] float32 (read).
 *   scores            [B, H, C, C] float32 (written): row = query cube.
 *   o_coarse          [B, H, C, D] float32 (written).
 *   workspace         device buffer of vsa_coarse_workspace_bytes(shape),
 *                     256-byte aligned (the split inputs and per-row softmax
 *                     statistics; contents on return unspecified).
 */
size_t vsa_coarse_workspace_bytes(const vsa_shape* shape);
vsa_status vsa_coarse(const vsa_shape* shape, const float* qbar, const float* kbar, const float* vbar,
                      float scale, float* scores, float* o_coarse, void* workspace, size_t workspace_bytes,
                      vsa_stream_t stream);

/*
 * vsa_topk — per query cube, the k key cubes with the highest coarse score
 * (same section: the candidates are ranked and the top-k kept; 78 of 624 at
 * 87.5% sparsity).  Equal scores go to the lower cube index; each row of the
 * result is in ascending cube order.  Bit-exact for a given scores array.
 *   scores  [B, H, C, C] float32 (read).   idx [B, H, C, k] int32 (written).
 */
vsa_status vsa_topk(const vsa_shape* shape, const float* scores, int32_t k, int32_t* idx, vsa_stream_t stream);

/*
 * vsa_group — work order for vsa_fine (a schedule, not a step of the method):
 * per (b, h), the query cubes sorted by the indices of their three
 * highest-scoring key cubes (ties to the lower index).  Consecutive entries
 * then tend to select the same key cubes, and vsa_fine processes groups of
 * four consecutive entries over one shared key/value stream.  The output of
 * vsa_fine does not depend on the order.
 *   scores  [B, H, C, C] float32 (read).   order [B, H, C] int32 (written): a
 *           permutation of [0, C) per (b, h).   Requires C <= 4096.
 */
vsa_status vsa_group(const vsa_shape* shape, const float* scores, int32_t* order, vsa_stream_t stream);

/*
 * vsa_fine — token-level attention of every 64-token query cube over the
 * tokens of its selected key cubes (same section, part 2 "fine attention"),
 * padded key tokens excluded, online softmax in float32 (teardown section
 * "Fixed-max softmax is a numerical contract"), QK^T and PV on the tensor
 * cores in bf16 with float32 accumulation.
 *   qt, kt, vt  [B, H, Npad, D] bf16 tiled (read).  Padded rows of vt must be
 *               finite (vsa_tile writes zeros); padded rows of kt may hold
 *               anything finite.
 *   idx         [B, H, C, k] int32 cube indices in [0, C), or NULL for all C
 *               cubes in order (dense attention).  A cube listed twice is
 *               attended twice.  Out-of-range entries are treated as an empty
 *               cube (no memory outside the tensors is read).
 *   k           entries per row of idx (ignored, taken as C, when idx is NULL).
 *   order       [B, H, C] int32 per-head permutation of the query cubes that
 *               sets the work order (groups of four consecutive entries share
 *               one key/value stream; see vsa_group), or NULL for 0..C-1.  An
 *               entry outside [0, C) is skipped; a cube missing from `order`
 *               leaves its output rows unwritten.
 *   scale       softmax scale, normally 1/sqrt(D).
 *   o_fine      [B, H, Npad, D] bf16 (written).  Rows of padded query
 *               positions are written but carry no meaning.
 *   lse         [B, H, Npad] float32 natural-log sum of exp(scale*q.k) over
 *               the attended keys (written), or NULL.
 */
vsa_status vsa_fine(const vsa_shape* shape, const vsa_bf16* qt, const vsa_bf16* kt, const vsa_bf16* vt,
                    const int32_t* idx, int32_t k, const int32_t* order, float scale, vsa_bf16* o_fine,
                    float* lse, vsa_stream_t stream);

/*
 * vsa_combine — gated merge (same section, part 3): per token and head,
 * O = g_coarse * o_coarse[cube] + g_fine * o_fine, float32 arithmetic, bf16
 * result.  Padded positions are written as zero.
 *   o_coarse  [B, H, C, D] float32;  o_fine [B, H, Npad, D] bf16 tiled.
 *   g_coarse, g_fine  [B, N, H] bf16 in token layout, or NULL (g_coarse = 0,
 *                     g_fine = 1).
 *   o_tiled   [B, H, Npad, D] bf16 (written).
 */
vsa_status vsa_combine(const vsa_shape* shape, const float* o_coarse, const vsa_bf16* o_fine,
                       const vsa_bf16* g_coarse, const vsa_bf16* g_fine, vsa_bf16* o_tiled,
                       vsa_stream_t stream);

/*
 * vsa_topk_order — the selection and a work order from one pass over the
 * scores: the k best key cubes of every query cube (identical to vsa_topk)
 * and, per (b, h), the query cubes sorted by their four smallest selected key
 * cubes, then by their own index (a schedule, not a step of the method: the
 * fine stage's tiles are pairs of consecutive cubes, and cubes whose
 * selections start alike share more of them than cubes with the same three
 * best cubes, which vsa_group sorts by).  Two launches: the selection, which
 * also writes each row's key to sig_scratch, then a per-head sort of the keys.
 *   scores       [B, H, C, C] float32 (read).
 *   idx          [B, H, C, k] int32 (written).
 *   order        [B, H, C] int32 (written).
 *   sig_scratch  [B, H, C] uint64 caller scratch (overwritten).
 * Supported for C <= 2048 (VSA_ERR_UNSUPPORTED otherwise; use vsa_topk and
 * vsa_group, which vsa_forward then does as well).
 */
vsa_status vsa_topk_order(const vsa_shape* shape, const float* scores, int32_t k, int32_t* idx, int32_t* order,
                          uint64_t* sig_scratch, vsa_stream_t stream);

/*
 * vsa_qk_norm_rope — the pre-attention pass of a Wan DiT block: RMSNorm of each
 * token's query and key over all H*D channels, then the 3D rotary position
 * embedding, in one read and one write of Q and K (WorldFoundry inference guide,
 * "推理优化", exact-kernel table, row fused_rope; Wan2.2 teardown, zharfai.com,
 * section "Fusion targets launch overhead and memory").
 *   q, k           [B, n_tokens, H, D] bf16 (read): rows of global tokens
 *                  token_offset .. token_offset + n_tokens - 1 (a sequence-
 *                  parallel shard, or the whole sequence with offset 0).
 *   w_q, w_k       [H*D] bf16 RMSNorm weights, or NULL (weight 1).
 *   eps            > 0: y = x / sqrt(mean(x^2) + eps) * w, in float32.
 *   theta          > 1: RoPE base.  The D/2 channel pairs (2i, 2i+1) of each
 *                  head form three bands, for the token's t, x and y
 *                  coordinates in that order (x and y floor(D/6) pairs each, t
 *                  the rest); pair j of a band of P pairs turns by
 *                  pos * theta^(-j/P) radians (angles in float64, rotation in
 *                  float32), (a, b) -> (a cos - b sin, a sin + b cos).
 *   q_out, k_out   [B, n_tokens, H, D] bf16 (written, rounded once); q_out may
 *                  be q and k_out may be k (in place); no other overlap.
 * Rows whose global token index is >= N (the padding that evens out shards)
 * are written as zeros.  Needs H*D <= 8192 (VSA_ERR_UNSUPPORTED otherwise).
 * With n_tokens = 0 nothing is read or written and the pointers may be NULL.
 */
vsa_status vsa_qk_norm_rope(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* w_q,
                            const vsa_bf16* w_k, float eps, float theta, int64_t token_offset, int64_t n_tokens,
                            vsa_bf16* q_out, vsa_bf16* k_out, vsa_stream_t stream);

/*
 * vsa_pool_qkv — the cube mean-pool of vsa_pool applied to q, k and v in one
 * launch, read straight from the token layout (no tiled copy).  Each mean is
 * summed in the same float32 order as vsa_pool on the tiled tensor, so the two
 * give identical bits.  Same section, part 1.
 *   q, k, v           [B, N, H, D] bf16 token layout (read).
 *   qbar, kbar, vbar  [B, H, C, D] float32 (written).
 */
vsa_status vsa_pool_qkv(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                        float* qbar, float* kbar, float* vbar, vsa_stream_t stream);

/*
 * vsa_fine_fused — the fine stage (part 2) and the gated merge (part 3) in
 * one kernel, on the token layout: key/value cubes are gathered from q, k, v
 * by the copy engine (padded positions read as zeros, so no vsa_tile pass),
 * and each query row's result g_coarse * o_coarse[cube] + g_fine * O_fine is
 * written to its token's row of `out` (no vsa_combine / vsa_untile pass).
 * O_fine is not rounded to bf16 before the merge.
 * With idx == NULL every key is attended (dense attention, the Wan2.1
 * article's section 4.2): the kernel then walks blocks of 64 consecutive real
 * tokens instead of cubes, so no padded position is computed at all.
 *   q, k, v    [B, N, H, D] bf16 token layout (read).
 *   idx, k, order, scale   as in vsa_fine (idx NULL: dense; order then unused).
 *   steps      vsa_schedule's output for this idx and order, or NULL (the
 *              kernel then walks the selection itself, in index order).
 *   o_coarse   [B, H, C, D] float32, or NULL (no coarse term; g_coarse ignored).
 *   g_coarse, g_fine  [B, N, H] bf16 or NULL (g_coarse = 0, g_fine = 1).
 *   out        [B, N, H, D] bf16 (written at every real token).
 *   overflow   two int32 of caller-owned device memory (4-byte aligned);
 *              required with `steps` and with idx == NULL
 *              (VSA_ERR_INVALID_ARGUMENT otherwise), ignored otherwise.
 *              overflow[0] is the overflow word below; overflow[1] is the
 *              one-tile kernel's work counter (its CTAs claim work items from
 *              it, so that items of unequal length balance across the SMs),
 *              cleared by the call with word 0.
 *              With steps, and for dense attention, the stage runs on the
 *              one-tile kernel, which keeps each query row's first selected
 *              (dense: first block's) maximum fixed for the whole row
 *              (teardown section "Fixed-max softmax is a numerical contract"):
 *              the call clears the word, the kernel sets it to 1 when a
 *              probability would exceed 2^64 or a row sum is not finite, and a
 *              second launch then re-runs the whole stage with online
 *              rescaling (it returns at once when the word is 0).  When the
 *              stream has passed the call the word tells whether the re-run
 *              happened.  Calls running at the same time need distinct words.
 */
vsa_status vsa_fine_fused(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                          const int32_t* idx, int32_t topk, const int32_t* order, const void* steps, float scale,
                          const float* o_coarse, const vsa_bf16* g_coarse, const vsa_bf16* g_fine,
                          vsa_bf16* out, int32_t* overflow, vsa_stream_t stream);

/* Bytes of the step list vsa_schedule writes for this shape and top-k. */
size_t vsa_schedule_bytes(const vsa_shape* shape, int32_t topk);

/*
 * vsa_schedule — the fine stage's work, precomputed: for every group of four
 * query cubes (four consecutive entries of `order`), the merged union of their
 * selections, paired two key cubes per step, cubes that only the first two
 * query cubes selected first, then those only the last two selected, then
 * those both pairs selected (fewer half-used 128-row tiles).  The fine kernel
 * given these steps does no list walking of its own; the result equals the
 * kernel's own walk up to the order of the float32 sums.
 *   idx, topk, order  as in vsa_fine (order may be NULL for 0..C-1).
 *   steps             device buffer of vsa_schedule_bytes(shape, topk) (written).
 * Returns VSA_ERR_UNSUPPORTED when its shared memory, 4 x (C/8 + 1 + 4 topk)
 * 32-bit words, exceeds 48 KB (C = 624, topk = 32 needs 3.3 KB); vsa_forward
 * then lets the fine kernel walk the selection itself.  A list that holds a
 * cube twice is visited as often as it holds it.
 */
vsa_status vsa_schedule(const vsa_shape* shape, const int32_t* idx, int32_t topk, const int32_t* order,
                        void* steps, vsa_stream_t stream);

/* Bytes of device workspace vsa_forward needs for this shape and top-k
 * (0 for a malformed shape). */
size_t vsa_workspace_bytes(const vsa_shape* shape, int32_t topk);

/*
 * vsa_forward — the whole attention call on one stream, as eight launches for
 * top-k < C with a coarse gate:
 *   vsa_pool_qkv (writing the pooled vectors as their three bf16 parts; v only
 *   with g_coarse, since only the coarse output uses it) ->
 *   the coarse scores (tensor cores; with g_coarse they also keep each row's
 *   softmax statistics) -> vsa_topk_order (2) -> the coarse output (tensor
 *   cores; skipped when g_coarse is NULL, since only the merge uses it) ->
 *   vsa_schedule -> vsa_fine_fused (the one-tile kernel and its re-run guard)
 * (vsa_topk -> vsa_group instead when C > 2048; the grouping step is skipped
 * when C > 4096).  The scores and the selection are the bits of vsa_coarse and
 * vsa_topk_order; the result equals
 *   tile -> pool -> coarse -> topk -> group -> fine -> combine -> untile
 * up to the bf16 rounding of O_fine that the staged path makes.
 * When topk == C every cube is selected and the fine stage is dense attention
 * over the real tokens: vsa_fine_fused with idx == NULL, preceded by
 * vsa_pool_qkv -> vsa_coarse only when g_coarse is given.  With both gates
 * NULL that is dense attention in two launches (the one-tile kernel and its
 * re-run guard, which returns at once unless the fixed maxima overflowed).
 *   q, k, v      [B, N, H, D] bf16 token layout (read).
 *   g_coarse, g_fine  [B, N, H] bf16 or NULL (see vsa_combine).
 *   workspace    device buffer of at least vsa_workspace_bytes(shape, topk),
 *                256-byte aligned (that size covers both gates; a call without
 *                g_coarse at topk == C needs only 256 bytes); its contents on
 *                return are unspecified.
 *   out          [B, N, H, D] bf16 (written).
 */
vsa_status vsa_forward(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                       const vsa_bf16* g_coarse, const vsa_bf16* g_fine, int32_t topk, float scale,
                       void* workspace, size_t workspace_bytes, vsa_bf16* out, vsa_stream_t stream);

/*
 * vsa_forward_rerun — whether the last vsa_forward call on `workspace` (with
 * this shape, top-k and coarse gate given or not: has_g_coarse 0 or 1) had to
 * re-run its fine stage with online rescaling because the fixed per-row
 * maxima overflowed (see the `overflow` argument of vsa_fine_fused; the
 * forward call keeps that word in its workspace).  Synchronizes `stream`,
 * then sets *rerun to 1 or 0.  A sparse call whose fine stage walked the
 * selection itself (no precomputed steps: C above the schedule's limit),
 * which rescales online from the start, always gives 0 without touching the
 * device.
 */
vsa_status vsa_forward_rerun(const vsa_shape* shape, int32_t topk, int32_t has_g_coarse, const void* workspace,
                             int32_t* rerun, vsa_stream_t stream);

/* Bytes of device workspace vsa_forward_host needs: vsa_workspace_bytes plus
 * device staging for the inputs and the output. */
size_t vsa_workspace_bytes_host(const vsa_shape* shape, int32_t topk);

/*
 * vsa_forward_host — vsa_forward on HOST tensors.  The heads are independent
 * (Wan2.2 teardown, zharfai.com, section "Video sparse attention selects
 * cubes": attention per head), so with two or more heads the call runs in up
 * to eight groups of heads: each group's q, k and v are copied host->device
 * (2-D copies of its head range into compact staging), its call runs on
 * `stream`, and its output is copied back into its head range of `out`; the
 * copies run on two copy streams of the library's, ordered against `stream`
 * by events, so the uploads of one group and the download of another overlap
 * the compute of a third.  With 27 or more heads the last groups shrink (4,
 * 2, 1 heads), so little compute and download follow the last upload.  The
 * gates are copied whole and gathered per group
 * on the device.  The result is bit-identical to vsa_forward on the same
 * inputs.  Everything already enqueued on `stream` happens before the copies,
 * and the call's last copy is complete when `stream` reaches the point after
 * the call.  Host buffers must be pinned for the copies to be asynchronous
 * (pageable buffers work, without overlap); the call returns once the work
 * is enqueued and `out` is valid after the stream is synchronized.
 *   q, k, v, g_coarse, g_fine, out: HOST pointers (gates may be NULL).
 *   workspace: DEVICE buffer of vsa_workspace_bytes_host(shape, topk) bytes.
 */
vsa_status vsa_forward_host(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                            const vsa_bf16* g_coarse, const vsa_bf16* g_fine, int32_t topk, float scale,
                            void* workspace, size_t workspace_bytes, vsa_bf16* out, vsa_stream_t stream);

/* Size of the static device workspace used by vsa_forward_noalloc (32 MiB). */
#define VSA_NOALLOC_WORKSPACE_BYTES ((size_t)32 << 20)

/*
 * vsa_forward_noalloc — vsa_forward for callers that cannot allocate device
 * memory.  The pages have no counterpart; this is an interface convenience.
 * Examples are a plugin that a host runtime hands only its input and output
 * buffers, a runtime whose memory pool owns the device and forbids
 * out-of-band cudaMalloc (which synchronizes the device and fragments the
 * pool), and real-time code that must not allocate after start-up.
 * Arguments are those of vsa_forward without the workspace: q, k, v, gates
 * and out are caller-owned DEVICE buffers.  The workspace is a static
 * device array of VSA_NOALLOC_WORKSPACE_BYTES inside the library, so the
 * call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine).  Each GPU on which the library's module is loaded holds that
 * array until the process exits.
 *   - A shape whose vsa_workspace_bytes() exceeds VSA_NOALLOC_WORKSPACE_BYTES
 *     is rejected with VSA_ERR_WORKSPACE before anything is enqueued.
 *   - The first call on a device looks the array's device address up
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents (nothing in it needs to start at zero).  Calls that overlap on
 *     the GPU race on it: serialize them (one stream, or events).
 */
vsa_status vsa_forward_noalloc(const vsa_shape* shape, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                               const vsa_bf16* g_coarse, const vsa_bf16* g_fine, int32_t topk, float scale,
                               vsa_bf16* out, vsa_stream_t stream);

/*
 * vsa_device_status — synchronizes `stream`, then reads and clears the
 * current device's watchdog word.  Returns VSA_ERR_TIMEOUT if a kernel of
 * this library gave up on a device-side wait since the last read (its output
 * is then incomplete), VSA_ERR_CUDA if the synchronization failed, else VSA_OK.
 */
vsa_status vsa_device_status(vsa_stream_t stream);

/*
 * vsa_debug_wait_probe — diagnostic for the watchdog: launches one block that
 * waits on a shared-memory barrier nothing arrives on, with the library's
 * bounded wait, giving up after `limit_ns` nanoseconds (1 ms .. 10 s) and
 * recording VSA_ERR_TIMEOUT for vsa_device_status().  Faults nothing and
 * leaves the context usable.
 */
vsa_status vsa_debug_wait_probe(uint64_t limit_ns, vsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* VSA_B200_H */
