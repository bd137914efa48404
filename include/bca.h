/*
 * bca.h - C ABI of the block-causal attention library (libbca.so) for NVIDIA B200
 * (sm_100a).  Plain pointers and sizes only; no C++ or framework types cross it.
 *
 * The operation (all citations name the MAGI-1 pages by title and section):
 *
 *   Block-causal attention: tokens attend fully to the tokens of their own video
 *   chunk and to every token of earlier chunks, never to later chunks
 *   ("Magi-1 开源&刷屏" (163.com), the block-causal attention bullets; MAGI-1
 *   research notes (zhao9797.github.io), "Model architecture > Overall pipeline").
 *   The mask is a union of AttnSlices (q-range, k-range, full|causal), which also
 *   expresses packed variable-length videos and KV-range limits (MAGI-1 research
 *   notes, "Infra > MagiAttention > Flex-Flash-Attention" and "Inference tricks >
 *   KV Cache"; interview with Zhang Zheng (zhengguannews), the q_range/k_range
 *   answer).  Queries and keys pass through QK-Norm and a 3D (t, h, w) RoPE before
 *   the dot product, and heads are grouped (GQA, 128 query heads over 8 KV heads)
 *   (MAGI-1 research notes, "Autoregressive denoising DiT" and Table 2).
 *
 *   For query token i, query head h, KV head g = h / (Hq / Hkv):
 *     qh_i = RoPE(pos_i, RMSNorm(q_i))   kh_j = RoPE(pos_j, RMSNorm(k_j))
 *     s_ij = qh_i . kh_j / sqrt(D) over the keys j visible to i,
 *     LSE_i = log sum_j exp(s_ij),  O_i = sum_j exp(s_ij - LSE_i) v_j.
 *   A row that sees no key has O = 0 and LSE = -inf.
 *
 * Key index space = [cache keys | new keys]: cache key c has index c, new token n
 * has key index num_cache_keys + n.  Cache keys are taken as already normalised
 * and rotated (they are the features of earlier chunks) and are used as given.
 *
 * Layouts (token-major, contiguous, row-major):
 *   q, dout, o, dq ........ [Nq][Hq][D]
 *   k, v, dk, dv .......... [Nq][Hkv][D]       (new tokens)
 *   k_cache, v_cache, dk_cache, dv_cache [Nc][Hkv][D]
 *   lse ................... [Hq][Nq] fp32, natural log
 *   bf16 tensors are IEEE bfloat16; every pointer must be 16-byte aligned.
 *
 * Ownership: the caller owns every tensor, the workspace and the stream.  A plan
 * owns its host tables and the device metadata it uploads, freed by
 * bca_plan_destroy.  bca_fwd and bca_bwd are asynchronous on the given stream and
 * never allocate.
 *
 * Errors: every int-returning call returns BCA_OK (0) or a negative BCA_ERR_*.
 * Argument checks happen on the host before any launch; a failed check launches
 * nothing.  No call traps the GPU.  Device-side waits are bounded: a wait that runs
 * out records BCA_ERR_DEVICE_TIMEOUT in the plan's status word (read it with
 * bca_status).
 */
#ifndef BCA_H
#define BCA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BCA_OK 0
#define BCA_ERR_INVALID_ARGUMENT (-1)  /* NULL pointer, bad size, bad flag */
#define BCA_ERR_BAD_SLICE (-2)         /* slice out of range, begin > end, bad type */
#define BCA_ERR_UNSUPPORTED (-3)       /* head_dim / head grouping / geometry not supported */
#define BCA_ERR_MISALIGNED (-4)        /* a pointer is not 16-byte aligned */
#define BCA_ERR_CUDA (-5)              /* a CUDA runtime call failed */
#define BCA_ERR_DEVICE_TIMEOUT (-6)    /* a device-side wait ran out (see bca_status) */
#define BCA_ERR_HOST_ONLY_PLAN (-7)    /* plan was built with BCA_PLAN_HOST_ONLY */
#define BCA_ERR_NO_MEMORY (-8)         /* host or device allocation failed in bca_plan_create */
#define BCA_ERR_TOO_LARGE (-9)         /* problem needs more scratch than the static workspace holds */

/* AttnSlice type */
#define BCA_SLICE_FULL 0
#define BCA_SLICE_CAUSAL 1 /* bottom-right aligned: j-k0 <= (i-q0) + (|k| - |q|) */

/* bca_problem.flags */
#define BCA_O_FP32 0x1u          /* write O as fp32 instead of bf16 */
#define BCA_PLAN_HOST_ONLY 0x2u  /* compile the mask on the host only (no CUDA calls) */
#define BCA_TEST_FORCE_TIMEOUT 0x4u /* failure-detection test: the attention kernels of bca_fwd
                                       and bca_bwd issue none of their tile loads and their
                                       waits give up after 1 ms, so every CTA records
                                       BCA_ERR_DEVICE_TIMEOUT and exits cleanly (outputs are
                                       then meaningless) */
#define BCA_FWD_FP8_E4M3 0x8u /* forward with e4m3 tensor-core operands (the 8-bit float
                                 MMAs of sm_100a): Q-hat and K-hat rounded to e4m3, V to
                                 e4m3 after division by a power of two per KV head (from
                                 max|V|, undone in the epilogue), P to e4m3; accumulation,
                                 softmax and LSE stay fp32.  The MAGI-1 pages quantise
                                 their linear layers to FP8 at inference (Notes,
                                 inference infrastructure, real-time streaming scenario:
                                 W8A8 SmoothQuant); this applies the format to attention.
                                 Error: each score and each P carries a relative rounding
                                 error of at most 2^-4 (e4m3's 3-bit significand), so
                                 O is accurate to a few percent of |V| / sqrt(effective
                                 number of keys), not to bf16 precision.  Forward only:
                                 bca_bwd / bca_bwd_ex on such a plan return
                                 BCA_ERR_UNSUPPORTED (train with bf16 plans). */
#define BCA_NO_PROLOGUE 0x10u /* q and k are given post-prologue: no QK-Norm and no RoPE
                                 is applied (the attention alone, s = q.k / sqrt(D)), and
                                 the gradients are w.r.t. the given q and k.  The kernels
                                 stage q and k as fp16 (11-bit significand), so every
                                 element must satisfy |x| < 60000 (else it rounds to
                                 infinity).  q_gain, k_gain and the parameter gradients of
                                 bca_bwd_ex do not exist then: passing any of them returns
                                 BCA_ERR_INVALID_ARGUMENT.  bca_k_prologue copies k (bf16)
                                 and bca_k_prologue_bwd passes dk_hat through.  Not
                                 combinable with BCA_FWD_FP8_E4M3 (BCA_ERR_UNSUPPORTED). */
#define BCA_DQ_DETERMINISTIC 0x20u /* bca_bwd / bca_bwd_ex form dQ by a separate pass, one CTA
                                      per (query tile, query head) walking its key tiles in a
                                      fixed order (S and dP are recomputed there), instead of
                                      summing the key-tile CTAs' shares with reduce-adds whose
                                      order varies: dQ is then bit-identical from run to run,
                                      like dK and dV.  Costs two more matrix products per
                                      visible tile.  (The parameter gradients of bca_bwd_ex
                                      still use atomic adds.) */
#define BCA_CACHE_K_FP16 0x40u /* k_cache is IEEE fp16 instead of bf16, and bca_k_prologue
                                  writes fp16 K-hat.  The kernels stage K-hat as fp16
                                  anyway, so a cache key given in fp16 enters the scores
                                  with the same rounding as a new key of the plan; context
                                  parallelism uses this for keys borrowed from other ranks.
                                  Cache keys must then stay below 65,504 in magnitude.
                                  Not combinable with BCA_FWD_FP8_E4M3. */

/* bca_workspace_bytes(pass) */
#define BCA_PASS_FWD 0
#define BCA_PASS_BWD 1

/* One AttnSlice: query rows [q_begin, q_end) see keys [k_begin, k_end), fully or
 * causally.  Same memory layout as int64 [5]. */
typedef struct {
    int64_t q_begin, q_end, k_begin, k_end, type;
} bca_slice;

/* Geometry of the new tokens of one video, packed in order: tokens are numbered
 * chunk, latent frame, row, column (raster order); token (c, f, y, x) has RoPE
 * position (t0 + c*frames + f, y, x).  Same layout as int32 [5]. */
typedef struct {
    int32_t num_chunks, frames, height, width, t0;
} bca_video;

typedef struct {
    int32_t num_q_heads;        /* Hq */
    int32_t num_kv_heads;       /* Hkv; Hq % Hkv == 0.  An even group size Hq / Hkv runs two
                                   query heads per forward work item (each K/V tile loaded
                                   once for both), an odd one (MHA, Hkv = Hq, included) one */
    int32_t head_dim;           /* D in {24, 32, 48} */
    int32_t num_videos;
    const bca_video *videos;    /* Nq = sum of chunks*frames*height*width */
    int64_t num_cache_keys;     /* Nc */
    int32_t num_slices;
    const bca_slice *slices;    /* NULL => block-causal per video, cache visible to
                                   every chunk of the first video */
    float rope_base[3];         /* RoPE base per axis (t, h, w) */
    float norm_eps;             /* QK-Norm epsilon */
    uint32_t flags;             /* BCA_O_FP32 | BCA_PLAN_HOST_ONLY | BCA_TEST_FORCE_TIMEOUT |
                                   BCA_FWD_FP8_E4M3 | BCA_NO_PROLOGUE | BCA_DQ_DETERMINISTIC |
                                   BCA_CACHE_K_FP16 */
} bca_problem;

typedef struct bca_plan_s *bca_plan_t;

/* Plan statistics (host introspection; used by tests and the benchmark). */
typedef struct {
    int64_t num_q, num_k, num_cache;
    int64_t num_q_tiles, num_k_tiles;
    int64_t num_runs;            /* runs of consecutive k-tiles over all q-tiles */
    int64_t num_full_tiles, num_partial_tiles;
    int64_t num_items;           /* forward work items (q-tile x 2 query heads of one KV
                                    group, or x 1 head for an odd group size) */
    int64_t visible_pairs;       /* visible (query, key) pairs per head */
    int32_t head_dim_padded;     /* D rounded up to the MMA k-granule (16) */
    int32_t tile_q, tile_k;
} bca_plan_info;

/* Compile the mask and build a plan: validates the problem, classifies every
 * (128 x 128) tile as empty / full / partial (with a bitmask), orders the forward
 * work items longest-first by visible area (the load-balancing idea of the pages'
 * dispatch solver: balance mask area, MAGI-1 research notes, "Infra > MagiAttention
 * > Dispatch solver"), and, unless BCA_PLAN_HOST_ONLY, uploads the metadata to the
 * current device.  On success *out owns everything; on failure *out is NULL. */
int bca_plan_create(const bca_problem *problem, bca_plan_t *out);
void bca_plan_destroy(bca_plan_t plan);
int bca_plan_get_info(bca_plan_t plan, bca_plan_info *info);

/* Expand the compiled tiles of query rows [row_begin, row_end) back into a dense
 * coverage map: out[(i - row_begin) * Nk + j] = number of compiled tiles that
 * mark pair (i, j) visible (0 or 1 for a correct plan).  Host only. */
int bca_plan_expand_rows(bca_plan_t plan, int64_t row_begin, int64_t row_end, uint8_t *out);

/* The same from the backward's transposed tables (for each key tile, the runs of
 * query tiles that see it), for keys [key_begin, key_end):
 * out[(j - key_begin) * Nq + i].  Host only. */
int bca_plan_expand_cols(bca_plan_t plan, int64_t key_begin, int64_t key_end, uint8_t *out);

/* Streaming reuse of a plan (MAGI-1 research notes, "Inference tricks > KV Cache": the
 * denoising window slides one chunk at a time).  Replace the plan's videos by `videos`
 * that differ only in t0 (same count, chunks, frames, height, width): the mask, tiles and
 * work items are unchanged and only the new tokens' positions and RoPE tables are
 * rewritten (cudaMemcpyAsync on `stream`, after any launch already queued there; the
 * host arguments may be freed on return).  Tables are stored relative to the smallest t0,
 * so shifting every t0 by the same amount keeps their size.  The table layout (where the
 * t, h and w sections start, and its size) is fixed when the plan is created: videos may
 * move by different amounts as long as the span of frames they cover is not longer than
 * the plan's first one; a longer span returns BCA_ERR_UNSUPPORTED and changes nothing.
 * Launches captured in a CUDA graph keep working: they read the rewritten positions,
 * tables and first frame (used by the RoPE-base gradient of bca_bwd_ex) in place.
 * Returns BCA_ERR_INVALID_ARGUMENT for a changed geometry or a negative t0. */
int bca_plan_update_positions(bca_plan_t plan, const bca_video *videos, int num_videos, void *stream);

/* Bytes of caller-provided device workspace a pass needs (16-byte aligned).  The
 * forward's size covers both operand formats: the bf16/fp16 tile images, or for
 * BCA_FWD_FP8_E4M3 plans the smaller e4m3 images plus one float of max|V| per KV head. */
size_t bca_workspace_bytes(bca_plan_t plan, int pass);

/* Forward.  q, k, v, k_cache, v_cache: bf16 (k_cache fp16 for BCA_CACHE_K_FP16 plans;
 * k_cache/v_cache NULL iff Nc == 0);
 * q_gain, k_gain: fp32 [D] QK-Norm gains or NULL (= ones); o: bf16 or fp32
 * (BCA_O_FP32) [Nq][Hq][D]; lse: fp32 [Hq][Nq]; workspace: bca_workspace_bytes(FWD)
 * bytes; stream: a cudaStream_t (NULL = legacy default stream). */
int bca_fwd(bca_plan_t plan, const void *q, const void *k, const void *v,
            const void *k_cache, const void *v_cache, const float *q_gain,
            const float *k_gain, void *o, float *lse, void *workspace, void *stream);

/* Forward without a caller-provided workspace, for callers that may not allocate
 * device memory themselves: for example a plug-in running inside a host process
 * whose allocator owns all device memory and forbids raw allocations from library
 * code, or a C caller with no allocator of its own on this path.  (The pages have
 * no counterpart: this is a property of the library, not of the method.)
 *
 * Same arguments, layouts and results as bca_fwd, minus `workspace`.  The scratch
 * that bca_fwd takes from the workspace (the K-hat and V tile images) lives instead
 * in one file-scope device array of BCA_STATIC_WORKSPACE_BYTES that every GPU which
 * loads the library holds until the process exits.  The call allocates nothing.
 *  - Limit: problems whose bca_workspace_bytes(plan, BCA_PASS_FWD) exceeds
 *    BCA_STATIC_WORKSPACE_BYTES are rejected with BCA_ERR_TOO_LARGE, before any
 *    launch.  (16 MiB holds, e.g., 6144 keys x 8 KV heads at head_dim 48.)
 *  - The array occupies BCA_STATIC_WORKSPACE_BYTES on every GPU on which the library's
 *    module is loaded, whether or not this entry point is ever called.
 *  - The plan must belong to the current device (the one it was created on), else the
 *    call returns BCA_ERR_INVALID_ARGUMENT.
 *  - The first call on a device looks up the array's device address once (with
 *    that device current); make that first call before any stream capture begins.
 *    The address is kept for the life of the process: after a cudaDeviceReset (or any
 *    other teardown of the device's primary context) it is stale, so do not call this
 *    entry point again in that process after such a reset.
 *  - Every call on a device shares the one array and leaves its contents behind.
 *    Each call rewrites every byte it reads before reading it, so nothing needs to
 *    start at zero, but calls whose kernels overlap on the GPU (other streams, or
 *    other threads) race on it: serialise them.
 *  - Per-kernel profiling (bca_profile_enable) creates CUDA events; the call
 *    returns BCA_ERR_INVALID_ARGUMENT while it is enabled on the plan. */
#define BCA_STATIC_WORKSPACE_BYTES (16u << 20)
int bca_fwd_static_workspace(bca_plan_t plan, const void *q, const void *k, const void *v,
                             const void *k_cache, const void *v_cache, const float *q_gain,
                             const float *k_gain, void *o, float *lse, void *stream);

/* Backward.  Same q ... k_gain as bca_fwd; o and lse: the forward's outputs; dout:
 * bf16 [Nq][Hq][D] upstream gradient of O.  Outputs (fp32): dq [Nq][Hq][D],
 * dk, dv [Nq][Hkv][D] (new tokens, through QK-Norm and RoPE), dk_cache, dv_cache
 * [Nc][Hkv][D] (cache keys are used as given, so their gradient is taken at the
 * rotated keys; NULL = not wanted).  workspace: bca_workspace_bytes(BWD) bytes.
 * dk, dv, dk_cache and dv_cache are reduced in a fixed order (bit-reproducible run to
 * run); dq is accumulated with atomics, so its last bits may vary between runs, unless
 * the plan was created with BCA_DQ_DETERMINISTIC. */
int bca_bwd(bca_plan_t plan, const void *q, const void *k, const void *v,
            const void *k_cache, const void *v_cache, const float *q_gain,
            const float *k_gain, const void *o, const float *lse, const void *dout,
            float *dq, float *dk, float *dv, float *dk_cache, float *dv_cache,
            void *workspace, void *stream);

/* bca_bwd plus the gradients of the prologue's parameters (MAGI-1 research notes,
 * "Autoregressive denoising DiT": QK-Norm, and 3D RoPE with a learnable base frequency):
 *   dq_gain    : fp32 [D], dL/d(q_gain), summed over every query row and head;
 *   dk_gain    : fp32 [D], dL/d(k_gain), summed over every new key row and KV head (cache
 *                keys are given post-prologue, so they do not depend on the gain);
 *   drope_base : fp32 [3], dL/d(rope_base[t, h, w]), summed over Q and new K rows.
 * Any of the three may be NULL (not computed); non-NULL ones are overwritten (4-byte
 * aligned).  The sums are formed with atomic adds, so their last bits may differ between
 * runs.  accumulate != 0 adds dq, dk, dv, dk_cache and dv_cache into the given arrays
 * instead of overwriting them (the three parameter gradients are still overwritten): the
 * gradients of a problem whose keys are split over several plans are the sums of the
 * plans' gradients, each plan given the O and LSE of the whole problem.  Everything else
 * is as bca_bwd, which is this call with the three pointers NULL and accumulate = 0. */
int bca_bwd_ex(bca_plan_t plan, const void *q, const void *k, const void *v,
               const void *k_cache, const void *v_cache, const float *q_gain,
               const float *k_gain, const void *o, const float *lse, const void *dout,
               float *dq, float *dk, float *dv, float *dk_cache, float *dv_cache,
               float *dq_gain, float *dk_gain, float *drope_base, int accumulate, void *workspace,
               void *stream);

/* O and LSE of one problem from two partial attentions over disjoint key subsets (the
 * Flex-Flash-Attention merge of partial results by their log-sum-exps: MAGI-1 research
 * notes, "Infra > MagiAttention"), so that context parallelism can attend to the keys a
 * rank holds while the borrowed ones are in flight.  o_a, o_b: fp32 [Nq][Hq][D] (plans
 * with BCA_O_FP32); lse_a, lse_b, lse: fp32 [Hq][Nq] (natural log, -inf = no key);
 * o: [Nq][Hq][D] in this plan's O type.  With m = max(lse_a, lse_b) and w = exp(lse - m):
 * O = (w_a O_a + w_b O_b) / (w_a + w_b), LSE = m + log(w_a + w_b); rows with no key in
 * either part get O = 0, LSE = -inf.  Sizes from the plan (Nq, Hq, D). */
int bca_attn_merge(bca_plan_t plan, const float *o_a, const float *lse_a, const float *o_b,
                   const float *lse_b, void *o, float *lse, void *stream);

/* The key prologue of bca_fwd (QK-Norm + 3D RoPE at the plan's positions of its new
 * tokens) as a stand-alone pass, and its backward.  Used by context parallelism: the
 * rank that owns a token computes its post-prologue key once and sends it to the ranks
 * whose queries see it (there it is a cache key); the gradients they return w.r.t. that
 * key are mapped back through the prologue by the owner (MAGI-1 research notes,
 * "Infra > MagiAttention": group-cast and group-reduce).
 *   k      : bf16 [Nq][Hkv][D], the plan's new tokens' raw keys; k_gain: fp32 [D] or NULL;
 *   k_hat  : bf16 [Nq][Hkv][D] out (RNE of the fp32 result; fp16 for BCA_CACHE_K_FP16 plans);
 *   dk_hat : fp32 [Nq][Hkv][D], dL/dk_hat;  dk: fp32 [Nq][Hkv][D] out, overwritten, or
 *            added to when accumulate != 0.
 * 16-byte aligned pointers; asynchronous on `stream`. */
int bca_k_prologue(bca_plan_t plan, const void *k, const float *k_gain, void *k_hat, void *stream);
int bca_k_prologue_bwd(bca_plan_t plan, const void *k, const float *k_gain, const float *dk_hat, float *dk,
                       int accumulate, void *stream);

/* Kernel kinds for per-kernel timing */
#define BCA_KERNEL_KV_IMAGE 0      /* K-hat prologue + K/V tile images */
#define BCA_KERNEL_FWD 1           /* attention forward */
#define BCA_KERNEL_BWD_PREP 2      /* Q-hat / dO images, LSE, Dsum */
#define BCA_KERNEL_BWD_KV_IMAGE 3  /* K-hat / V images for the backward */
#define BCA_KERNEL_BWD 4           /* attention backward */
#define BCA_KERNEL_BWD_DQ 5        /* dQ prologue backward */
#define BCA_KERNEL_BWD_DQ_PASS 6   /* deterministic dQ pass (BCA_DQ_DETERMINISTIC) */
#define BCA_KERNEL_COUNT 7

/* Per-kernel device timing, a tracing aid.  While enabled (enable != 0), every
 * kernel that bca_fwd or bca_bwd launches for this plan is bracketed by two CUDA events
 * recorded on its stream.  bca_profile_read waits for those events and returns, for
 * one kernel kind, the number of launches and their summed device time in ms since
 * the last read (or enable), then forgets them.  Disabled by default. */
int bca_profile_enable(bca_plan_t plan, int enable);
int bca_profile_read(bca_plan_t plan, int kernel, int64_t *launches, double *total_ms);

/* Device status word of the plan (timeouts recorded by its kernels).  Synchronises
 * the stream, returns BCA_OK or the recorded error, and clears it. */
int bca_status(bca_plan_t plan, void *stream);

const char *bca_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* BCA_H */
