// C ABI of libbca.so: argument checks, plan lifetime, launches.  See include/bca.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <new>
#include <vector>

#include "kernels.hpp"
#include "plan.hpp"

namespace bca {

ProfScope::ProfScope(Plan &p, int k, cudaStream_t s) : plan(p), kernel(k), stream(s) {
    if (!plan.profiling) return;
    if (cudaEventCreate(&start) != cudaSuccess) {
        start = nullptr;
        return;
    }
    cudaEventRecord(start, stream);
}

ProfScope::~ProfScope() {
    if (!start) return;
    cudaEvent_t stop = nullptr;
    if (cudaEventCreate(&stop) != cudaSuccess) {
        cudaEventDestroy(start);
        return;
    }
    cudaEventRecord(stop, stream);
    plan.prof.push_back({kernel, start, stop});
}

}  // namespace bca

namespace {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Upload the plan's tables into one device allocation owned by the plan.
int upload(bca::Plan &P) {
    using namespace bca;
    const size_t s_runoff = round256(P.run_off.size() * sizeof(int32_t));
    const size_t s_runs = round256(std::max<size_t>(1, P.runs.size()) * sizeof(Run));
    const size_t s_masks = round256(std::max<size_t>(1, P.masks.size()) * sizeof(uint32_t));
    const size_t s_items = round256(std::max<size_t>(1, P.items.size()) * sizeof(Item));
    const size_t s_pos = round256(std::max<size_t>(1, P.pos.size()) * sizeof(uint32_t));
    const size_t s_rope = round256(std::max<size_t>(1, P.rope.size()) * sizeof(float));
    const size_t s_coloff = round256(P.col_off.size() * sizeof(int32_t));
    const size_t s_colruns = round256(std::max<size_t>(1, P.col_runs.size()) * sizeof(Run));
    const size_t s_bitems = round256(std::max<size_t>(1, P.bwd_items.size()) * sizeof(int32_t));
    const size_t s_status = 256;  // the status word, then rope_tbase at byte 128
    const size_t total = s_runoff + s_runs + s_masks + s_items + s_pos + s_rope + s_coloff + s_colruns +
                         s_bitems + s_status;
    if (cudaGetDevice(&P.device) != cudaSuccess) return BCA_ERR_CUDA;
    void *blob = nullptr;
    if (cudaMalloc(&blob, total) != cudaSuccess) return BCA_ERR_NO_MEMORY;
    P.d_blob = blob;
    uint8_t *b = static_cast<uint8_t *>(blob);
    size_t off = 0;
    auto put = [&](const void *src, size_t bytes, size_t slot) -> void * {
        void *dst = b + off;
        off += slot;
        if (bytes && cudaMemcpy(dst, src, bytes, cudaMemcpyHostToDevice) != cudaSuccess) return nullptr;
        return dst;
    };
    P.d_run_off = static_cast<const int32_t *>(put(P.run_off.data(), P.run_off.size() * sizeof(int32_t), s_runoff));
    P.d_runs = static_cast<const Run *>(put(P.runs.data(), P.runs.size() * sizeof(Run), s_runs));
    P.d_masks = static_cast<const uint32_t *>(put(P.masks.data(), P.masks.size() * sizeof(uint32_t), s_masks));
    P.d_items = static_cast<const Item *>(put(P.items.data(), P.items.size() * sizeof(Item), s_items));
    P.d_pos = static_cast<const uint32_t *>(put(P.pos.data(), P.pos.size() * sizeof(uint32_t), s_pos));
    P.d_rope = static_cast<const float *>(put(P.rope.data(), P.rope.size() * sizeof(float), s_rope));
    P.d_col_off = static_cast<const int32_t *>(put(P.col_off.data(), P.col_off.size() * sizeof(int32_t), s_coloff));
    P.d_col_runs = static_cast<const Run *>(put(P.col_runs.data(), P.col_runs.size() * sizeof(Run), s_colruns));
    P.d_bwd_items =
        static_cast<const int32_t *>(put(P.bwd_items.data(), P.bwd_items.size() * sizeof(int32_t), s_bitems));
    P.d_status = static_cast<int *>(static_cast<void *>(b + off));
    P.d_tbase = static_cast<int32_t *>(static_cast<void *>(b + off + 128));
    if (!P.d_run_off || !P.d_runs || !P.d_masks || !P.d_items || !P.d_pos || !P.d_rope || !P.d_col_off ||
        !P.d_col_runs || !P.d_bwd_items)
        return BCA_ERR_CUDA;
    if (cudaMemset(P.d_status, 0, sizeof(int)) != cudaSuccess) return BCA_ERR_CUDA;
    if (cudaMemcpy(P.d_tbase, &P.rope_tbase, sizeof(int32_t), cudaMemcpyHostToDevice) != cudaSuccess)
        return BCA_ERR_CUDA;
    P.rope_capacity = P.rope.size();
    int rc = prepare_fwd(P);
    if (rc == BCA_OK) rc = prepare_bwd(P);
    return rc;
}

int check_device(const bca::Plan &P) {
    if (P.flags & BCA_PLAN_HOST_ONLY) return BCA_ERR_HOST_ONLY_PLAN;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return BCA_ERR_CUDA;
    if (dev != P.device) return BCA_ERR_INVALID_ARGUMENT;
    return BCA_OK;
}

}  // namespace

extern "C" {

int bca_plan_create(const bca_problem *problem, bca_plan_t *out) {
    if (!out) return BCA_ERR_INVALID_ARGUMENT;
    *out = nullptr;
    bca_plan_s *h = new (std::nothrow) bca_plan_s();
    if (!h) return BCA_ERR_NO_MEMORY;
    int rc = bca::validate_problem(problem, h->plan);
    if (rc == BCA_OK) {
        try {
            rc = bca::compile_plan(h->plan);
        } catch (const std::bad_alloc &) {
            rc = BCA_ERR_NO_MEMORY;
        }
    }
    if (rc == BCA_OK && !(h->plan.flags & BCA_PLAN_HOST_ONLY)) rc = upload(h->plan);
    if (rc != BCA_OK) {
        bca_plan_destroy(h);
        return rc;
    }
    *out = h;
    return BCA_OK;
}

int bca_plan_update_positions(bca_plan_t plan, const bca_video *videos, int num_videos, void *stream) {
    if (!plan || num_videos < 0 || (num_videos > 0 && !videos)) return BCA_ERR_INVALID_ARGUMENT;
    bca::Plan &P = plan->plan;
    if ((size_t)num_videos != P.videos.size()) return BCA_ERR_INVALID_ARGUMENT;
    for (int i = 0; i < num_videos; ++i) {
        const bca_video &a = videos[i], &b = P.videos[i];
        if (a.num_chunks != b.num_chunks || a.frames != b.frames || a.height != b.height || a.width != b.width)
            return BCA_ERR_INVALID_ARGUMENT;
        if (a.t0 < 0 || (int64_t)a.t0 + (int64_t)a.num_chunks * a.frames > INT32_MAX) return BCA_ERR_INVALID_ARGUMENT;
    }
    const bool on_device = !(P.flags & BCA_PLAN_HOST_ONLY);
    if (on_device) {
        int rc = check_device(P);
        if (rc != BCA_OK) return rc;
    }
    bca::Plan next;  // positions only: build into a scratch plan, then commit
    next.videos.assign(videos, videos + num_videos);
    next.nq = P.nq;
    next.d = P.d;
    for (int a = 0; a < 3; ++a) next.base[a] = P.base[a];
    int rc;
    try {
        // on the device the table keeps the plan's layout (a t range that grew does not fit)
        rc = bca::build_positions(next, on_device ? &P : nullptr);
    } catch (const std::bad_alloc &) {
        rc = BCA_ERR_NO_MEMORY;
    }
    if (rc != BCA_OK) return rc;
    if (on_device) {
        cudaStream_t s = static_cast<cudaStream_t>(stream);
        // pageable sources: the copies are staged before return, ordered on the stream
        if (cudaMemcpyAsync(const_cast<uint32_t *>(P.d_pos), next.pos.data(), next.pos.size() * sizeof(uint32_t),
                            cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(const_cast<float *>(P.d_rope), next.rope.data(), next.rope.size() * sizeof(float),
                            cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(P.d_tbase, &next.rope_tbase, sizeof(int32_t), cudaMemcpyHostToDevice, s) != cudaSuccess)
            return BCA_ERR_CUDA;
    }
    P.videos.swap(next.videos);
    P.pos.swap(next.pos);
    P.rope.swap(next.rope);
    P.rope_tbase = next.rope_tbase;
    for (int a = 0; a < 3; ++a) P.rope_axis_off[a] = next.rope_axis_off[a];
    return BCA_OK;
}

static void drop_profile(bca::Plan &P) {
    for (auto &r : P.prof) {
        cudaEventDestroy(static_cast<cudaEvent_t>(r.start));
        cudaEventDestroy(static_cast<cudaEvent_t>(r.stop));
    }
    P.prof.clear();
}

void bca_plan_destroy(bca_plan_t plan) {
    if (!plan) return;
    drop_profile(plan->plan);
    if (plan->plan.d_blob) {
        int cur = -1;
        cudaGetDevice(&cur);
        if (cur != plan->plan.device) cudaSetDevice(plan->plan.device);
        cudaFree(plan->plan.d_blob);
        if (cur >= 0 && cur != plan->plan.device) cudaSetDevice(cur);
    }
    delete plan;
}

int bca_plan_get_info(bca_plan_t plan, bca_plan_info *info) {
    if (!plan || !info) return BCA_ERR_INVALID_ARGUMENT;
    const bca::Plan &P = plan->plan;
    std::memset(info, 0, sizeof(*info));
    info->num_q = P.nq;
    info->num_k = P.nk;
    info->num_cache = P.nc;
    info->num_q_tiles = P.nqt;
    info->num_k_tiles = P.nkt;
    info->num_runs = (int64_t)P.runs.size();
    info->num_full_tiles = P.nfull;
    info->num_partial_tiles = P.npartial;
    info->num_items = (int64_t)P.items.size();
    info->visible_pairs = P.visible_pairs;
    info->head_dim_padded = P.dpad;
    info->tile_q = bca::kTileQ;
    info->tile_k = bca::kTileK;
    return BCA_OK;
}

int bca_plan_expand_rows(bca_plan_t plan, int64_t row_begin, int64_t row_end, uint8_t *out) {
    if (!plan) return BCA_ERR_INVALID_ARGUMENT;
    return bca::expand_rows(plan->plan, row_begin, row_end, out);
}

int bca_plan_expand_cols(bca_plan_t plan, int64_t key_begin, int64_t key_end, uint8_t *out) {
    if (!plan) return BCA_ERR_INVALID_ARGUMENT;
    return bca::expand_cols(plan->plan, key_begin, key_end, out);
}

size_t bca_workspace_bytes(bca_plan_t plan, int pass) {
    if (!plan) return 0;
    if (pass == BCA_PASS_FWD) return bca::fwd_workspace_bytes(plan->plan);
    if (pass == BCA_PASS_BWD) return bca::bwd_workspace_bytes(plan->plan);
    return 0;
}

int bca_fwd(bca_plan_t plan, const void *q, const void *k, const void *v, const void *k_cache,
            const void *v_cache, const float *q_gain, const float *k_gain, void *o, float *lse,
            void *workspace, void *stream) {
    if (!plan) return BCA_ERR_INVALID_ARGUMENT;
    bca::Plan &P = plan->plan;
    int rc = check_device(P);
    if (rc != BCA_OK) return rc;
    if (P.nq == 0) return BCA_OK;
    if (!q || !k || !v || !o || !lse || !workspace) return BCA_ERR_INVALID_ARGUMENT;
    if (P.nc > 0 && (!k_cache || !v_cache)) return BCA_ERR_INVALID_ARGUMENT;
    if ((P.flags & BCA_NO_PROLOGUE) && (q_gain || k_gain)) return BCA_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {q, k, v, k_cache, v_cache, q_gain, k_gain, o, lse, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return BCA_ERR_MISALIGNED;
    bca::FwdIO io{q, k, v, k_cache, v_cache, q_gain, k_gain, o, lse, workspace};
    return bca::launch_fwd(P, io, static_cast<cudaStream_t>(stream));
}

int bca_bwd_ex(bca_plan_t plan, const void *q, const void *k, const void *v, const void *k_cache,
               const void *v_cache, const float *q_gain, const float *k_gain, const void *o, const float *lse,
               const void *dout, float *dq, float *dk, float *dv, float *dk_cache, float *dv_cache,
               float *dq_gain, float *dk_gain, float *drope_base, int accumulate, void *workspace, void *stream) {
    if (!plan) return BCA_ERR_INVALID_ARGUMENT;
    bca::Plan &P = plan->plan;
    if (P.flags & BCA_FWD_FP8_E4M3) return BCA_ERR_UNSUPPORTED;  // the e4m3 path is forward only
    int rc = check_device(P);
    if (rc != BCA_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (P.nq == 0) {
        // no query: every gradient is zero
        const size_t cb = (size_t)P.nc * P.hkv * P.d * sizeof(float);
        if (!accumulate && dk_cache && cudaMemsetAsync(dk_cache, 0, cb, s) != cudaSuccess) return BCA_ERR_CUDA;
        if (!accumulate && dv_cache && cudaMemsetAsync(dv_cache, 0, cb, s) != cudaSuccess) return BCA_ERR_CUDA;
        if (dq_gain && cudaMemsetAsync(dq_gain, 0, P.d * sizeof(float), s) != cudaSuccess) return BCA_ERR_CUDA;
        if (dk_gain && cudaMemsetAsync(dk_gain, 0, P.d * sizeof(float), s) != cudaSuccess) return BCA_ERR_CUDA;
        if (drope_base && cudaMemsetAsync(drope_base, 0, 3 * sizeof(float), s) != cudaSuccess) return BCA_ERR_CUDA;
        return BCA_OK;
    }
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace) return BCA_ERR_INVALID_ARGUMENT;
    if ((P.flags & BCA_NO_PROLOGUE) && (q_gain || k_gain || dq_gain || dk_gain || drope_base))
        return BCA_ERR_INVALID_ARGUMENT;
    if (P.nc > 0 && (!k_cache || !v_cache)) return BCA_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {q, k, v, k_cache, v_cache, q_gain, k_gain, o, lse, dout, dq, dk, dv, dk_cache, dv_cache,
                          workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return BCA_ERR_MISALIGNED;
    const void *pptrs[] = {dq_gain, dk_gain, drope_base};
    for (const void *p : pptrs)
        if (p && !aligned4(p)) return BCA_ERR_MISALIGNED;
    bca::BwdIO io{q,  k,  v,  k_cache,  v_cache,  q_gain,    k_gain,  o,       lse,       dout,      dq,
                  dk, dv, dk_cache, dv_cache, workspace, dq_gain, dk_gain, drope_base, accumulate != 0};
    return bca::launch_bwd(P, io, s);
}

int bca_bwd(bca_plan_t plan, const void *q, const void *k, const void *v, const void *k_cache,
            const void *v_cache, const float *q_gain, const float *k_gain, const void *o, const float *lse,
            const void *dout, float *dq, float *dk, float *dv, float *dk_cache, float *dv_cache,
            void *workspace, void *stream) {
    return bca_bwd_ex(plan, q, k, v, k_cache, v_cache, q_gain, k_gain, o, lse, dout, dq, dk, dv, dk_cache, dv_cache,
                      nullptr, nullptr, nullptr, 0, workspace, stream);
}

int bca_attn_merge(bca_plan_t plan, const float *o_a, const float *lse_a, const float *o_b, const float *lse_b,
                   void *o, float *lse, void *stream) {
    if (!plan) return BCA_ERR_INVALID_ARGUMENT;
    bca::Plan &P = plan->plan;
    int rc = check_device(P);
    if (rc != BCA_OK) return rc;
    if (P.nq == 0) return BCA_OK;
    if (!o_a || !lse_a || !o_b || !lse_b || !o || !lse) return BCA_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {o_a, o_b, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return BCA_ERR_MISALIGNED;
    if (!aligned4(lse_a) || !aligned4(lse_b) || !aligned4(lse)) return BCA_ERR_MISALIGNED;
    return bca::launch_attn_merge(P, o_a, lse_a, o_b, lse_b, o, lse, static_cast<cudaStream_t>(stream));
}

int bca_k_prologue(bca_plan_t plan, const void *k, const float *k_gain, void *k_hat, void *stream) {
    if (!plan) return BCA_ERR_INVALID_ARGUMENT;
    bca::Plan &P = plan->plan;
    int rc = check_device(P);
    if (rc != BCA_OK) return rc;
    if (P.nq == 0) return BCA_OK;
    if (!k || !k_hat) return BCA_ERR_INVALID_ARGUMENT;
    if ((P.flags & BCA_NO_PROLOGUE) && k_gain) return BCA_ERR_INVALID_ARGUMENT;
    if (!aligned16(k) || !aligned16(k_hat) || (k_gain && !aligned16(k_gain))) return BCA_ERR_MISALIGNED;
    return bca::launch_k_prologue(P, k, k_gain, k_hat, static_cast<cudaStream_t>(stream));
}

int bca_k_prologue_bwd(bca_plan_t plan, const void *k, const float *k_gain, const float *dk_hat, float *dk,
                       int accumulate, void *stream) {
    if (!plan) return BCA_ERR_INVALID_ARGUMENT;
    bca::Plan &P = plan->plan;
    int rc = check_device(P);
    if (rc != BCA_OK) return rc;
    if (P.nq == 0) return BCA_OK;
    if (!k || !dk_hat || !dk) return BCA_ERR_INVALID_ARGUMENT;
    if ((P.flags & BCA_NO_PROLOGUE) && k_gain) return BCA_ERR_INVALID_ARGUMENT;
    if (!aligned16(k) || !aligned16(dk_hat) || !aligned16(dk) || (k_gain && !aligned16(k_gain)))
        return BCA_ERR_MISALIGNED;
    return bca::launch_k_prologue_bwd(P, k, k_gain, dk_hat, dk, accumulate, static_cast<cudaStream_t>(stream));
}

int bca_profile_enable(bca_plan_t plan, int enable) {
    if (!plan) return BCA_ERR_INVALID_ARGUMENT;
    drop_profile(plan->plan);
    plan->plan.profiling = enable != 0;
    return BCA_OK;
}

int bca_profile_read(bca_plan_t plan, int kernel, int64_t *launches, double *total_ms) {
    if (!plan || !launches || !total_ms || kernel < 0 || kernel >= BCA_KERNEL_COUNT)
        return BCA_ERR_INVALID_ARGUMENT;
    bca::Plan &P = plan->plan;
    *launches = 0;
    *total_ms = 0.0;
    std::vector<bca::Plan::ProfRecord> keep;
    int rc = BCA_OK;
    for (auto &r : P.prof) {
        if (r.kernel != kernel) {
            keep.push_back(r);
            continue;
        }
        float ms = 0.f;
        cudaEvent_t a = static_cast<cudaEvent_t>(r.start), b = static_cast<cudaEvent_t>(r.stop);
        if (cudaEventSynchronize(b) != cudaSuccess || cudaEventElapsedTime(&ms, a, b) != cudaSuccess)
            rc = BCA_ERR_CUDA;
        *launches += 1;
        *total_ms += ms;
        cudaEventDestroy(a);
        cudaEventDestroy(b);
    }
    P.prof.swap(keep);
    return rc;
}

int bca_status(bca_plan_t plan, void *stream) {
    if (!plan) return BCA_ERR_INVALID_ARGUMENT;
    const bca::Plan &P = plan->plan;
    int rc = check_device(P);
    if (rc != BCA_OK) return rc;
    int h = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&h, P.d_status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return BCA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return BCA_ERR_CUDA;
    if (h == 0) return BCA_OK;
    if (cudaMemsetAsync(P.d_status, 0, sizeof(int), s) != cudaSuccess) return BCA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return BCA_ERR_CUDA;
    return (h & bca::kStatusTimeout) ? BCA_ERR_DEVICE_TIMEOUT : BCA_ERR_CUDA;
}

const char *bca_error_string(int code) {
    switch (code) {
        case BCA_OK: return "ok";
        case BCA_ERR_INVALID_ARGUMENT: return "invalid argument";
        case BCA_ERR_BAD_SLICE: return "bad AttnSlice (out of range, begin > end, or unknown type)";
        case BCA_ERR_UNSUPPORTED: return "unsupported head_dim, head grouping or geometry";
        case BCA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case BCA_ERR_CUDA: return "CUDA runtime error";
        case BCA_ERR_DEVICE_TIMEOUT: return "a device-side wait timed out";
        case BCA_ERR_HOST_ONLY_PLAN: return "plan was built host-only (BCA_PLAN_HOST_ONLY)";
        case BCA_ERR_NO_MEMORY: return "out of memory";
        case BCA_ERR_TOO_LARGE: return "problem needs more scratch than the static workspace holds";
        default: return "unknown error";
    }
}

}  // extern "C"
