// Launch interface between the C ABI (api.cpp) and the CUDA kernels.
#pragma once

#include <cuda_runtime.h>

#include "plan.hpp"

namespace bca {

// status-word bits written by kernels
constexpr int kStatusTimeout = 0x1;

struct FwdIO {
    const void *q, *k, *v, *k_cache, *v_cache;
    const float *q_gain, *k_gain;
    void *o;
    float *lse;
    void *workspace;
};

struct BwdIO {
    const void *q, *k, *v, *k_cache, *v_cache;
    const float *q_gain, *k_gain;
    const void *o;
    const float *lse;
    const void *dout;
    float *dq, *dk, *dv, *dk_cache, *dv_cache;
    void *workspace;
    float *dq_gain, *dk_gain, *drope_base;  // optional parameter gradients (NULL = not wanted)
    int accumulate;                         // add dq, dk, dv, dk_cache, dv_cache into the outputs
};

// Bytes of each K-hat / V image (all KV heads, all k-tiles), 256-byte rounded.
size_t kv_image_bytes(const Plan &plan);
size_t fwd_workspace_bytes(const Plan &plan);
// Bytes of each Q-hat / dO image (all query heads, all q-tiles) and of each padded
// per-query vector (LSE, Dsum); and the whole backward workspace.
size_t q_image_bytes(const Plan &plan);
size_t q_vector_bytes(const Plan &plan);
// Bytes of the backward's fp32 dQ-hat accumulator ([Hq][query tile][2][128][Dpad / 2]).
size_t dq_acc_bytes(const Plan &plan);
size_t bwd_workspace_bytes(const Plan &plan);

// K prologue over the plan's new tokens (bf16 K-hat rows) and its backward
// (dk = or += J^T dk_hat), for context-parallel exchange of post-prologue keys.
// O and LSE of one problem from the O (fp32) and LSE of two disjoint key subsets.
int launch_attn_merge(const Plan &plan, const float *o_a, const float *lse_a, const float *o_b, const float *lse_b,
                      void *o, float *lse, cudaStream_t stream);
int launch_k_prologue(const Plan &plan, const void *k, const float *k_gain, void *k_hat, cudaStream_t stream);
int launch_k_prologue_bwd(const Plan &plan, const void *k, const float *k_gain, const float *dk_hat, float *dk,
                          int accumulate, cudaStream_t stream);

// One-time per-plan kernel attributes (dynamic shared memory), on the plan's device.
int prepare_fwd(const Plan &plan);
int prepare_bwd(const Plan &plan);

// Bracket a launch with events when the plan is profiling (no-op otherwise).
struct ProfScope {
    Plan &plan;
    int kernel;
    cudaStream_t stream;
    cudaEvent_t start = nullptr;
    ProfScope(Plan &p, int k, cudaStream_t s);
    ~ProfScope();
};

// Enqueue the forward on `stream`.  Returns BCA_OK or BCA_ERR_CUDA.
int launch_fwd(Plan &plan, const FwdIO &io, cudaStream_t stream);
// Enqueue the backward on `stream`.
int launch_bwd(Plan &plan, const BwdIO &io, cudaStream_t stream);

}  // namespace bca
