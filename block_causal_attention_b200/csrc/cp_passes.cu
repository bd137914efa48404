// Passes for context parallelism.  (1) The key prologue (QK-Norm + 3D RoPE) and its
// backward over the rows of a plan's new tokens, as stand-alone passes.  (2) The merge of
// two partial attentions over disjoint key subsets by their log-sum-exps, so that a rank
// can attend to the keys it holds while the borrowed ones are still in flight.  The attention kernels fuse these steps; the passes
// exist for context-parallel use, where a key row's post-prologue value K-hat is computed
// once by the rank that owns the token and sent to the ranks that attend to it, and the
// gradients those ranks return for K-hat are mapped back through the prologue by the
// owner (MAGI-1 research notes, "Infra > MagiAttention": dispatch, group-cast and
// group-reduce of key/value chunks).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.hpp"
#include "prologue.cuh"
#include "sm100.cuh"

namespace bca {

namespace {

struct RowArgs {
    const __nv_bfloat16 *k;
    const float *k_gain;
    const uint32_t *pos;
    const float *rope;
    int32_t off0, off1, off2;
    int64_t rows;  // tokens * heads
    int heads;
    float eps;
    int prologue;            // 0: keys given post-prologue (BCA_NO_PROLOGUE): both passes copy
    int khat_f16;            // write K-hat as fp16 (BCA_CACHE_K_FP16), else bf16
    __nv_bfloat16 *k_hat;    // forward output
    const float *dk_hat;     // backward input
    float *dk;               // backward output
    int accumulate;
};

template <int D>
__global__ void __launch_bounds__(128) k_prologue_kernel(RowArgs a) {
    const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= a.rows) return;
    const int64_t t = row / a.heads;
    float x[D];
    load_row_bf16<D>(a.k + (size_t)row * D, x);
    qk_prologue<D>(x, __ldg(a.pos + t), a.k_gain, a.rope, a.off0, a.off1, a.off2, a.eps, 1.0f, a.prologue != 0);
    uint4 *dst = reinterpret_cast<uint4 *>(a.k_hat + (size_t)row * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) dst[c] = a.khat_f16 ? pack_chunk_f16<D>(x, c) : pack_chunk_bf16<D>(x, c);
}

template <int D>
__global__ void __launch_bounds__(128) k_prologue_bwd_kernel(RowArgs a) {
    const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= a.rows) return;
    const int64_t t = row / a.heads;
    float x[D], g[D];
    load_row_bf16<D>(a.k + (size_t)row * D, x);
    const float4 *src = reinterpret_cast<const float4 *>(a.dk_hat + (size_t)row * D);
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
        const float4 f = src[c];
        g[4 * c] = f.x;
        g[4 * c + 1] = f.y;
        g[4 * c + 2] = f.z;
        g[4 * c + 3] = f.w;
    }
    qk_prologue_bwd<D>(x, g, __ldg(a.pos + t), a.k_gain, a.rope, a.off0, a.off1, a.off2, a.eps, a.prologue != 0);
    float4 *dst = reinterpret_cast<float4 *>(a.dk + (size_t)row * D);
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
        float4 v = make_float4(g[4 * c], g[4 * c + 1], g[4 * c + 2], g[4 * c + 3]);
        if (a.accumulate) {
            const float4 o = dst[c];
            v.x += o.x;
            v.y += o.y;
            v.z += o.z;
            v.w += o.w;
        }
        dst[c] = v;
    }
}

RowArgs row_args(const Plan &P, const void *k, const float *k_gain) {
    RowArgs a{};
    a.k = static_cast<const __nv_bfloat16 *>(k);
    a.k_gain = k_gain;
    a.pos = P.d_pos;
    a.rope = P.d_rope;
    a.off0 = P.rope_axis_off[0];
    a.off1 = P.rope_axis_off[1];
    a.off2 = P.rope_axis_off[2];
    a.rows = P.nq * P.hkv;
    a.heads = P.hkv;
    a.eps = P.eps;
    a.prologue = (P.flags & BCA_NO_PROLOGUE) ? 0 : 1;
    a.khat_f16 = (P.flags & BCA_CACHE_K_FP16) ? 1 : 0;
    return a;
}

template <int D>
int launch_rows(const RowArgs &a, bool backward, cudaStream_t stream) {
    const unsigned blocks = (unsigned)((a.rows + 127) / 128);
    if (backward)
        k_prologue_bwd_kernel<D><<<blocks, 128, 0, stream>>>(a);
    else
        k_prologue_kernel<D><<<blocks, 128, 0, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? BCA_OK : BCA_ERR_CUDA;
}

int dispatch_rows(const Plan &P, const RowArgs &a, bool backward, cudaStream_t stream) {
    if (a.rows == 0) return BCA_OK;
    switch (P.d) {
        case 24: return launch_rows<24>(a, backward, stream);
        case 32: return launch_rows<32>(a, backward, stream);
        case 48: return launch_rows<48>(a, backward, stream);
        default: return BCA_ERR_UNSUPPORTED;
    }
}

struct MergeArgs {
    const float *o_a, *lse_a, *o_b, *lse_b;
    void *o;
    float *lse;
    int o_fp32;
    int64_t nq;
    int hq;
};

// one thread per (query, head): with m = max(lse_a, lse_b), w = exp(lse - m):
// O = (w_a O_a + w_b O_b) / (w_a + w_b), LSE = m + log(w_a + w_b); no visible key in
// either part gives O = 0, LSE = -inf
template <int D>
__global__ void __launch_bounds__(128) attn_merge_kernel(MergeArgs a) {
    const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int h = blockIdx.y;
    if (q >= a.nq) return;
    const size_t row = (size_t)q * a.hq + h;
    const size_t li = (size_t)h * a.nq + q;
    const float la = a.lse_a[li], lb = a.lse_b[li];
    const float m = fmaxf(la, lb);
    float wa = 0.f, wb = 0.f, lse = -INFINITY;
    if (m > -INFINITY) {
        wa = la > -INFINITY ? __expf(la - m) : 0.f;
        wb = lb > -INFINITY ? __expf(lb - m) : 0.f;
        const float s = wa + wb;
        lse = m + __logf(s);
        wa /= s;
        wb /= s;
    }
    float o[D];
    const float4 *pa = reinterpret_cast<const float4 *>(a.o_a + row * D);
    const float4 *pb = reinterpret_cast<const float4 *>(a.o_b + row * D);
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
        const float4 x = pa[c], y = pb[c];
        o[4 * c] = wa * x.x + wb * y.x;
        o[4 * c + 1] = wa * x.y + wb * y.y;
        o[4 * c + 2] = wa * x.z + wb * y.z;
        o[4 * c + 3] = wa * x.w + wb * y.w;
    }
    if (a.o_fp32) {
        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.o) + row * D);
#pragma unroll
        for (int c = 0; c < D / 4; ++c) dst[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
    } else {
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.o) + row * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) dst[c] = pack_chunk_bf16<D>(o, c);
    }
    a.lse[li] = lse;
}

template <int D>
int launch_merge(const MergeArgs &a, cudaStream_t stream) {
    attn_merge_kernel<D><<<dim3((unsigned)((a.nq + 127) / 128), (unsigned)a.hq), 128, 0, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? BCA_OK : BCA_ERR_CUDA;
}

}  // namespace

int launch_attn_merge(const Plan &P, const float *o_a, const float *lse_a, const float *o_b, const float *lse_b,
                      void *o, float *lse, cudaStream_t stream) {
    if (P.nq == 0) return BCA_OK;
    MergeArgs a{o_a, lse_a, o_b, lse_b, o, lse, (P.flags & BCA_O_FP32) ? 1 : 0, P.nq, P.hq};
    switch (P.d) {
        case 24: return launch_merge<24>(a, stream);
        case 32: return launch_merge<32>(a, stream);
        case 48: return launch_merge<48>(a, stream);
        default: return BCA_ERR_UNSUPPORTED;
    }
}

int launch_k_prologue(const Plan &P, const void *k, const float *k_gain, void *k_hat, cudaStream_t stream) {
    RowArgs a = row_args(P, k, k_gain);
    a.k_hat = static_cast<__nv_bfloat16 *>(k_hat);
    return dispatch_rows(P, a, false, stream);
}

int launch_k_prologue_bwd(const Plan &P, const void *k, const float *k_gain, const float *dk_hat, float *dk,
                          int accumulate, cudaStream_t stream) {
    RowArgs a = row_args(P, k, k_gain);
    a.dk_hat = dk_hat;
    a.dk = dk;
    a.accumulate = accumulate;
    return dispatch_rows(P, a, true, stream);
}

}  // namespace bca
