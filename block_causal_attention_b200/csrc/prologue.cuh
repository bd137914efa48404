// Device helpers shared by the forward and backward kernels: the QK-Norm + 3D RoPE
// prologue (and its backward) on one (token, head) row held in registers, row loads
// and packing into 16-byte chunks.
//
// QK-Norm and the learnable-base 3D RoPE on Q and K: MAGI-1 research notes
// (zhao9797.github.io), "Autoregressive denoising DiT" bullets; "清华特奖得主团队视频生成AI
// 一夜刷屏" (dakule.com), "3D RoPE" and "QK-Norm and GQA".
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sm100.cuh"

namespace bca {

template <int D>
struct Geo {
    static constexpr int DPAD = (D + 15) / 16 * 16;     // MMA k-granule for bf16 is 16
    static constexpr int PAIRS = (D / 2) / 3;           // RoPE pairs per axis
    static constexpr int TILE_BYTES = 128 * DPAD * 2;   // one K-hat or V tile image
    // 8-bit operands: the MMA k-granule is 32 elements, a core-matrix row 16 elements
    static constexpr int DP8 = (D + 31) / 32 * 32;      // head dim of the e4m3 Q-hat / K-hat images
    static constexpr int K8_TILE_BYTES = 128 * DP8;     // one e4m3 K-hat tile image
    static constexpr int V8_TILE_BYTES = DPAD * 128;    // one e4m3 V^T tile image
};

// ------------------------------------------------------------------ prologue math

// RMS QK-Norm with gain, 3D RoPE at the packed position, then a scale; in place.  With
// apply = false (plans created with BCA_NO_PROLOGUE: the rows are given post-prologue)
// only the scale is applied.
template <int D>
__device__ __forceinline__ void qk_prologue(float (&x)[D], uint32_t pos, const float *gain, const float *rope,
                                            int32_t off0, int32_t off1, int32_t off2, float eps, float scale,
                                            bool apply = true) {
    constexpr int P = Geo<D>::PAIRS;
    if (!apply) {
#pragma unroll
        for (int d = 0; d < D; ++d) x[d] *= scale;
        return;
    }
    float ss = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) ss = fmaf(x[d], x[d], ss);
    const float r = rsqrtf(ss * (1.0f / D) + eps);
#pragma unroll
    for (int d = 0; d < D; ++d) x[d] = x[d] * r * (gain ? __ldg(gain + d) : 1.0f);
    const int32_t p[3] = {(int32_t)(pos >> 16), (int32_t)((pos >> 8) & 255u), (int32_t)(pos & 255u)};
    const int32_t off[3] = {off0, off1, off2};
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        const float2 *tab = reinterpret_cast<const float2 *>(rope) + (size_t)(off[a] + p[a]) * P;
#pragma unroll
        for (int k = 0; k < P; ++k) {
            const float2 cs = __ldg(tab + k);
            const int c0 = 2 * P * a + 2 * k;
            const float y0 = x[c0], y1 = x[c0 + 1];
            x[c0] = y0 * cs.x - y1 * cs.y;
            x[c0 + 1] = y0 * cs.y + y1 * cs.x;
        }
    }
#pragma unroll
    for (int d = 0; d < D; ++d) x[d] *= scale;
}

template <int D>
__device__ __forceinline__ void load_row_bf16(const __nv_bfloat16 *src, float (&x)[D]) {
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        uint4 u = __ldg(s + c);
        const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = __bfloat1622float2(b[e]);
            x[c * 8 + 2 * e] = f.x;
            x[c * 8 + 2 * e + 1] = f.y;
        }
    }
}

// A row of 16-bit values: bf16, or fp16 when f16 (cache keys of plans created with
// BCA_CACHE_K_FP16).
template <int D>
__device__ __forceinline__ void load_row_16(const void *src, bool f16, float (&x)[D]) {
    if (!f16) {
        load_row_bf16<D>(static_cast<const __nv_bfloat16 *>(src), x);
        return;
    }
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        uint4 u = __ldg(s + c);
        const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = __half22float2(h[e]);
            x[c * 8 + 2 * e] = f.x;
            x[c * 8 + 2 * e + 1] = f.y;
        }
    }
}

// Pack values [8c, 8c+8) of x (zero past D) into one 16-byte chunk of fp16.
template <int D>
__device__ __forceinline__ uint4 pack_chunk_f16(const float (&x)[D], int c) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int d0 = c * 8 + 2 * e;
        const float lo = d0 < D ? x[d0] : 0.f;
        const float hi = d0 + 1 < D ? x[d0 + 1] : 0.f;
        w[e] = sm100::pack_f16x2(lo, hi);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Pack values [16c, 16c+16) of x (zero past D), each multiplied by mul, into one
// 16-byte chunk of e4m3.
template <int D>
__device__ __forceinline__ uint4 pack_chunk_e4m3(const float (&x)[D], int c, float mul = 1.f) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int d = c * 16 + 4 * e + u;
            v[u] = d < D ? x[d] * mul : 0.f;
        }
        w[e] = sm100::pack_e4m3x4(v[0], v[1], v[2], v[3]);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}


// Backward of qk_prologue (with scale 1) for one row: g holds dL/d(output) on entry
// and dL/dx on exit; x is the raw input row.  RoPE^T rotates by -angle; the
// RMS-norm backward is dx = gain*dz*r - x * sum(gain*dz*x) * r^3 / D, r = 1/rms.
// With apply = false (no prologue) the gradient passes through unchanged.
template <int D>
__device__ __forceinline__ void qk_prologue_bwd(const float (&x)[D], float (&g)[D], uint32_t pos, const float *gain,
                                                const float *rope, int32_t off0, int32_t off1, int32_t off2,
                                                float eps, bool apply = true) {
    constexpr int P = Geo<D>::PAIRS;
    if (!apply) return;
    const int32_t p[3] = {(int32_t)(pos >> 16), (int32_t)((pos >> 8) & 255u), (int32_t)(pos & 255u)};
    const int32_t off[3] = {off0, off1, off2};
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        const float2 *tab = reinterpret_cast<const float2 *>(rope) + (size_t)(off[a] + p[a]) * P;
#pragma unroll
        for (int k = 0; k < P; ++k) {
            const float2 cs = __ldg(tab + k);
            const int c0 = 2 * P * a + 2 * k;
            const float y0 = g[c0], y1 = g[c0 + 1];
            g[c0] = y0 * cs.x + y1 * cs.y;
            g[c0 + 1] = -y0 * cs.y + y1 * cs.x;
        }
    }
    float ss = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) ss = fmaf(x[d], x[d], ss);
    const float r = rsqrtf(ss * (1.0f / D) + eps);
    float dot = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) {
        g[d] *= (gain ? __ldg(gain + d) : 1.0f);
        dot = fmaf(g[d], x[d], dot);
    }
    const float c = dot * r * r * r * (1.0f / D);
#pragma unroll
    for (int d = 0; d < D; ++d) g[d] = g[d] * r - x[d] * c;
}

// Gradients of the prologue's parameters for one row, accumulated into dg / db.  With
// r = 1/rms(x), z = x r, xh = gain z and y = R(angle) xh (dy = dL/dy on entry):
//   dg_d += (R^T dy)_d z_d;
//   for pair k of axis a: dL/dangle = dy1 y0 - dy0 y1, and angle = pos_a base_a^(-k/P), so
//   db_a += dL/dangle * pos_a * coef[8 a + k] with coef[8 a + k] = d(base_a^(-k/P))/d(base_a).
// The packed t is relative to the plan's first frame tbase; pos_t = t + tbase.
template <int D>
__device__ __forceinline__ void qk_param_grads(const float (&x)[D], const float (&dy)[D], uint32_t pos,
                                               const float *gain, const float *rope, int32_t off0, int32_t off1,
                                               int32_t off2, float eps, const float *coef, int32_t tbase,
                                               float (&dg)[D], float (&db)[3]) {
    constexpr int P = Geo<D>::PAIRS;
    float ss = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) ss = fmaf(x[d], x[d], ss);
    const float r = rsqrtf(ss * (1.0f / D) + eps);
#pragma unroll
    for (int d = 6 * P; d < D; ++d) dg[d] = fmaf(dy[d], x[d] * r, dg[d]);  // channels RoPE leaves alone
    const int32_t p[3] = {(int32_t)(pos >> 16), (int32_t)((pos >> 8) & 255u), (int32_t)(pos & 255u)};
    const int32_t off[3] = {off0, off1, off2};
    const float pabs[3] = {(float)(p[0] + tbase), (float)p[1], (float)p[2]};
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        const float2 *tab = reinterpret_cast<const float2 *>(rope) + (size_t)(off[a] + p[a]) * P;
#pragma unroll
        for (int k = 0; k < P; ++k) {
            const float2 cs = __ldg(tab + k);
            const int c0 = 2 * P * a + 2 * k;
            const float z0 = x[c0] * r, z1 = x[c0 + 1] * r;
            const float h0 = z0 * (gain ? __ldg(gain + c0) : 1.0f), h1 = z1 * (gain ? __ldg(gain + c0 + 1) : 1.0f);
            const float y0 = h0 * cs.x - h1 * cs.y, y1 = h0 * cs.y + h1 * cs.x;
            const float dang = dy[c0 + 1] * y0 - dy[c0] * y1;
            db[a] = fmaf(dang * pabs[a], coef[8 * a + k], db[a]);
            dg[c0] = fmaf(dy[c0] * cs.x + dy[c0 + 1] * cs.y, z0, dg[c0]);
            dg[c0 + 1] = fmaf(-dy[c0] * cs.y + dy[c0 + 1] * cs.x, z1, dg[c0 + 1]);
        }
    }
}

// Pack values [8c, 8c+8) of x (zero past D) into one 16-byte chunk of bf16.
template <int D>
__device__ __forceinline__ uint4 pack_chunk_bf16(const float (&x)[D], int c) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int d0 = c * 8 + 2 * e;
        const float lo = d0 < D ? x[d0] : 0.f;
        const float hi = d0 + 1 < D ? x[d0 + 1] : 0.f;
        w[e] = sm100::pack_bf16x2(lo, hi);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace bca
