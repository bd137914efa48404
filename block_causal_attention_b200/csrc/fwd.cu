// Forward pass of block-causal GQA attention on sm_100a.
//
//   kv_image_kernel : QK-Norm + 3D RoPE of the new keys (cache keys are copied as
//                     given) and re-layout of K-hat and V into MMA-ready tile images
//                     in the workspace, so that the attention kernel moves each K or
//                     V tile with one bulk copy.
//   fwd_kernel      : one CTA per work item (q-tile x two query heads of one KV
//                     group).  Warp 0 streams K/V tiles with bulk copies (TMA engine)
//                     into a 4-stage ring; warp 1 issues tcgen05 MMAs (S = Q K^T and
//                     O += P V, fp32 accumulators in tensor memory); warps 4-7 and
//                     8-11 each own one query head: they normalise, rotate and scale
//                     their Q tile into shared memory, run the online softmax on S
//                     rows read from tensor memory, write P (bf16) for the second MMA,
//                     and finish with O / l and the LSE.
//   e4m3 variant    : the same kernel instantiated with F8 = true (plans created with
//                     BCA_FWD_FP8_E4M3): v_amax_kernel finds max|V| per KV head,
//                     kv_image8_kernel writes e4m3 K-hat and V / 2^e images, and the
//                     MMAs run as kind::f8f6f4 with e4m3 Q-hat and P.
//
// The operation: attention restricted to the union of AttnSlices, with QK-Norm and
// 3D RoPE applied to Q and K and 128/8 grouped query heads (MAGI-1 research notes
// (zhao9797.github.io), "Autoregressive denoising DiT" and "Infra > MagiAttention >
// Flex-Flash-Attention").  Those pages build the kernel on FlashAttention-3 for
// Hopper; here the same online-softmax algorithm is mapped onto tcgen05 + TMEM.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "kernels.hpp"
#include "prologue.cuh"
#include "sm100.cuh"

namespace bca {

using namespace sm100;

namespace {

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s per wait; a healthy wait is microseconds

struct KVArgs {
    const __nv_bfloat16 *k, *v, *kc, *vc;
    const float *k_gain;
    const uint32_t *pos;
    const float *rope;
    int32_t axis_off0, axis_off1, axis_off2;
    int64_t nc, nk, nkt;
    int hkv;
    float eps;
    int prologue;  // 0: keys given post-prologue (BCA_NO_PROLOGUE)
    int kc_f16;    // cache keys are fp16 (BCA_CACHE_K_FP16)
    __half *kimg;
    __nv_bfloat16 *vimg;
    // e4m3 images (plans with BCA_FWD_FP8_E4M3)
    uint8_t *kimg8, *vimg8;
    float *vamax;  // [hkv] max |V| over the new and the cache rows
};

struct FwdArgs {
    const __nv_bfloat16 *q;
    const float *q_gain;
    const uint32_t *pos;
    const float *rope;
    int32_t axis_off0, axis_off1, axis_off2;
    const __half *kimg;
    const __nv_bfloat16 *vimg;
    const uint8_t *kimg8, *vimg8;  // e4m3 images (FP8 kernel only)
    const float *vamax;            // [hkv] max |V|, for the power-of-two V scale (FP8 only)
    const Item *items;
    const int32_t *run_off;
    const Run *runs;
    const uint32_t *masks;
    int64_t nq, nkt;
    int hq, hkv;
    int prologue;       // 0: queries given post-prologue (BCA_NO_PROLOGUE)
    float eps, qscale;  // qscale = log2(e) / sqrt(D)
    int o_fp32;
    void *o;
    float *lse;
    int *status;
    uint64_t timeout_ns;  // per wait
    int skip_loads;       // failure-detection test: issue no K/V loads
};

// ------------------------------------------------------------------ K-hat / V images

// Tile image layout (128 x DPAD 16-bit values per (KV head, k-tile)), made of 8x8
// core matrices of 128 contiguous bytes.  K-hat is stored as fp16: it is RMS-
// normalised (|x| <= sqrt(D) * max|gain|), so fp16's range suffices and its 11-bit
// significand keeps the scores 8x more precise than bf16 would; V stays bf16.
//   K-hat: core (key group kg, d group kc) at ((kc * 16 + kg) * 64) elements,
//          element (key, d) at + (key % 8) * 8 + d % 8.          [K-major B of S=QK^T]
//   V    : core (d group dg, key group kc) at ((kc * DPAD/8 + dg) * 64) elements,
//          element (d, key) at + (d % 8) * 8 + key % 8.          [K-major B of O=PV]
template <int D>
__global__ void __launch_bounds__(128) kv_image_kernel(KVArgs a) {
    constexpr int DPAD = Geo<D>::DPAD;
    __shared__ __nv_bfloat16 sv[128][DPAD + 8];
    const int t = threadIdx.x;
    const int64_t kt = blockIdx.x;
    const int g = blockIdx.y;
    const int64_t key = kt * 128 + t;
    const size_t tile = ((size_t)g * a.nkt + kt) * (128 * DPAD);

    float x[D];
    if (key < a.nc) {
        load_row_16<D>(a.kc + ((size_t)key * a.hkv + g) * D, a.kc_f16 != 0, x);
    } else if (key < a.nk) {
        const int64_t n = key - a.nc;
        load_row_bf16<D>(a.k + ((size_t)n * a.hkv + g) * D, x);
        qk_prologue<D>(x, __ldg(a.pos + n), a.k_gain, a.rope, a.axis_off0, a.axis_off1, a.axis_off2, a.eps,
                       1.0f, a.prologue != 0);
    } else {
#pragma unroll
        for (int d = 0; d < D; ++d) x[d] = 0.f;
    }
    uint4 *kout = reinterpret_cast<uint4 *>(a.kimg + tile);
#pragma unroll
    for (int c = 0; c < DPAD / 8; ++c) kout[(c * 16 + t / 8) * 8 + (t % 8)] = pack_chunk_f16<D>(x, c);

    // V: stage the row, then write the transposed core-matrix image
    if (key < a.nc) {
        load_row_bf16<D>(a.vc + ((size_t)key * a.hkv + g) * D, x);
    } else if (key < a.nk) {
        load_row_bf16<D>(a.v + ((size_t)(key - a.nc) * a.hkv + g) * D, x);
    } else {
#pragma unroll
        for (int d = 0; d < D; ++d) x[d] = 0.f;
    }
#pragma unroll
    for (int d = 0; d < DPAD; ++d) sv[t][d] = __float2bfloat16_rn(d < D ? x[d] : 0.f);
    __syncthreads();
    uint4 *vout = reinterpret_cast<uint4 *>(a.vimg + tile);
#pragma unroll
    for (int i = 0; i < DPAD / 8; ++i) {
        const int c = t + 128 * i;  // chunk index = (kc * DPAD/8 + dg) * 8 + dd
        const int dd = c % 8, dg = (c / 8) % (DPAD / 8), kc = c / DPAD;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 b;
            b.x = sv[kc * 8 + 2 * e][dg * 8 + dd];
            b.y = sv[kc * 8 + 2 * e + 1][dg * 8 + dd];
            w[e] = *reinterpret_cast<uint32_t *>(&b);
        }
        vout[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// ------------------------------------------------------------------ e4m3 images
//
// The FP8 forward (plans created with BCA_FWD_FP8_E4M3) feeds the tensor cores e4m3
// operands: K-hat as it is (RMS-normalised, so |x| <= sqrt(D) * max|gain| stays far
// inside e4m3's +-448), and V divided by a power of two 2^e per KV head, chosen from the
// largest |V| so that V / 2^e <= 448; the epilogue multiplies O by 2^e again (exact).

// Exponent e of the power-of-two V scale: amax / 448 in [2^(e-1), 2^e), so V / 2^e < 448
// (0 for amax == 0).  Exact, from amax's own binary exponent: amax = m * 2^f with m in
// [0.5, 1) and 448 = 0.875 * 2^9, so e = f - 8 when m >= 0.875, else f - 9.
__device__ __forceinline__ int v8_scale_exp(float amax) {
    if (!(amax > 0.f)) return 0;
    int f;
    const float m = frexpf(amax, &f);
    return m >= 0.875f ? f - 8 : f - 9;
}

// amax[g] = max |V| over the new rows and the cache rows of KV head g (amax zeroed before).
template <int D>
__global__ void __launch_bounds__(256) v_amax_kernel(KVArgs a) {
    const int64_t row = (int64_t)blockIdx.x * 256 + threadIdx.x;  // key row in [0, nk)
    const int g = blockIdx.y;
    float m = 0.f;
    if (row < a.nk) {
        float x[D];
        if (row < a.nc) load_row_bf16<D>(a.vc + ((size_t)row * a.hkv + g) * D, x);
        else load_row_bf16<D>(a.v + ((size_t)(row - a.nc) * a.hkv + g) * D, x);
#pragma unroll
        for (int d = 0; d < D; ++d) m = fmaxf(m, fabsf(x[d]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    // non-negative floats order like their bit patterns
    if ((threadIdx.x & 31) == 0 && m > 0.f) atomicMax(reinterpret_cast<int *>(a.vamax + g), __float_as_int(m));
}

// e4m3 tile images, one (k-tile, KV head) per block:
//   K-hat: 128 keys x DP8, K-major; core (d chunk c of 16, key group kg of 8) at
//          (c * 16 + kg) * 128 bytes, element (key, d) at + (key % 8) * 16 + d % 16.
//   V^T  : DPAD x 128 keys, K-major; core (key chunk kc of 16, d group dg of 8) at
//          (kc * DPAD/8 + dg) * 128 bytes, element (d, key) at + (d % 8) * 16 + key % 16.
template <int D>
__global__ void __launch_bounds__(128) kv_image8_kernel(KVArgs a) {
    constexpr int DPAD = Geo<D>::DPAD;
    constexpr int DP8 = Geo<D>::DP8;
    __shared__ float sv[128][DPAD + 1];
    const int t = threadIdx.x;
    const int64_t kt = blockIdx.x;
    const int g = blockIdx.y;
    const int64_t key = kt * 128 + t;
    const size_t tile = (size_t)g * a.nkt + kt;

    float x[D];
    if (key < a.nc) {
        load_row_16<D>(a.kc + ((size_t)key * a.hkv + g) * D, a.kc_f16 != 0, x);
    } else if (key < a.nk) {
        const int64_t n = key - a.nc;
        load_row_bf16<D>(a.k + ((size_t)n * a.hkv + g) * D, x);
        qk_prologue<D>(x, __ldg(a.pos + n), a.k_gain, a.rope, a.axis_off0, a.axis_off1, a.axis_off2, a.eps,
                       1.0f, a.prologue != 0);
    } else {
#pragma unroll
        for (int d = 0; d < D; ++d) x[d] = 0.f;
    }
    uint4 *kout = reinterpret_cast<uint4 *>(a.kimg8 + tile * Geo<D>::K8_TILE_BYTES);
#pragma unroll
    for (int c = 0; c < DP8 / 16; ++c) kout[(c * 16 + t / 8) * 8 + (t % 8)] = pack_chunk_e4m3<D>(x, c);

    const float mul = ldexpf(1.0f, -v8_scale_exp(a.vamax[g]));
    if (key < a.nc) {
        load_row_bf16<D>(a.vc + ((size_t)key * a.hkv + g) * D, x);
    } else if (key < a.nk) {
        load_row_bf16<D>(a.v + ((size_t)(key - a.nc) * a.hkv + g) * D, x);
    } else {
#pragma unroll
        for (int d = 0; d < D; ++d) x[d] = 0.f;
    }
#pragma unroll
    for (int d = 0; d < DPAD; ++d) sv[t][d] = d < D ? x[d] * mul : 0.f;
    __syncthreads();
    uint4 *vout = reinterpret_cast<uint4 *>(a.vimg8 + tile * Geo<D>::V8_TILE_BYTES);
#pragma unroll
    for (int i = 0; i < DPAD / 16; ++i) {
        const int c = t + 128 * i;  // 16-byte row index = (kc * DPAD/8 + dg) * 8 + dd
        const int dd = c % 8, dg = (c / 8) % (DPAD / 8), kc = c / DPAD;
        const int d = dg * 8 + dd;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            w[e] = pack_e4m3x4(sv[kc * 16 + 4 * e][d], sv[kc * 16 + 4 * e + 1][d], sv[kc * 16 + 4 * e + 2][d],
                               sv[kc * 16 + 4 * e + 3][d]);
        vout[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// ------------------------------------------------------------------ attention kernel

// F8: e4m3 Q-hat, K-hat, P and V^T (k-granule 32), else fp16 Q-hat / K-hat and bf16 P / V.
template <int D, bool F8>
struct FwdSmem {
    static constexpr int DPAD = Geo<D>::DPAD;
    static constexpr int DP8 = Geo<D>::DP8;
    static constexpr int STAGES = 4;
    static constexpr int Q_BYTES = F8 ? 128 * DP8 : 128 * DPAD * 2;
    static constexpr int P_BYTES = F8 ? 128 * 128 : 128 * 128 * 2;
    static constexpr int KTILE = F8 ? Geo<D>::K8_TILE_BYTES : Geo<D>::TILE_BYTES;
    static constexpr int VTILE = F8 ? Geo<D>::V8_TILE_BYTES : Geo<D>::TILE_BYTES;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_P = OFF_Q + 2 * Q_BYTES;
    static constexpr int OFF_K = OFF_P + 2 * P_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES * KTILE;
    static constexpr int OFF_BAR = OFF_V + STAGES * VTILE;
    // barriers
    static constexpr int B_KV_FULL = 0;
    static constexpr int B_KV_EMPTY = STAGES;
    static constexpr int B_S_FULL = 2 * STAGES;      // [2]
    static constexpr int B_S_FREE = B_S_FULL + 2;    // [2]
    static constexpr int B_P_FULL = B_S_FREE + 2;    // [2]
    static constexpr int B_O_DONE = B_P_FULL + 2;    // [2]
    static constexpr int B_Q_READY = B_O_DONE + 2;   // [2]
    static constexpr int B_MMA_DONE = B_Q_READY + 2;
    static constexpr int NBAR = B_MMA_DONE + 1;
    static constexpr int OFF_TMEM_PTR = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEM_PTR + 4;
    static constexpr int BYTES = OFF_ABORT + 12;
    // tensor memory columns
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S = 0;    // + 128 * slot
    static constexpr uint32_t COL_O = 256;  // + 64 * slot
};

struct RunCursor {
    const Run *r;
    const Run *end;
    int32_t kt;
    __device__ __forceinline__ RunCursor(const Run *b, const Run *e) : r(b), end(e), kt(b < e ? b->kt_begin : 0) {}
    __device__ __forceinline__ bool valid() const { return r < end; }
    __device__ __forceinline__ void next() {
        if (++kt >= r->kt_end) {
            ++r;
            if (r < end) kt = r->kt_begin;
        }
    }
};

__device__ __forceinline__ void record_timeout(int *status, volatile int *abort_flag) {
    atomicOr(status, kStatusTimeout);
    *abort_flag = 1;
}

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, int *status, volatile int *abort_flag,
                                              uint64_t timeout_ns = kWaitTimeoutNs) {
    // A completed phase needs no look at the abort flag: the flag is a volatile shared
    // load on every waiter's path (the MMA issuer waits several times per tile), and only
    // a wait that would block has to know whether the CTA is giving up.
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, timeout_ns)) return true;
    record_timeout(status, abort_flag);
    return false;
}

// Same, with the outcome made uniform across the warp (for warps that go on to
// issue warp-collective tcgen05 loads/stores).
__device__ __forceinline__ bool warp_wait_or_abort(uint32_t bar, uint32_t parity, int *status,
                                                   volatile int *abort_flag, uint64_t timeout_ns = kWaitTimeoutNs) {
    const bool ok = wait_or_abort(bar, parity, status, abort_flag, timeout_ns);
    return __all_sync(0xffffffffu, ok);
}

// NH: query heads per work item, 2 (their softmax warps 4-7 and 8-11 share each K/V tile)
// or 1 for an odd group size (warps 8-11 idle).  A compile-time count keeps the MMA
// issuer's per-tile loop over heads unrolled.
template <int D, bool F8, int NH>
__global__ void __launch_bounds__(384, 1) fwd_kernel(FwdArgs a) {
    using L = FwdSmem<D, F8>;
    constexpr int DPAD = L::DPAD;
    constexpr int STAGES = L::STAGES;
    constexpr uint32_t IDESC_S = idesc_f32acc(128, 128, F8 ? kFmtE4M3 : kFmtF16);
    constexpr uint32_t IDESC_PV = idesc_f32acc(128, DPAD, F8 ? kFmtE4M3 : kFmtBF16);

    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::OFF_BAR;
    auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::OFF_ABORT);
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + L::OFF_TMEM_PTR);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const Item item = a.items[blockIdx.x];
    const int64_t qt = item.q_tile;
    const int G = a.hq / a.hkv;
    const int h0 = item.head0;
    const int g = h0 / G;
    const Run *rb = a.runs + a.run_off[qt];
    const Run *re = a.runs + a.run_off[qt + 1];
    int n = 0;
    for (const Run *r = rb; r < re; ++r) n += r->kt_end - r->kt_begin;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(bar(L::B_KV_FULL + i), 1);
            mbar_init(bar(L::B_KV_EMPTY + i), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(L::B_S_FULL + s), 1);
            mbar_init(bar(L::B_S_FREE + s), 128);
            mbar_init(bar(L::B_P_FULL + s), 128);
            mbar_init(bar(L::B_O_DONE + s), 1);
            mbar_init(bar(L::B_Q_READY + s), 128);
        }
        mbar_init(bar(L::B_MMA_DONE), 1);
        mbar_fence_init();
        fence_proxy_async_smem();
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_ptr), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_ptr;

    // Registers: 384 threads x 168 at launch.  The producer / MMA warpgroup (warps 0-3) needs
    // few and gives them up (96), the softmax warpgroups take 184 (128 x 96 + 256 x 184 =
    // 59,392 <= 64,512), which removes most of their spills.  Each warpgroup executes its
    // instruction together (warps 0-3 here, the softmax warpgroup at the top of its branch).
    if (warp < 4) regs_dec<96>();
    if (warp == 0) {
        // ------------------------------------------------ producer: K/V tiles
        if (lane == 0 && n > 0 && !a.skip_loads) {
            int issued = 0;
            RunCursor cur(rb, re);
            for (int j = 0; j < n; ++j, cur.next()) {
                const int stage = j % STAGES;
                if (j >= STAGES &&
                    !wait_or_abort(bar(L::B_KV_EMPTY + stage), ((j / STAGES) - 1) & 1, a.status, abort_flag, a.timeout_ns))
                    break;
                const size_t tile = (size_t)g * a.nkt + cur.kt;
                const void *ksrc = F8 ? (const void *)(a.kimg8 + tile * L::KTILE)
                                      : (const void *)(a.kimg + tile * (128 * DPAD));
                const void *vsrc = F8 ? (const void *)(a.vimg8 + tile * L::VTILE)
                                      : (const void *)(a.vimg + tile * (128 * DPAD));
                mbar_arrive_expect_tx(bar(L::B_KV_FULL + stage), L::KTILE + L::VTILE);
                bulk_g2s(sbase + L::OFF_K + stage * L::KTILE, ksrc, L::KTILE, bar(L::B_KV_FULL + stage));
                bulk_g2s(sbase + L::OFF_V + stage * L::VTILE, vsrc, L::VTILE, bar(L::B_KV_FULL + stage));
                ++issued;
            }
            // every issued copy must have landed before the CTA may exit
            for (int j = (issued > STAGES ? issued - STAGES : 0); j < issued; ++j)
                if (!mbar_wait(bar(L::B_KV_FULL + j % STAGES), (j / STAGES) & 1, a.timeout_ns))
                    record_timeout(a.status, abort_flag);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            bool ok = wait_or_abort(bar(L::B_Q_READY + 0), 0, a.status, abort_flag, a.timeout_ns) &&
                      (NH < 2 || wait_or_abort(bar(L::B_Q_READY + 1), 0, a.status, abort_flag, a.timeout_ns)) &&
                      wait_or_abort(bar(L::B_KV_FULL + 0), 0, a.status, abort_flag, a.timeout_ns);
            tc_fence_after();
            // Both operands K-major with no swizzle: a core matrix is 8 rows x 16 bytes (8
            // fp16/bf16 or 16 e4m3 elements), core matrices adjacent in K lie 2048 bytes
            // apart (V: (DPAD/8) * 128), adjacent in M/N 128 bytes apart.  One MMA consumes
            // two core matrices of K (16 elements at 16 bits, 32 at 8 bits).
            auto issue_s = [&](int slot, int stage) {
                const uint32_t qa = sbase + L::OFF_Q + slot * L::Q_BYTES;
                const uint32_t kb = sbase + L::OFF_K + stage * L::KTILE;
                constexpr int KSTEPS = F8 ? L::DP8 / 32 : DPAD / 16;
#pragma unroll
                for (int kk = 0; kk < KSTEPS; ++kk) {
                    const uint64_t ad = smem_desc(qa + kk * 4096, 2048, 128);
                    const uint64_t bd = smem_desc(kb + kk * 4096, 2048, 128);
                    if constexpr (F8) mma_f8(tbase + L::COL_S + 128 * slot, ad, bd, IDESC_S, kk > 0);
                    else mma_f16(tbase + L::COL_S + 128 * slot, ad, bd, IDESC_S, kk > 0);
                }
            };
            auto issue_pv = [&](int slot, int stage, bool acc) {
                const uint32_t pa = sbase + L::OFF_P + slot * L::P_BYTES;
                const uint32_t vb = sbase + L::OFF_V + stage * L::VTILE;
                constexpr uint32_t VLBO = (DPAD / 8) * 128;
#pragma unroll
                for (int kk = 0; kk < (F8 ? 4 : 8); ++kk) {
                    const uint64_t ad = smem_desc(pa + kk * 4096, 2048, 128);
                    const uint64_t bd = smem_desc(vb + kk * 2 * VLBO, VLBO, 128);
                    if constexpr (F8) mma_f8(tbase + L::COL_O + 64 * slot, ad, bd, IDESC_PV, (acc || kk > 0) ? 1u : 0u);
                    else mma_f16(tbase + L::COL_O + 64 * slot, ad, bd, IDESC_PV, (acc || kk > 0) ? 1u : 0u);
                }
            };
            if (ok) {
                for (int s = 0; s < NH; ++s) {
                    issue_s(s, 0);
                    mma_commit(bar(L::B_S_FULL + s));
                }
                for (int j = 0; j < n && ok; ++j) {
                    const int stage = j % STAGES;
                    const bool more = j + 1 < n;
                    const int nstage = (j + 1) % STAGES;
                    if (more) {
                        ok = wait_or_abort(bar(L::B_KV_FULL + nstage), ((j + 1) / STAGES) & 1, a.status, abort_flag, a.timeout_ns);
                        tc_fence_after();
                    }
                    for (int s = 0; s < NH && ok; ++s) {
                        if (more) {
                            ok = wait_or_abort(bar(L::B_S_FREE + s), j & 1, a.status, abort_flag, a.timeout_ns);
                            if (!ok) break;
                            tc_fence_after();
                            issue_s(s, nstage);
                            mma_commit(bar(L::B_S_FULL + s));
                        }
                        ok = wait_or_abort(bar(L::B_P_FULL + s), j & 1, a.status, abort_flag, a.timeout_ns);
                        if (!ok) break;
                        tc_fence_after();
                        issue_pv(s, stage, j > 0);
                        mma_commit(bar(L::B_O_DONE + s));
                    }
                    mma_commit(bar(L::B_KV_EMPTY + stage));
                }
            }
            // all issued MMAs must be complete before TMEM is released
            mma_commit(bar(L::B_MMA_DONE));
            if (!mbar_wait(bar(L::B_MMA_DONE), 0, a.timeout_ns)) record_timeout(a.status, abort_flag);
        }
        __syncwarp();
    } else if (warp >= 4 && (warp - 4) / 4 < NH) {
        regs_inc<184>();
        // ------------------------------------------------ softmax / prologue / epilogue
        const int slot = (warp - 4) / 4;
        const int quarter = warp % 4;  // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;
        const int h = h0 + slot;
        const int64_t qrow = qt * 128 + row;
        const bool live = qrow < a.nq;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;

        {   // Q prologue into shared memory (core-matrix layout, K-major A operand): fp16 with
            // the softmax scale folded in, or e4m3 unscaled (the scale is applied to S in fp32,
            // keeping the normalised values in e4m3's normal range)
            float x[D];
            if (live) {
                load_row_bf16<D>(a.q + ((size_t)qrow * a.hq + h) * D, x);
                qk_prologue<D>(x, __ldg(a.pos + qrow), a.q_gain, a.rope, a.axis_off0, a.axis_off1, a.axis_off2,
                               a.eps, F8 ? 1.0f : a.qscale, a.prologue != 0);
            } else {
#pragma unroll
                for (int d = 0; d < D; ++d) x[d] = 0.f;
            }
            uint4 *qs = reinterpret_cast<uint4 *>(smem + L::OFF_Q + slot * L::Q_BYTES);
            if constexpr (F8) {
#pragma unroll
                for (int c = 0; c < L::DP8 / 16; ++c) qs[(c * 16 + row / 8) * 8 + row % 8] = pack_chunk_e4m3<D>(x, c);
            } else {
#pragma unroll
                for (int c = 0; c < DPAD / 8; ++c) qs[(c * 16 + row / 8) * 8 + row % 8] = pack_chunk_f16<D>(x, c);
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(L::B_Q_READY + slot));
        }

        const uint32_t tS = tbase + lane_off + L::COL_S + 128 * slot;
        const uint32_t tO = tbase + lane_off + L::COL_O + 64 * slot;
        uint4 *ps = reinterpret_cast<uint4 *>(smem + L::OFF_P + slot * L::P_BYTES);
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        RunCursor cur(rb, re);
        for (int j = 0; j < n; ++j, cur.next()) {
            ok = warp_wait_or_abort(bar(L::B_S_FULL + slot), j & 1, a.status, abort_flag, a.timeout_ns);
            if (!ok) break;
            tc_fence_after();
            float s[128];
            {
                uint32_t r[128];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 128; ++e) s[e] = __uint_as_float(r[e]);
            }
            tc_fence_before();
            mbar_arrive(bar(L::B_S_FREE + slot));

            if (cur.r->mask_idx >= 0) {
                const uint4 mw = reinterpret_cast<const uint4 *>(a.masks)[(size_t)cur.r->mask_idx * 128 + row];
                const uint32_t w4[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (!((w4[c / 32] >> (c % 32)) & 1u)) s[c] = -INFINITY;
            }
            float mx = s[0];
#pragma unroll
            for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
            if constexpr (F8) mx *= a.qscale;  // S in log2 units (the scale is positive)
            float alpha = 1.f;
            bool rescale = false;
            if (mx > m_ref + 8.0f) {  // lazy rescaling: move the reference only when it grows by > 2^8
                alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - mx);
                rescale = j > 0;
                m_ref = mx;
            }
            const float msub = (m_ref == -INFINITY) ? 0.f : m_ref;
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                s[c] = F8 ? ex2(fmaf(s[c], a.qscale, -msub)) : ex2(s[c] - msub);
                sum += s[c];
            }
            l = l * alpha + sum;

            if (j > 0) {
                ok = warp_wait_or_abort(bar(L::B_O_DONE + slot), (j - 1) & 1, a.status, abort_flag, a.timeout_ns);
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
                    const float f = rescale ? alpha : 1.f;
#pragma unroll
                    for (int c = 0; c < DPAD / 16; ++c) {
                        uint32_t o16[16];
                        tmem_ld16(tO + 16 * c, o16);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) o16[e] = __float_as_uint(__uint_as_float(o16[e]) * f);
                        tmem_st16(tO + 16 * c, o16);
                    }
                    tmem_wait_st();
                }
            }
            // P (bf16, or e4m3: P <= 2^8 under the lazy rescale, inside e4m3's range) in the
            // core-matrix layout of the K-major A operand
            if constexpr (F8) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float *v = s + 16 * c;
                    ps[(c * 16 + row / 8) * 8 + row % 8] =
                        make_uint4(pack_e4m3x4(v[0], v[1], v[2], v[3]), pack_e4m3x4(v[4], v[5], v[6], v[7]),
                                   pack_e4m3x4(v[8], v[9], v[10], v[11]), pack_e4m3x4(v[12], v[13], v[14], v[15]));
                }
            } else {
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const uint4 u =
                        make_uint4(pack_bf16x2(s[8 * c + 0], s[8 * c + 1]), pack_bf16x2(s[8 * c + 2], s[8 * c + 3]),
                                   pack_bf16x2(s[8 * c + 4], s[8 * c + 5]), pack_bf16x2(s[8 * c + 6], s[8 * c + 7]));
                    ps[(c * 16 + row / 8) * 8 + row % 8] = u;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar(L::B_P_FULL + slot));
        }

        // epilogue: O / l and LSE
        float o[DPAD];
#pragma unroll
        for (int d = 0; d < DPAD; ++d) o[d] = 0.f;
        if (n > 0 && ok) {
            ok = warp_wait_or_abort(bar(L::B_O_DONE + slot), (n - 1) & 1, a.status, abort_flag, a.timeout_ns);
            tc_fence_after();
            if (ok) {
#pragma unroll
                for (int c = 0; c < DPAD / 16; ++c) {
                    uint32_t o16[16];
                    tmem_ld16(tO + 16 * c, o16);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[16 * c + e] = __uint_as_float(o16[e]);
                }
            }
        }
        if (live) {
            const bool any = l > 0.f;
            float inv = any ? 1.0f / l : 0.f;
            if constexpr (F8) inv = ldexpf(inv, v8_scale_exp(a.vamax[g]));  // undo V / 2^e
            if (a.o_fp32) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.o) + ((size_t)qrow * a.hq + h) * D);
#pragma unroll
                for (int c = 0; c < D / 4; ++c)
                    dst[c] = make_float4(o[4 * c] * inv, o[4 * c + 1] * inv, o[4 * c + 2] * inv, o[4 * c + 3] * inv);
            } else {
                uint4 *dst =
                    reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.o) + ((size_t)qrow * a.hq + h) * D);
#pragma unroll
                for (int c = 0; c < D / 8; ++c)
                    dst[c] = make_uint4(pack_bf16x2(o[8 * c] * inv, o[8 * c + 1] * inv),
                                        pack_bf16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv),
                                        pack_bf16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv),
                                        pack_bf16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv));
            }
            a.lse[(size_t)h * a.nq + qrow] = any ? (m_ref + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tbase, L::TMEM_COLS);
    }
}

template <int D>
int launch_fwd_d(Plan &P, const FwdIO &io, cudaStream_t stream) {
    const bool f8 = (P.flags & BCA_FWD_FP8_E4M3) != 0;
    const size_t img = kv_image_bytes(P);
    auto *kimg = static_cast<__half *>(io.workspace);
    auto *vimg = reinterpret_cast<__nv_bfloat16 *>(static_cast<uint8_t *>(io.workspace) + img);
    // e4m3 images share the workspace: K-hat at 0, V^T after it, the V amax after both
    uint8_t *ws8 = static_cast<uint8_t *>(io.workspace);
    const size_t k8 = ((size_t)P.hkv * (size_t)P.nkt * Geo<D>::K8_TILE_BYTES + 255) / 256 * 256;
    const size_t v8 = ((size_t)P.hkv * (size_t)P.nkt * Geo<D>::V8_TILE_BYTES + 255) / 256 * 256;
    float *vamax = reinterpret_cast<float *>(ws8 + k8 + v8);

    KVArgs ka;
    ka.k = static_cast<const __nv_bfloat16 *>(io.k);
    ka.v = static_cast<const __nv_bfloat16 *>(io.v);
    ka.kc = static_cast<const __nv_bfloat16 *>(io.k_cache);
    ka.vc = static_cast<const __nv_bfloat16 *>(io.v_cache);
    ka.k_gain = io.k_gain;
    ka.pos = P.d_pos;
    ka.rope = P.d_rope;
    ka.axis_off0 = P.rope_axis_off[0];
    ka.axis_off1 = P.rope_axis_off[1];
    ka.axis_off2 = P.rope_axis_off[2];
    ka.nc = P.nc;
    ka.nk = P.nk;
    ka.nkt = P.nkt;
    ka.hkv = P.hkv;
    ka.eps = P.eps;
    ka.prologue = (P.flags & BCA_NO_PROLOGUE) ? 0 : 1;
    ka.kc_f16 = (P.flags & BCA_CACHE_K_FP16) ? 1 : 0;
    ka.kimg = kimg;
    ka.vimg = vimg;
    ka.kimg8 = ws8;
    ka.vimg8 = ws8 + k8;
    ka.vamax = vamax;
    if (f8) {
        if (cudaMemsetAsync(vamax, 0, (size_t)P.hkv * sizeof(float), stream) != cudaSuccess) return BCA_ERR_CUDA;
        ProfScope ps(P, BCA_KERNEL_KV_IMAGE, stream);
        if (P.nk > 0)
            v_amax_kernel<D><<<dim3((unsigned)((P.nk + 255) / 256), (unsigned)P.hkv), 256, 0, stream>>>(ka);
        kv_image8_kernel<D><<<dim3((unsigned)P.nkt, (unsigned)P.hkv), 128, 0, stream>>>(ka);
    } else {
        ProfScope ps(P, BCA_KERNEL_KV_IMAGE, stream);
        kv_image_kernel<D><<<dim3((unsigned)P.nkt, (unsigned)P.hkv), 128, 0, stream>>>(ka);
    }
    if (cudaGetLastError() != cudaSuccess) return BCA_ERR_CUDA;

    FwdArgs fa;
    fa.q = static_cast<const __nv_bfloat16 *>(io.q);
    fa.q_gain = io.q_gain;
    fa.pos = P.d_pos;
    fa.rope = P.d_rope;
    fa.axis_off0 = P.rope_axis_off[0];
    fa.axis_off1 = P.rope_axis_off[1];
    fa.axis_off2 = P.rope_axis_off[2];
    fa.kimg = kimg;
    fa.vimg = vimg;
    fa.kimg8 = ws8;
    fa.vimg8 = ws8 + k8;
    fa.vamax = vamax;
    fa.items = P.d_items;
    fa.run_off = P.d_run_off;
    fa.runs = P.d_runs;
    fa.masks = P.d_masks;
    fa.nq = P.nq;
    fa.nkt = P.nkt;
    fa.hq = P.hq;
    fa.hkv = P.hkv;
    fa.prologue = (P.flags & BCA_NO_PROLOGUE) ? 0 : 1;
    fa.eps = P.eps;
    fa.qscale = 1.4426950408889634f / sqrtf((float)D);
    fa.o_fp32 = (P.flags & BCA_O_FP32) ? 1 : 0;
    fa.o = io.o;
    fa.lse = io.lse;
    fa.status = P.d_status;
    fa.timeout_ns = (P.flags & BCA_TEST_FORCE_TIMEOUT) ? 1000000ull : kWaitTimeoutNs;
    fa.skip_loads = (P.flags & BCA_TEST_FORCE_TIMEOUT) ? 1 : 0;
    {
        ProfScope ps(P, BCA_KERNEL_FWD, stream);
        const unsigned grid = (unsigned)P.items.size();
        const bool two = P.heads_per_item == 2;
        if (f8 && two) fwd_kernel<D, true, 2><<<grid, 384, FwdSmem<D, true>::BYTES, stream>>>(fa);
        else if (f8) fwd_kernel<D, true, 1><<<grid, 384, FwdSmem<D, true>::BYTES, stream>>>(fa);
        else if (two) fwd_kernel<D, false, 2><<<grid, 384, FwdSmem<D, false>::BYTES, stream>>>(fa);
        else fwd_kernel<D, false, 1><<<grid, 384, FwdSmem<D, false>::BYTES, stream>>>(fa);
    }
    if (cudaGetLastError() != cudaSuccess) return BCA_ERR_CUDA;
    return BCA_OK;
}

}  // namespace

size_t kv_image_bytes(const Plan &P) {
    const size_t b = (size_t)P.hkv * (size_t)P.nkt * 128 * (size_t)P.dpad * 2;
    return (b + 255) / 256 * 256;
}

// The bf16 K-hat and V images, or (FP8 plans) the smaller e4m3 images plus 256 bytes for
// the per-KV-head V amax.
size_t fwd_workspace_bytes(const Plan &P) { return 2 * kv_image_bytes(P) + ((size_t)P.hkv * 4 + 255) / 256 * 256; }

// The attention kernel needs more than 48 KB of dynamic shared memory; the attribute
// is set once per plan (at creation, on the plan's device) so that no launch path makes
// a non-stream call (launches stay capturable into CUDA graphs).
int prepare_fwd(const Plan &P) {
    auto set = [](const void *f, int bytes) {
        return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
    };
    const bool f8 = (P.flags & BCA_FWD_FP8_E4M3) != 0;
    const bool two = P.heads_per_item == 2;
    auto pick = [&](auto d_c) -> bool {
        constexpr int D = decltype(d_c)::value;
        if (f8 && two) return set((const void *)fwd_kernel<D, true, 2>, FwdSmem<D, true>::BYTES);
        if (f8) return set((const void *)fwd_kernel<D, true, 1>, FwdSmem<D, true>::BYTES);
        if (two) return set((const void *)fwd_kernel<D, false, 2>, FwdSmem<D, false>::BYTES);
        return set((const void *)fwd_kernel<D, false, 1>, FwdSmem<D, false>::BYTES);
    };
    bool ok = true;
    switch (P.d) {
        case 24: ok = pick(std::integral_constant<int, 24>{}); break;
        case 32: ok = pick(std::integral_constant<int, 32>{}); break;
        case 48: ok = pick(std::integral_constant<int, 48>{}); break;
        default: return BCA_ERR_UNSUPPORTED;
    }
    return ok ? BCA_OK : BCA_ERR_CUDA;
}

int launch_fwd(Plan &P, const FwdIO &io, cudaStream_t stream) {
    if (P.nq == 0) return BCA_OK;
    switch (P.d) {
        case 24: return launch_fwd_d<24>(P, io, stream);
        case 32: return launch_fwd_d<32>(P, io, stream);
        case 48: return launch_fwd_d<48>(P, io, stream);
        default: return BCA_ERR_UNSUPPORTED;
    }
}

}  // namespace bca
