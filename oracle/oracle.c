/*
 * fp64 CPU oracle for block-causal attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference legs may load this library.  It shares no code, header,
 * table or helper with the CUDA path (block_causal_attention_b200/csrc): every
 * quantity here is recomputed from its definition, in double precision, over an
 * explicitly materialised mask row.  It is deliberately plain and slow.
 *
 * Sources (the MAGI-1 pages):
 *  - block-causal mask: full attention inside a chunk, causal across chunks
 *    ("Magi-1 开源&刷屏" (163.com), block-causal attention bullets;
 *    MAGI-1 research notes (zhao9797.github.io), "Model architecture >
 *    Overall pipeline");
 *  - the mask as a union of AttnSlices (q-range, k-range, full|causal)
 *    (MAGI-1 research notes, "Infra > MagiAttention > Flex-Flash-Attention";
 *    interview with Zhang Zheng (zhengguannews), the FFA q_range/k_range answer);
 *  - GQA 128/8, QK-Norm, learnable 3D RoPE (MAGI-1 research notes,
 *    "Autoregressive denoising DiT" bullets and Table 2).
 *
 * Readings where the pages are silent (each is also listed with the design notes):
 *  - causal slice with |q| != |k|: bottom-right aligned, j-k0 <= (i-q0)+(|k|-|q|);
 *  - overlapping slices: union (a pair is visible once);
 *  - row with no visible key: O = 0, LSE = -inf, all gradients 0;
 *  - softmax scale 1/sqrt(D);
 *  - QK-Norm = RMS over D per head: xhat = g*x/sqrt(mean(x^2)+eps);
 *  - 3D RoPE: P = D/2 channel pairs, p = floor(P/3) per axis; channels [0,2p) rotate
 *    with t, [2p,4p) with h, [4p,6p) with w, the rest are not rotated; pair k of an
 *    axis is channels (2k, 2k+1) of its segment, angle = pos * base^(-k/p),
 *    (a, b) -> (a cos - b sin, a sin + b cos);
 *  - positions: new token of video v, chunk c, frame f, row y, col x has
 *    (t, h, w) = (t0 + c*F + f, y, x);
 *  - GQA head map: query head h uses KV head floor(h / (Hq/Hkv)).
 *
 * Layouts: token-major.  q: [n][Hq][D]; k, v: [Nk][Hkv][D]; slices: int64 [ns][5]
 * = (q0, q1, k0, k1, type) with type 0 = FULL, 1 = CAUSAL.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_FULL 0
#define ORC_CAUSAL 1

/* Pair (i, j) is visible through slice s iff q0 <= i < q1, k0 <= j < k1 and the slice
 * is FULL or, for CAUSAL, j - k0 <= (i - q0) + (|k| - |q|). */
static int slice_visible(const int64_t *s, int64_t i, int64_t j)
{
    int64_t q0 = s[0], q1 = s[1], k0 = s[2], k1 = s[3];
    if (i < q0 || i >= q1 || j < k0 || j >= k1)
        return 0;
    if (s[4] == ORC_CAUSAL)
        return (j - k0) <= (i - q0) + ((k1 - k0) - (q1 - q0));
    return 1;
}

/* Row i of the dense mask: M[i][j] = OR over slices of slice_visible(s, i, j). */
void orc_mask_row(const int64_t *sl, int ns, int64_t nk, int64_t i, uint8_t *row)
{
    memset(row, 0, (size_t)nk);
    for (int s = 0; s < ns; ++s) {
        const int64_t *S = sl + 5 * s;
        if (i < S[0] || i >= S[1])
            continue;
        for (int64_t j = (S[2] > 0 ? S[2] : 0); j < S[3] && j < nk; ++j)
            if (slice_visible(S, i, j))
                row[j] = 1;
    }
}

/* Column j of the same mask (M[i][j] over all i). */
void orc_mask_col(const int64_t *sl, int ns, int64_t nq, int64_t j, uint8_t *col)
{
    memset(col, 0, (size_t)nq);
    for (int s = 0; s < ns; ++s) {
        const int64_t *S = sl + 5 * s;
        if (j < S[2] || j >= S[3])
            continue;
        for (int64_t i = (S[0] > 0 ? S[0] : 0); i < S[1] && i < nq; ++i)
            if (slice_visible(S, i, j))
                col[i] = 1;
    }
}

void orc_mask_dense(const int64_t *sl, int ns, int64_t nq, int64_t nk, uint8_t *mask)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < nq; ++i)
        orc_mask_row(sl, ns, nk, i, mask + (size_t)i * (size_t)nk);
}

/* (t, h, w) of every new token; videos: int32 [nv][5] = (chunks, frames, height, width, t0). */
void orc_positions(const int32_t *vid, int nv, int32_t *pos)
{
    int64_t n = 0;
    for (int v = 0; v < nv; ++v) {
        int nc = vid[5 * v], F = vid[5 * v + 1], Hh = vid[5 * v + 2], W = vid[5 * v + 3];
        int t0 = vid[5 * v + 4];
        for (int c = 0; c < nc; ++c)
            for (int f = 0; f < F; ++f)
                for (int y = 0; y < Hh; ++y)
                    for (int x = 0; x < W; ++x) {
                        pos[3 * n + 0] = t0 + c * F + f;
                        pos[3 * n + 1] = y;
                        pos[3 * n + 2] = x;
                        ++n;
                    }
    }
}

/* angle of pair k on axis a for position p */
static double rope_angle(int32_t p, double base, int k, int pairs_per_axis)
{
    return (double)p * pow(base, -(double)k / (double)pairs_per_axis);
}

/* QK-Norm then 3D RoPE, per (token, head).  x, out: [n][H][D]; pos: [n][3];
 * gain: [D] or NULL (= ones); base: [3]. */
void orc_prologue(const double *x, int64_t n, int H, int D, const int32_t *pos,
                  const double *gain, const double *base, double eps, double *out)
{
    int p = (D / 2) / 3;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
        for (int h = 0; h < H; ++h) {
            const double *xr = x + ((size_t)t * H + h) * D;
            double *o = out + ((size_t)t * H + h) * D;
            double ss = 0.0;
            for (int d = 0; d < D; ++d)
                ss += xr[d] * xr[d];
            double r = sqrt(ss / D + eps);
            for (int d = 0; d < D; ++d)
                o[d] = (gain ? gain[d] : 1.0) * xr[d] / r;
            for (int a = 0; a < 3; ++a) {
                for (int k = 0; k < p; ++k) {
                    int c0 = 2 * p * a + 2 * k;
                    double ang = rope_angle(pos[3 * t + a], base[a], k, p);
                    double cs = cos(ang), sn = sin(ang);
                    double y0 = o[c0], y1 = o[c0 + 1];
                    o[c0] = y0 * cs - y1 * sn;
                    o[c0 + 1] = y0 * sn + y1 * cs;
                }
            }
        }
    }
}

/* Backward of orc_prologue: dy = dL/d(out), dx = dL/dx.
 * RoPE^T rotates by -angle; RMSNorm^T: dx = g*dz/r - x * sum(g*dz*x) / (D r^3). */
void orc_prologue_bwd(const double *x, int64_t n, int H, int D, const int32_t *pos,
                      const double *gain, const double *base, double eps,
                      const double *dy, double *dx)
{
    int p = (D / 2) / 3;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
        double dz[256];
        for (int h = 0; h < H; ++h) {
            const double *xr = x + ((size_t)t * H + h) * D;
            const double *g = dy + ((size_t)t * H + h) * D;
            double *o = dx + ((size_t)t * H + h) * D;
            for (int d = 0; d < D; ++d)
                dz[d] = g[d];
            for (int a = 0; a < 3; ++a) {
                for (int k = 0; k < p; ++k) {
                    int c0 = 2 * p * a + 2 * k;
                    double ang = rope_angle(pos[3 * t + a], base[a], k, p);
                    double cs = cos(ang), sn = sin(ang);
                    double y0 = dz[c0], y1 = dz[c0 + 1];
                    dz[c0] = y0 * cs + y1 * sn;
                    dz[c0 + 1] = -y0 * sn + y1 * cs;
                }
            }
            double ss = 0.0;
            for (int d = 0; d < D; ++d)
                ss += xr[d] * xr[d];
            double r = sqrt(ss / D + eps);
            double acc = 0.0;
            for (int d = 0; d < D; ++d)
                acc += (gain ? gain[d] : 1.0) * dz[d] * xr[d];
            for (int d = 0; d < D; ++d)
                o[d] = (gain ? gain[d] : 1.0) * dz[d] / r - xr[d] * acc / ((double)D * r * r * r);
        }
    }
}

/* Gradients of the prologue's parameters, accumulated (+=) over rows: the QK-Norm gain
 * and the three RoPE bases (MAGI-1 research notes, "Autoregressive denoising DiT":
 * QK-Norm, and 3D RoPE with a learnable base frequency).  dy = dL/d(out) per row.
 * With z = x / r, xh = gain * z and y = R(angles) xh:
 *   dL/dgain_d = sum over rows of (R^T dy)_d z_d;
 *   for pair k of axis a, angle = pos_a * base_a^(-k/p), dy/dangle = (-y1, y0), so
 *   dL/dangle = dy1 y0 - dy0 y1 and dangle/dbase_a = -(k/p) angle / base_a. */
void orc_prologue_param_grads(const double *x, int64_t n, int H, int D, const int32_t *pos,
                              const double *gain, const double *base, double eps,
                              const double *dy, double *dgain, double *dbase)
{
    int p = (D / 2) / 3;
    for (int64_t t = 0; t < n; ++t) {
        for (int h = 0; h < H; ++h) {
            const double *xr = x + ((size_t)t * H + h) * D;
            const double *g = dy + ((size_t)t * H + h) * D;
            double z[256], xh[256], dz[256];
            double ss = 0.0;
            for (int d = 0; d < D; ++d)
                ss += xr[d] * xr[d];
            double r = sqrt(ss / D + eps);
            for (int d = 0; d < D; ++d) {
                z[d] = xr[d] / r;
                xh[d] = (gain ? gain[d] : 1.0) * z[d];
                dz[d] = g[d];
            }
            for (int a = 0; a < 3; ++a) {
                for (int k = 0; k < p; ++k) {
                    int c0 = 2 * p * a + 2 * k;
                    double ang = rope_angle(pos[3 * t + a], base[a], k, p);
                    double cs = cos(ang), sn = sin(ang);
                    double y0 = xh[c0] * cs - xh[c0 + 1] * sn;
                    double y1 = xh[c0] * sn + xh[c0 + 1] * cs;
                    double dang = g[c0 + 1] * y0 - g[c0] * y1;
                    dbase[a] += dang * (-(double)k / (double)p) * ang / base[a];
                    dz[c0] = g[c0] * cs + g[c0 + 1] * sn;
                    dz[c0 + 1] = -g[c0] * sn + g[c0 + 1] * cs;
                }
            }
            for (int d = 0; d < D; ++d)
                dgain[d] += dz[d] * z[d];
        }
    }
}

/* One (row, head): scores over the visible keys, LSE and O.  Returns LSE (-inf when
 * the row sees no key, with O = 0). */
static double attend_row(const double *q, const double *kh, const double *v, int64_t nk,
                         const uint8_t *row, int Hkv, int g, int D, double scale, double *o)
{
    double m = -INFINITY;
    for (int64_t j = 0; j < nk; ++j) {
        if (!row[j])
            continue;
        const double *kj = kh + ((size_t)j * Hkv + g) * D;
        double s = 0.0;
        for (int d = 0; d < D; ++d)
            s += q[d] * kj[d];
        s *= scale;
        if (s > m)
            m = s;
    }
    for (int d = 0; d < D; ++d)
        o[d] = 0.0;
    if (m == -INFINITY)
        return -INFINITY;
    double l = 0.0;
    for (int64_t j = 0; j < nk; ++j) {
        if (!row[j])
            continue;
        const double *kj = kh + ((size_t)j * Hkv + g) * D;
        double s = 0.0;
        for (int d = 0; d < D; ++d)
            s += q[d] * kj[d];
        l += exp(s * scale - m);
    }
    double lse = m + log(l);
    for (int64_t j = 0; j < nk; ++j) {
        if (!row[j])
            continue;
        const double *kj = kh + ((size_t)j * Hkv + g) * D;
        const double *vj = v + ((size_t)j * Hkv + g) * D;
        double s = 0.0;
        for (int d = 0; d < D; ++d)
            s += q[d] * kj[d];
        double pr = exp(s * scale - lse);
        for (int d = 0; d < D; ++d)
            o[d] += pr * vj[d];
    }
    return lse;
}

/* Dense mask rows for a list of query rows: masks[r * nk + j]. */
static uint8_t *mask_rows(const int64_t *sl, int ns, int64_t nk, const int64_t *rows, int64_t nr)
{
    uint8_t *m = (uint8_t *)malloc((size_t)(nr > 0 ? nr : 1) * (size_t)(nk > 0 ? nk : 1));
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nr; ++r)
        orc_mask_row(sl, ns, nk, rows[r], m + (size_t)r * (size_t)nk);
    return m;
}

/* Forward for a list of query rows, every head.
 * qh: [nr][Hq][D] = post-prologue queries of those rows (in list order);
 * kh, v: [nk][Hkv][D]; O: [nr][Hq][D]; lse: [nr][Hq] (natural log). */
void orc_fwd_rows(const double *qh, const int64_t *rows, int64_t nr,
                  const double *kh, const double *v, int64_t nk,
                  const int64_t *sl, int ns, int Hq, int Hkv, int D,
                  double *O, double *lse)
{
    int G = Hq / Hkv;
    double scale = 1.0 / sqrt((double)D);
    uint8_t *m = mask_rows(sl, ns, nk, rows, nr);
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t r = 0; r < nr; ++r)
        for (int h = 0; h < Hq; ++h)
            lse[r * Hq + h] = attend_row(qh + ((size_t)r * Hq + h) * D, kh, v, nk, m + (size_t)r * (size_t)nk,
                                         Hkv, h / G, D, scale, O + ((size_t)r * Hq + h) * D);
    free(m);
}

/* dq-hat for a list of rows: forward of the row, Di = dO_i . O_i,
 * dS_ij = P_ij (dO_i . v_j - Di), dqh_i = sum_j dS_ij kh_j / sqrt(D).
 * Also returns the rows' O and LSE. */
void orc_bwd_rows(const double *qh, const int64_t *rows, int64_t nr,
                  const double *kh, const double *v, int64_t nk, const double *dO,
                  const int64_t *sl, int ns, int Hq, int Hkv, int D,
                  double *dqh, double *O, double *lse)
{
    int G = Hq / Hkv;
    double scale = 1.0 / sqrt((double)D);
    orc_fwd_rows(qh, rows, nr, kh, v, nk, sl, ns, Hq, Hkv, D, O, lse);
    uint8_t *m = mask_rows(sl, ns, nk, rows, nr);
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t r = 0; r < nr; ++r) {
        for (int h = 0; h < Hq; ++h) {
            const uint8_t *row = m + (size_t)r * (size_t)nk;
            int g = h / G;
            const double *q = qh + ((size_t)r * Hq + h) * D;
            const double *doi = dO + ((size_t)r * Hq + h) * D;
            const double *oi = O + ((size_t)r * Hq + h) * D;
            double *dq = dqh + ((size_t)r * Hq + h) * D;
            double L = lse[r * Hq + h];
            double Di = 0.0;
            for (int d = 0; d < D; ++d) {
                Di += doi[d] * oi[d];
                dq[d] = 0.0;
            }
            if (L == -INFINITY)
                continue;
            for (int64_t j = 0; j < nk; ++j) {
                if (!row[j])
                    continue;
                const double *kj = kh + ((size_t)j * Hkv + g) * D;
                const double *vj = v + ((size_t)j * Hkv + g) * D;
                double s = 0.0, dp = 0.0;
                for (int d = 0; d < D; ++d) {
                    s += q[d] * kj[d];
                    dp += doi[d] * vj[d];
                }
                double P = exp(s * scale - L);
                double dS = P * (dp - Di);
                for (int d = 0; d < D; ++d)
                    dq[d] += dS * kj[d] * scale;
            }
        }
    }
    free(m);
}

/* dk-hat and dv for a list of keys, for query heads [h_begin, h_end) only (all heads
 * of the KV groups involved must be included for a complete gradient).
 * qh, dO: [nq][Hq][D] for ALL query rows; lse, Dsum: [nq][Hq] from the forward
 * (Dsum_i = dO_i . O_i).  dkh, dv: [nkeys][Hkv][D]; only the groups of
 * [h_begin, h_end) are written (others are zeroed). */
void orc_bwd_keys(const double *qh, const double *dO, const double *lse, const double *Dsum,
                  int64_t nq, const double *kh, const double *v, int64_t nk,
                  const int64_t *keys, int64_t nkeys, int h_begin, int h_end,
                  const int64_t *sl, int ns, int Hq, int Hkv, int D,
                  double *dkh, double *dv)
{
    int G = Hq / Hkv;
    double scale = 1.0 / sqrt((double)D);
    (void)nk;
    memset(dkh, 0, sizeof(double) * (size_t)nkeys * Hkv * D);
    memset(dv, 0, sizeof(double) * (size_t)nkeys * Hkv * D);
#pragma omp parallel
    {
        uint8_t *col = (uint8_t *)malloc((size_t)(nq > 0 ? nq : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t kk = 0; kk < nkeys; ++kk) {
            int64_t j = keys[kk];
            orc_mask_col(sl, ns, nq, j, col);
            for (int64_t i = 0; i < nq; ++i) {
                if (!col[i])
                    continue;
                for (int h = h_begin; h < h_end; ++h) {
                    int g = h / G;
                    double L = lse[i * Hq + h];
                    const double *q = qh + ((size_t)i * Hq + h) * D;
                    const double *doi = dO + ((size_t)i * Hq + h) * D;
                    const double *kj = kh + ((size_t)j * Hkv + g) * D;
                    const double *vj = v + ((size_t)j * Hkv + g) * D;
                    double s = 0.0, dp = 0.0;
                    for (int d = 0; d < D; ++d) {
                        s += q[d] * kj[d];
                        dp += doi[d] * vj[d];
                    }
                    double P = exp(s * scale - L);
                    double dS = P * (dp - Dsum[i * Hq + h]);
                    double *dk = dkh + ((size_t)kk * Hkv + g) * D;
                    double *dvv = dv + ((size_t)kk * Hkv + g) * D;
                    for (int d = 0; d < D; ++d) {
                        dk[d] += dS * q[d] * scale;
                        dvv[d] += P * doi[d];
                    }
                }
            }
        }
        free(col);
    }
}

/* Full backward for small problems: every query row and every key. */
void orc_bwd_dense(const double *qh, const double *kh, const double *v, const double *dO,
                   int64_t nq, int64_t nk, const int64_t *sl, int ns, int Hq, int Hkv, int D,
                   double *dqh, double *dkh, double *dv, double *O, double *lse)
{
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nq > 0 ? nq : 1));
    int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nk > 0 ? nk : 1));
    double *Dsum = (double *)malloc(sizeof(double) * (size_t)(nq > 0 ? nq : 1) * Hq);
    for (int64_t i = 0; i < nq; ++i)
        rows[i] = i;
    for (int64_t j = 0; j < nk; ++j)
        keys[j] = j;
    orc_bwd_rows(qh, rows, nq, kh, v, nk, dO, sl, ns, Hq, Hkv, D, dqh, O, lse);
    for (int64_t i = 0; i < nq; ++i)
        for (int h = 0; h < Hq; ++h) {
            double s = 0.0;
            for (int d = 0; d < D; ++d)
                s += dO[((size_t)i * Hq + h) * D + d] * O[((size_t)i * Hq + h) * D + d];
            Dsum[i * Hq + h] = s;
        }
    orc_bwd_keys(qh, dO, lse, Dsum, nq, kh, v, nk, keys, nk, 0, Hq, sl, ns, Hq, Hkv, D, dkh, dv);
    free(rows);
    free(keys);
    free(Dsum);
}
