// Mask compiler: AttnSlices -> per-(128 x 128) tile classes -> runs -> work items.
//
// The mask is the union of the slices (MAGI-1 research notes (zhao9797.github.io),
// "Infra > MagiAttention > Flex-Flash-Attention": masks are compositions of
// (QRange, KRange, MaskType) slices; interview with Zhang Zheng (zhengguannews),
// the q_range / k_range answer).  Work items are ordered by the visible area of
// their q-tile, largest first, which is the pages' "balance the unmasked area"
// cost model (interview, the dispatch-solver answer; research notes, "Dispatch
// solver") applied to the SMs of one GPU instead of CP ranks.
#include "plan.hpp"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <thread>

namespace bca {

namespace {

struct Interval {
    int64_t a, b;  // [a, b)
};

// Visible keys of row i through slice s, as one interval (may be empty).
inline Interval slice_row_interval(const bca_slice &s, int64_t i) {
    if (s.type == BCA_SLICE_FULL) return {s.k_begin, s.k_end};
    // causal, bottom-right aligned: j - k0 <= (i - q0) + (|k| - |q|)
    int64_t lim = s.k_begin + (i - s.q_begin) + ((s.k_end - s.k_begin) - (s.q_end - s.q_begin)) + 1;
    return {s.k_begin, std::min(s.k_end, std::max(lim, s.k_begin))};
}

// Per-q-tile compile output, merged in q-tile order afterwards.
struct TileOut {
    std::vector<Run> runs;          // mask_idx local to this q-tile
    std::vector<uint32_t> masks;    // local partial masks
    int64_t pairs = 0, nfull = 0, npartial = 0;
    int32_t ntiles = 0;
};

void compile_q_tile(const Plan &P, int64_t qt, TileOut &out) {
    const int64_t r0 = qt * kTileQ;
    const int nr = (int)std::min<int64_t>(kTileQ, P.nq - r0);
    // 1. merged visible intervals of every row
    std::vector<std::vector<Interval>> iv(nr);
    for (const bca_slice &s : P.slices) {
        int64_t lo = std::max(s.q_begin, r0), hi = std::min(s.q_end, r0 + nr);
        for (int64_t i = lo; i < hi; ++i) {
            Interval x = slice_row_interval(s, i);
            if (x.b > x.a) iv[i - r0].push_back(x);
        }
    }
    int64_t tmin = INT64_MAX, tmax = -1;
    for (auto &v : iv) {
        if (v.empty()) continue;
        std::sort(v.begin(), v.end(), [](const Interval &x, const Interval &y) { return x.a < y.a; });
        std::vector<Interval> m;
        for (const Interval &x : v) {
            if (!m.empty() && x.a <= m.back().b) m.back().b = std::max(m.back().b, x.b);
            else m.push_back(x);
        }
        v.swap(m);
        for (const Interval &x : v) {
            out.pairs += x.b - x.a;
            tmin = std::min(tmin, x.a / kTileK);
            tmax = std::max(tmax, (x.b - 1) / kTileK);
        }
    }
    if (tmax < 0) return;
    // 2. per k-tile: rows that cover it fully (difference array) and rows that
    //    cover it partly
    const int64_t span = tmax - tmin + 1;
    std::vector<int32_t> diff(span + 1, 0);
    std::vector<uint8_t> touched(span, 0);
    for (const auto &v : iv) {
        for (const Interval &x : v) {
            int64_t fa = (x.a + kTileK - 1) / kTileK, fb = x.b / kTileK;  // fully covered [fa, fb)
            if (fa < fb) {
                diff[fa - tmin] += 1;
                diff[fb - tmin] -= 1;
            }
            int64_t ta = x.a / kTileK, tb = (x.b - 1) / kTileK;
            if (!(fa <= ta && ta < fb)) touched[ta - tmin] = 1;
            if (!(fa <= tb && tb < fb)) touched[tb - tmin] = 1;
        }
    }
    // 3. classify and emit runs
    int32_t cnt = 0;
    for (int64_t t = tmin; t <= tmax; ++t) {
        cnt += diff[t - tmin];
        const bool in_range = (t + 1) * kTileK <= P.nk;
        const bool tch = touched[t - tmin] != 0;
        if (cnt == nr && !tch && in_range) {
            if (!out.runs.empty() && out.runs.back().mask_idx < 0 && out.runs.back().kt_end == t)
                out.runs.back().kt_end = (int32_t)(t + 1);
            else
                out.runs.push_back({(int32_t)t, (int32_t)(t + 1), -1, 0});
            out.nfull++;
            out.ntiles++;
        } else if (cnt == 0 && !tch) {
            continue;  // empty
        } else {
            const int32_t idx = (int32_t)(out.masks.size() / (kTileQ * 4));
            out.masks.resize(out.masks.size() + kTileQ * 4, 0u);
            uint32_t *mk = out.masks.data() + (size_t)idx * kTileQ * 4;
            const int64_t k0 = t * kTileK, k1 = k0 + kTileK;
            for (int r = 0; r < nr; ++r) {
                for (const Interval &x : iv[r]) {
                    int64_t a = std::max(x.a, k0), b = std::min(x.b, k1);
                    for (int64_t j = a; j < b; ++j) mk[r * 4 + (j - k0) / 32] |= 1u << ((j - k0) % 32);
                }
            }
            out.runs.push_back({(int32_t)t, (int32_t)(t + 1), idx, 0});
            out.npartial++;
            out.ntiles++;
        }
    }
}

}  // namespace

int validate_problem(const bca_problem *p, Plan &P) {
    if (!p) return BCA_ERR_INVALID_ARGUMENT;
    if (p->flags & ~(BCA_O_FP32 | BCA_PLAN_HOST_ONLY | BCA_TEST_FORCE_TIMEOUT | BCA_FWD_FP8_E4M3 | BCA_NO_PROLOGUE |
                     BCA_DQ_DETERMINISTIC | BCA_CACHE_K_FP16))
        return BCA_ERR_INVALID_ARGUMENT;
    if ((p->flags & BCA_FWD_FP8_E4M3) && (p->flags & (BCA_NO_PROLOGUE | BCA_CACHE_K_FP16))) return BCA_ERR_UNSUPPORTED;
    if (p->num_q_heads <= 0 || p->num_kv_heads <= 0) return BCA_ERR_INVALID_ARGUMENT;
    if (p->num_q_heads % p->num_kv_heads != 0) return BCA_ERR_UNSUPPORTED;
    if (p->head_dim != 24 && p->head_dim != 32 && p->head_dim != 48) return BCA_ERR_UNSUPPORTED;
    if (p->num_videos < 0 || (p->num_videos > 0 && !p->videos)) return BCA_ERR_INVALID_ARGUMENT;
    if (p->num_cache_keys < 0) return BCA_ERR_INVALID_ARGUMENT;
    if (p->num_slices < 0 || (p->num_slices > 0 && !p->slices)) return BCA_ERR_INVALID_ARGUMENT;
    for (int a = 0; a < 3; ++a)
        if (!(p->rope_base[a] > 0.0f) || !std::isfinite(p->rope_base[a])) return BCA_ERR_INVALID_ARGUMENT;
    if (!(p->norm_eps >= 0.0f) || !std::isfinite(p->norm_eps)) return BCA_ERR_INVALID_ARGUMENT;

    P.hq = p->num_q_heads;
    P.hkv = p->num_kv_heads;
    P.d = p->head_dim;
    P.dpad = (p->head_dim + 15) / 16 * 16;
    P.flags = p->flags;
    P.eps = p->norm_eps;
    for (int a = 0; a < 3; ++a) P.base[a] = p->rope_base[a];
    P.nc = p->num_cache_keys;
    int64_t nq = 0;
    P.videos.assign(p->videos, p->videos + p->num_videos);
    for (const bca_video &v : P.videos) {
        if (v.num_chunks < 0 || v.frames <= 0 || v.height <= 0 || v.width <= 0 || v.t0 < 0)
            return BCA_ERR_INVALID_ARGUMENT;
        // packed RoPE positions: t - (smallest t0) < 65536, h, w < 256
        if (v.height > 256 || v.width > 256) return BCA_ERR_UNSUPPORTED;
        if ((int64_t)v.t0 + (int64_t)v.num_chunks * v.frames > INT32_MAX) return BCA_ERR_UNSUPPORTED;
        nq += (int64_t)v.num_chunks * v.frames * v.height * v.width;  // <= 2^47 per video
        if (nq >= ((int64_t)1 << 31)) return BCA_ERR_UNSUPPORTED;      // checked per video: no wrap
    }
    P.nq = nq;
    P.nk = P.nc + nq;
    if (P.nq >= ((int64_t)1 << 31) || P.nk >= ((int64_t)1 << 31)) return BCA_ERR_UNSUPPORTED;

    if (p->slices) {
        P.slices.assign(p->slices, p->slices + p->num_slices);
        for (const bca_slice &s : P.slices) {
            if (s.type != BCA_SLICE_FULL && s.type != BCA_SLICE_CAUSAL) return BCA_ERR_BAD_SLICE;
            if (s.q_begin < 0 || s.q_begin > s.q_end || s.q_end > P.nq) return BCA_ERR_BAD_SLICE;
            if (s.k_begin < 0 || s.k_begin > s.k_end || s.k_end > P.nk) return BCA_ERR_BAD_SLICE;
        }
    } else {
        // default: block-causal per video; the cache is visible to the first video
        int64_t qoff = 0;
        for (size_t vi = 0; vi < P.videos.size(); ++vi) {
            const bca_video &v = P.videos[vi];
            const int64_t C = (int64_t)v.frames * v.height * v.width;
            const int64_t kbase = P.nc + qoff;
            for (int c = 0; c < v.num_chunks; ++c) {
                bca_slice s;
                s.q_begin = qoff + c * C;
                s.q_end = qoff + (c + 1) * C;
                s.k_begin = (vi == 0) ? 0 : kbase;
                s.k_end = kbase + (c + 1) * C;
                s.type = BCA_SLICE_FULL;
                P.slices.push_back(s);
            }
            qoff += (int64_t)v.num_chunks * C;
        }
    }
    return BCA_OK;
}

int compile_plan(Plan &P) {
    P.nqt = (P.nq + kTileQ - 1) / kTileQ;
    P.nkt = (P.nk + kTileK - 1) / kTileK;

    // ---- mask compile, parallel over q-tiles (static contiguous ranges) ----
    std::vector<TileOut> outs(P.nqt);
    unsigned nth = std::max(1u, std::min(32u, std::thread::hardware_concurrency()));
    if (P.nqt < 64) nth = 1;
    {
        std::vector<std::thread> th;
        for (unsigned t = 0; t < nth; ++t) {
            th.emplace_back([&, t]() {
                for (int64_t qt = t; qt < P.nqt; qt += nth) compile_q_tile(P, qt, outs[qt]);
            });
        }
        for (auto &x : th) x.join();
    }
    P.run_off.assign(P.nqt + 1, 0);
    P.qt_tiles.assign(P.nqt, 0);
    P.runs.clear();
    P.masks.clear();
    P.visible_pairs = P.nfull = P.npartial = 0;
    for (int64_t qt = 0; qt < P.nqt; ++qt) {
        TileOut &o = outs[qt];
        const int32_t base = (int32_t)(P.masks.size() / (kTileQ * 4));
        P.run_off[qt] = (int32_t)P.runs.size();
        for (Run r : o.runs) {
            if (r.mask_idx >= 0) r.mask_idx += base;
            P.runs.push_back(r);
        }
        P.masks.insert(P.masks.end(), o.masks.begin(), o.masks.end());
        P.qt_tiles[qt] = o.ntiles;
        P.visible_pairs += o.pairs;
        P.nfull += o.nfull;
        P.npartial += o.npartial;
        std::vector<Run>().swap(o.runs);
        std::vector<uint32_t>().swap(o.masks);
    }
    P.run_off[P.nqt] = (int32_t)P.runs.size();

    // ---- transposed runs for the backward (k-tile -> q-tiles), built by a
    //      counting pass over the forward runs in q-tile order ----
    {
        std::vector<int64_t> cnt(P.nkt + 1, 0);
        for (const Run &r : P.runs)
            for (int32_t t = r.kt_begin; t < r.kt_end; ++t) cnt[t + 1]++;
        for (int64_t t = 0; t < P.nkt; ++t) cnt[t + 1] += cnt[t];
        std::vector<int64_t> fill(cnt.begin(), cnt.end() - 1);
        std::vector<int32_t> ent_qt((size_t)cnt[P.nkt]), ent_mask((size_t)cnt[P.nkt]);
        for (int64_t qt = 0; qt < P.nqt; ++qt)
            for (int32_t ri = P.run_off[qt]; ri < P.run_off[qt + 1]; ++ri) {
                const Run &r = P.runs[ri];
                for (int32_t t = r.kt_begin; t < r.kt_end; ++t) {
                    const int64_t at = fill[t]++;
                    ent_qt[at] = (int32_t)qt;
                    ent_mask[at] = r.mask_idx;
                }
            }
        P.col_off.assign(P.nkt + 1, 0);
        P.kt_qtiles.assign(P.nkt, 0);
        P.col_runs.clear();
        for (int64_t t = 0; t < P.nkt; ++t) {
            P.col_off[t] = (int32_t)P.col_runs.size();
            for (int64_t e = cnt[t]; e < cnt[t + 1]; ++e) {
                const int32_t qt = ent_qt[e], mk = ent_mask[e];
                if (mk < 0 && !P.col_runs.empty() && (int64_t)P.col_off[t] < (int64_t)P.col_runs.size() &&
                    P.col_runs.back().mask_idx < 0 && P.col_runs.back().kt_end == qt)
                    P.col_runs.back().kt_end = qt + 1;
                else
                    P.col_runs.push_back({qt, qt + 1, mk, 0});
            }
            P.kt_qtiles[t] = (int32_t)(cnt[t + 1] - cnt[t]);
        }
        P.col_off[P.nkt] = (int32_t)P.col_runs.size();
        P.bwd_items.resize((size_t)P.nkt * P.hkv);
        for (int64_t t = 0; t < P.nkt; ++t)
            for (int g = 0; g < P.hkv; ++g) P.bwd_items[t * P.hkv + g] = (int32_t)(t * P.hkv + g);
        std::stable_sort(P.bwd_items.begin(), P.bwd_items.end(), [&](int32_t x, int32_t y) {
            const int32_t cx = P.kt_qtiles[x / P.hkv], cy = P.kt_qtiles[y / P.hkv];
            if (cx != cy) return cx > cy;
            const int gx = x % P.hkv, gy = y % P.hkv;
            if (gx != gy) return gx < gy;
            return x < y;
        });
    }

    // ---- items, longest first; ties grouped by KV group then q-tile so that CTAs
    //      running together stream the same K/V tiles ----
    const int G = P.hq / P.hkv;
    // two query heads of one KV group per forward CTA share each K/V tile; an odd group
    // size (MHA included) runs one head per CTA
    P.heads_per_item = (G % 2 == 0) ? 2 : 1;
    const int nsets = P.hq / P.heads_per_item;
    P.items.clear();
    P.items.reserve((size_t)P.nqt * nsets);
    for (int64_t qt = 0; qt < P.nqt; ++qt)
        for (int hs = 0; hs < nsets; ++hs) P.items.push_back({(int32_t)qt, hs * P.heads_per_item});
    std::stable_sort(P.items.begin(), P.items.end(), [&](const Item &x, const Item &y) {
        const int32_t cx = P.qt_tiles[x.q_tile], cy = P.qt_tiles[y.q_tile];
        if (cx != cy) return cx > cy;
        const int gx = x.head0 / G, gy = y.head0 / G;
        if (gx != gy) return gx < gy;
        if (x.q_tile != y.q_tile) return x.q_tile < y.q_tile;
        return x.head0 < y.head0;
    });

    return build_positions(P);
}

// Packed positions of the new tokens and the RoPE cos/sin tables, from P.videos.  The
// t field holds t - tbase (tbase = the smallest t0 of a non-empty video) and the t table
// covers [tbase, tbase + extent), so a window that slides by shifting every t0 keeps
// the same table size.  With `layout` (bca_plan_update_positions on an uploaded plan)
// the axis offsets and table size are taken from it, and a t or h extent that does not
// fit returns BCA_ERR_UNSUPPORTED.
int build_positions(Plan &P, const Plan *layout) {
    P.pos.resize(P.nq);
    int32_t tbase = INT32_MAX;
    for (const bca_video &v : P.videos)
        if (v.num_chunks > 0) tbase = std::min(tbase, v.t0);
    if (tbase == INT32_MAX) tbase = 0;
    int32_t tmax = 0, hmax = 0, wmax = 0;
    int64_t n = 0;
    for (const bca_video &v : P.videos) {
        for (int c = 0; c < v.num_chunks; ++c)
            for (int f = 0; f < v.frames; ++f)
                for (int y = 0; y < v.height; ++y)
                    for (int x = 0; x < v.width; ++x) {
                        const int64_t trel = (int64_t)v.t0 + (int64_t)c * v.frames + f - tbase;
                        if (trel >= 65536) return BCA_ERR_UNSUPPORTED;
                        const uint32_t t = (uint32_t)trel;
                        P.pos[n++] = (t << 16) | ((uint32_t)y << 8) | (uint32_t)x;
                        tmax = std::max<int32_t>(tmax, (int32_t)t);
                        hmax = std::max(hmax, y);
                        wmax = std::max(wmax, x);
                    }
    }
    const int pairs = (P.d / 2) / 3;
    P.rope_pairs = pairs;
    P.rope_tbase = tbase;
    const int32_t ext[3] = {tmax + 1, hmax + 1, wmax + 1};
    if (layout) {
        // Keep the table layout of an uploaded plan: its launches (also those captured in
        // CUDA graphs) hold the axis offsets by value, so only the entries may change.
        const int32_t *lo = layout->rope_axis_off;
        if (ext[0] > lo[1] || ext[1] > lo[2] - lo[1] ||
            (size_t)(lo[2] + ext[2]) * pairs * 2 > layout->rope_capacity)
            return BCA_ERR_UNSUPPORTED;
        for (int a = 0; a < 3; ++a) P.rope_axis_off[a] = lo[a];
        P.rope.assign(layout->rope_capacity, 0.0f);
    } else {
        P.rope_axis_off[0] = 0;
        P.rope_axis_off[1] = ext[0];
        P.rope_axis_off[2] = ext[0] + ext[1];
        P.rope.assign((size_t)(ext[0] + ext[1] + ext[2]) * pairs * 2, 0.0f);
    }
    for (int a = 0; a < 3; ++a) {
        for (int32_t pp = 0; pp < ext[a]; ++pp) {
            const double position = (double)pp + (a == 0 ? (double)tbase : 0.0);
            for (int k = 0; k < pairs; ++k) {
                const double ang = position * std::pow((double)P.base[a], -(double)k / (double)pairs);
                const size_t at = ((size_t)(P.rope_axis_off[a] + pp) * pairs + k) * 2;
                P.rope[at] = (float)std::cos(ang);
                P.rope[at + 1] = (float)std::sin(ang);
            }
        }
    }
    for (int a = 0; a < 3; ++a)
        for (int k = 0; k < pairs && k < 8; ++k) {
            const double e = -(double)k / (double)pairs;
            P.rope_base_coef[8 * a + k] = (float)(e * std::pow((double)P.base[a], e - 1.0));
        }
    return BCA_OK;
}

int expand_rows(const Plan &P, int64_t r0, int64_t r1, uint8_t *out) {
    if (r0 < 0 || r1 < r0 || r1 > P.nq || !out) return BCA_ERR_INVALID_ARGUMENT;
    std::memset(out, 0, (size_t)(r1 - r0) * (size_t)P.nk);
    for (int64_t i = r0; i < r1; ++i) {
        const int64_t qt = i / kTileQ;
        const int r = (int)(i - qt * kTileQ);
        uint8_t *row = out + (size_t)(i - r0) * (size_t)P.nk;
        for (int32_t ri = P.run_off[qt]; ri < P.run_off[qt + 1]; ++ri) {
            const Run &run = P.runs[ri];
            for (int32_t t = run.kt_begin; t < run.kt_end; ++t) {
                const int64_t k0 = (int64_t)t * kTileK;
                for (int j = 0; j < kTileK; ++j) {
                    const int64_t key = k0 + j;
                    bool vis;
                    if (run.mask_idx < 0) vis = true;
                    else vis = (P.masks[((size_t)run.mask_idx * kTileQ + r) * 4 + j / 32] >> (j % 32)) & 1u;
                    if (vis) {
                        if (key >= P.nk) return BCA_ERR_BAD_SLICE;  // a compiled key out of range
                        row[key] = (uint8_t)(row[key] + 1);
                    }
                }
            }
        }
    }
    return BCA_OK;
}

int expand_cols(const Plan &P, int64_t k0, int64_t k1, uint8_t *out) {
    if (k0 < 0 || k1 < k0 || k1 > P.nk || !out) return BCA_ERR_INVALID_ARGUMENT;
    std::memset(out, 0, (size_t)(k1 - k0) * (size_t)P.nq);
    for (int64_t j = k0; j < k1; ++j) {
        const int64_t kt = j / kTileK;
        const int c = (int)(j - kt * kTileK);
        uint8_t *col = out + (size_t)(j - k0) * (size_t)P.nq;
        for (int32_t ri = P.col_off[kt]; ri < P.col_off[kt + 1]; ++ri) {
            const Run &run = P.col_runs[ri];
            for (int32_t qt = run.kt_begin; qt < run.kt_end; ++qt) {
                for (int r = 0; r < kTileQ; ++r) {
                    const int64_t q = (int64_t)qt * kTileQ + r;
                    if (q >= P.nq) break;
                    const bool vis = run.mask_idx < 0 ||
                                     ((P.masks[((size_t)run.mask_idx * kTileQ + r) * 4 + c / 32] >> (c % 32)) & 1u);
                    if (vis) col[q] = (uint8_t)(col[q] + 1);
                }
            }
        }
    }
    return BCA_OK;
}

}  // namespace bca
