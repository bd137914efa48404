// Host-side plan: validated problem, compiled mask and scheduling tables.
#pragma once

#include <cstdint>
#include <vector>

#include "../../include/bca.h"

namespace bca {

constexpr int kTileQ = 128;  // query rows per tile (= MMA M)
constexpr int kTileK = 128;  // keys per tile (= S-tile N)

// A run of consecutive k-tiles of one q-tile.  mask_idx < 0: every tile in
// [kt_begin, kt_end) is fully visible.  mask_idx >= 0: a single partial tile whose
// 128x128 bitmask is masks[mask_idx] (row r: words 4r..4r+3, bit j%32 of word
// j/32 set iff key kt*128+j is visible to row qt*128+r).
struct Run {
    int32_t kt_begin, kt_end, mask_idx, pad;
};

// Forward work item: q-tile x a set of heads_per_item query heads starting at
// head0, all in one KV group so they stream the same K/V tiles.
struct Item {
    int32_t q_tile, head0;
};

struct Plan {
    // problem
    int hq = 0, hkv = 0, d = 0, dpad = 0;
    int heads_per_item = 2;  // query heads per forward CTA: 2, or 1 for an odd group size
    int64_t nq = 0, nk = 0, nc = 0;
    uint32_t flags = 0;
    float base[3] = {1e4f, 1e4f, 1e4f};
    float eps = 1e-6f;
    std::vector<bca_slice> slices;
    std::vector<bca_video> videos;

    // compiled mask
    int64_t nqt = 0, nkt = 0;
    std::vector<int32_t> run_off;    // [nqt + 1]
    std::vector<Run> runs;
    std::vector<uint32_t> masks;     // [npartial][128][4]
    std::vector<int32_t> qt_tiles;   // k-tiles per q-tile
    int64_t visible_pairs = 0, nfull = 0, npartial = 0;

    // transposed view for the backward: per k-tile, runs of q-tiles that see it
    // (Run.kt_begin/kt_end hold the q-tile range here; a partial tile is its own run)
    std::vector<int32_t> col_off;    // [nkt + 1]
    std::vector<Run> col_runs;
    std::vector<int32_t> kt_qtiles;  // q-tiles per k-tile
    std::vector<int32_t> bwd_items;  // k-tile * hkv + kv head, longest-first

    // schedule and prologue tables
    std::vector<Item> items;         // longest-first
    std::vector<uint32_t> pos;       // packed (t << 16 | h << 8 | w) per new token
    std::vector<float> rope;         // (cos, sin) pairs: [(axis_off[a] + p) * pairs + k]
    int32_t rope_axis_off[3] = {0, 0, 0};
    int32_t rope_pairs = 0;
    int32_t rope_tbase = 0;           // the t table starts at this absolute frame
    size_t rope_capacity = 0;         // floats of the device RoPE table (set at upload)
    // d(base_a^(-k/pairs))/d(base_a) at [8 a + k], for the gradient of the RoPE bases
    float rope_base_coef[24] = {};

    // device copies (owned)
    int device = -1;
    void *d_blob = nullptr;
    const int32_t *d_run_off = nullptr;
    const Run *d_runs = nullptr;
    const uint32_t *d_masks = nullptr;
    const Item *d_items = nullptr;
    const int32_t *d_col_off = nullptr;
    const Run *d_col_runs = nullptr;
    const int32_t *d_bwd_items = nullptr;
    const uint32_t *d_pos = nullptr;
    const float *d_rope = nullptr;
    int *d_status = nullptr;
    int32_t *d_tbase = nullptr;      // rope_tbase on the device (read by the backward's base gradient)

    // per-kernel timing (bca_profile_enable); events are CUDA event handles
    struct ProfRecord {
        int kernel;
        void *start, *stop;
    };
    bool profiling = false;
    std::vector<ProfRecord> prof;
};

// Validate a problem and fill the problem part of a plan.
int validate_problem(const bca_problem *p, Plan &plan);
// Compile the mask into runs / bitmasks, build the item schedule and the tables.
int compile_plan(Plan &plan);
// Positions and RoPE tables from plan.videos (part of compile_plan; also used when only
// the videos' start frames change).
int build_positions(Plan &plan, const Plan *layout = nullptr);
// Expand compiled tiles of rows [r0, r1) into a coverage map (host).
int expand_rows(const Plan &plan, int64_t r0, int64_t r1, uint8_t *out);
// Same from the transposed (backward) runs, for keys [k0, k1): out[(j - k0) * nq + i].
int expand_cols(const Plan &plan, int64_t k0, int64_t k1, uint8_t *out);

}  // namespace bca

// The opaque handle behind bca_plan_t.
struct bca_plan_s {
    bca::Plan plan;
};
