#pragma once
// Kernel-variant lookup and the choice of lane layout, shared by the plan-based
// entry points (abi.cu) and the allocation-free one (noalloc.cu).
#include <cstdint>

#include "scan_kernel.cuh"
#include "ssm_scan.h"

namespace ssm {

inline bool pick_variant(int dtype, int64_t N, bool head, bool vec, int w, int spl, Variant* v) {
    const bool bf = dtype == SSM_BF16;
    switch (N) {
        case 8: return bf ? pick_bf16_n8(head, vec, w, spl, v) : pick_f32_n8(head, vec, w, spl, v);
        case 16: return bf ? pick_bf16_n16(head, vec, w, spl, v) : pick_f32_n16(head, vec, w, spl, v);
        case 32: return bf ? pick_bf16_n32(head, vec, w, spl, v) : pick_f32_n32(head, vec, w, spl, v);
        case 64: return bf ? pick_bf16_n64(head, vec, w, spl, v) : pick_f32_n64(head, vec, w, spl, v);
        case 128: return bf ? pick_bf16_n128(head, vec, w, spl, v) : pick_f32_n128(head, vec, w, spl, v);
        default: return false;
    }
}

// Lane layout of a launch: w consumer warps per CTA, spl states per lane.
struct Layout {
    int w, spl;
    Variant v;   // the 16-byte (tensor-map) variant of that layout
};

// Channel tiles of a layout: every (batch row, group) splits its channels into tiles of CT.
inline int64_t layout_tiles(const ssm_dims_t& d, int ct) {
    const int64_t Dg = d.dim / d.ngroups;
    return d.batch * d.ngroups * ((Dg + ct - 1) / ct);
}

// The first layout in order of preference that gives every SM a channel tile,
// else the one with the most tiles.  A segment of a tile runs after the
// previous one, so tiles are the parallelism.  The kernel is latency-bound, so
// the order prefers many consumer warps per SM sub-partition and, among those,
// more states per lane (fewer instructions per state update).  Measured on B200
// with N = 16: 12 warps x 4 states beat 16 x 2 by about 7 % where they fill the
// SMs (4 x 4096 channels), 16 x 2 beat 8 x 4 by about 5 %, and 8 x 4 beat 4 x 4
// by about 30 %.  force_w / force_spl (0 =
// free) restrict the candidates; false: no variant fits them.
inline bool choose_layout(const ssm_dims_t& d, int sm_count, int force_w, int force_spl, Layout* out) {
    const bool head = d.nheads != d.dim;
    static const int order[][2] = {{12, 4}, {16, 2}, {8, 16}, {8, 8}, {8, 4}, {8, 2}, {4, 16}, {4, 8}, {4, 4}, {4, 2}};
    bool found = false;
    Layout best{};
    int64_t best_tiles = -1;
    for (const auto& c : order) {
        if ((force_w && c[0] != force_w) || (force_spl && c[1] != force_spl)) continue;
        Variant v;
        if (!pick_variant(d.io_dtype, d.dstate, head, true, c[0], c[1], &v)) continue;
        const int64_t tiles = layout_tiles(d, v.ch_per_tile);
        if (tiles >= sm_count) {
            *out = Layout{c[0], c[1], v};
            return true;
        }
        if (tiles > best_tiles) {
            best = Layout{c[0], c[1], v};
            best_tiles = tiles;
            found = true;
        }
    }
    if (found) *out = best;
    return found;
}

}  // namespace ssm
