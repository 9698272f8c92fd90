#pragma once
// Everything the forward entry points share: the shape check, the kernel-variant
// lookup, the choice of lane layout and schedule, the workspace layout, the tensor
// maps and the launch.  Both the plan-based entry points (abi.cu) and the
// allocation-free one (noalloc.cu) go through these, so the two cannot drift apart.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "scan_kernel.cuh"
#include "ssm_scan.h"

namespace ssm {

// Sizes and layout codes every forward entry point accepts.
inline bool dims_ok(const ssm_dims_t* d) {
    if (!d) return false;
    if (d->batch < 0 || d->dim <= 0 || d->seqlen < 0 || d->dstate <= 0) return false;
    if (d->nheads <= 0 || d->ngroups <= 0) return false;
    if (d->dim % d->nheads || d->dim % d->ngroups) return false;
    if (d->io_dtype != SSM_F32 && d->io_dtype != SSM_BF16) return false;
    if (d->reserved != 0) return false;
    const int64_t lim = (int64_t)1 << 46;
    const int64_t L = d->seqlen > 0 ? d->seqlen : 1;
    if (d->batch > lim / d->dim || d->batch * d->dim > lim / L) return false;
    if (d->batch * d->ngroups > lim / (d->dstate * L)) return false;
    return true;
}

inline bool head_mode(const ssm_dims_t& d) { return d.nheads != d.dim; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The kernel variant of a lane layout.  mode 0: the register kernel (every dtype, N and
// A layout; kt must be 1); mode 1: the tensor-memory kernel (bf16, N = 16, A per channel).
inline bool pick_variant(int dtype, int64_t N, bool head, bool vec, int w, int spl, int kt, int mode, Variant* v) {
    const bool bf = dtype == SSM_BF16;
    if (mode == 1) return bf && N == 16 && !head && pick_tc(vec, w, spl, kt, mode, v);
    switch (N) {
        case 8: return bf ? pick_bf16_n8(head, vec, w, spl, kt, mode, v) : pick_f32_n8(head, vec, w, spl, kt, mode, v);
        case 16: return bf ? pick_bf16_n16(head, vec, w, spl, kt, mode, v) : pick_f32_n16(head, vec, w, spl, kt, mode, v);
        case 32: return bf ? pick_bf16_n32(head, vec, w, spl, kt, mode, v) : pick_f32_n32(head, vec, w, spl, kt, mode, v);
        case 64: return bf ? pick_bf16_n64(head, vec, w, spl, kt, mode, v) : pick_f32_n64(head, vec, w, spl, kt, mode, v);
        case 128:
            return bf ? pick_bf16_n128(head, vec, w, spl, kt, mode, v) : pick_f32_n128(head, vec, w, spl, kt, mode, v);
        default: return false;
    }
}

// Lane layout of a launch: w consumer warps per CTA, spl states per lane, kt time
// sub-chunks per block (1: the state-parallel recurrence; 2 or 4: sequence-parallel
// blocks), mode (0: B and C through shared memory; 1: through tensor memory).
struct Layout {
    int w, spl, kt, mode;
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
// the order prefers many consumer warps per SM sub-partition and, among those, more
// states per lane.  Measured on B200 with the current readouts (bf16, N = 16):
// 4 x 4096 channels x 4096 steps, (16, 2) 0.449 ms, (12, 4) 0.461, (8, 4) 0.470,
// (8, 2) 0.504; 8 x 1536 x 2048, (16, 2) 0.189, (8, 4) 0.196, (8, 2) 0.202, (12, 4)
// 0.226 (128 tiles); 1 x 5120 x 65536, (8, 2) 2.41, (4, 4) 3.64 (before the loads
// ahead), (4, 2) 4.08, (8, 4) 4.32 (80 tiles).  The tensor-memory layouts (bf16, N = 16, A per channel: no bf16
// unpacking and no shared-memory traffic for B and C) come last: measured on B200
// they run no faster than the register kernel (mamba-130m 0.206 against 0.208 ms,
// mamba-1.4b 0.489 against 0.462 ms), and their sequence-parallel blocks (kt = 2),
// which double the warps on a tile at about 1.5 more instructions per state update,
// lose to the chained segments on the long batch-1 shape (5120 channels x 65536
// steps: 3.55 against 3.40 ms).  force_w / force_spl / force_kt (0 = free) and
// force_mode (0 = free, 1 = register kernel only, 2 = tensor-memory kernel only)
// restrict the candidates; false: no variant fits them.
inline bool choose_layout(const ssm_dims_t& d, int sm_count, int force_w, int force_spl, int force_kt,
                          int force_mode, Layout* out) {
    const bool head = head_mode(d);
    static const int order[][4] = {{16, 2, 1, 0}, {12, 4, 1, 0}, {8, 16, 1, 0}, {8, 8, 1, 0},  {8, 4, 1, 0},
                                   {8, 2, 1, 0},  {4, 16, 1, 0}, {4, 8, 1, 0},  {4, 4, 1, 0},  {4, 2, 1, 0},
                                   {16, 2, 1, 1}, {12, 4, 1, 1}, {8, 4, 1, 1},  {16, 2, 2, 1}, {8, 2, 2, 1}};
    bool found = false;
    Layout best{};
    int64_t best_tiles = -1;
    for (const auto& c : order) {
        if ((force_w && c[0] != force_w) || (force_spl && c[1] != force_spl) || (force_kt && c[2] != force_kt))
            continue;
        if ((force_mode == 1 && c[3] != 0) || (force_mode == 2 && c[3] != 1)) continue;
        Variant v;
        if (!pick_variant(d.io_dtype, d.dstate, head, true, c[0], c[1], c[2], c[3], &v)) continue;
        const int64_t tiles = layout_tiles(d, v.ch_per_tile);
        if (tiles >= sm_count) {
            *out = Layout{c[0], c[1], c[2], c[3], v};
            return true;
        }
        if (tiles > best_tiles) {
            best = Layout{c[0], c[1], c[2], c[3], v};
            best_tiles = tiles;
            found = true;
        }
    }
    if (found) *out = best;
    return found;
}

// The schedule of a forward launch and the layout of its workspace:
// header (64 bytes) | flags[n_tiles] (from flags_off) | carry[n_tiles][CT][N] fp32 (from carry_off).
struct FwdGeom {
    Layout lay;
    int64_t n_tiles, tiles_per_group, seg_len, n_seg, n_units, ctas;
    size_t flags_off, carry_off, ws_bytes;
};

// Layout, segment length and persistent-CTA count for `sm_count` SMs; the knobs
// (0 = free) force a layout, a segment length or fewer CTAs.  Checks that the
// kernel fits an SM (occupancy >= 1).  Allocates nothing.
inline int fwd_geometry(const ssm_dims_t& d, int sm_count, int force_w, int force_spl, int force_kt,
                        int force_mode, int64_t force_seg_len, int64_t force_workers, FwdGeom* g) {
    Layout lay;
    if (!choose_layout(d, sm_count, force_w, force_spl, force_kt, force_mode, &lay)) return SSM_ERR_UNSUPPORTED;
    const Variant& v = lay.v;
    if (v.smem > 48 * 1024 &&
        cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, v.smem) != cudaSuccess)
        return SSM_ERR_CUDA;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, v.fn, v.threads, v.smem) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (occ < 1) return SSM_ERR_UNSUPPORTED;
    const int64_t Dg = d.dim / d.ngroups;
    const int64_t n_tiles = layout_tiles(d, v.ch_per_tile);
    int64_t ctas = sm_count;  // one persistent CTA per SM
    if (force_workers > 0 && force_workers < ctas) ctas = force_workers;
    const int64_t L = d.seqlen;
    const int64_t tb = v.tb;   // segments hold whole blocks
    const int64_t seg_len = force_seg_len > 0 ? (force_seg_len + tb - 1) / tb * tb : default_seg_len(L, n_tiles, ctas);
    const int64_t n_seg = L > 0 ? (L + seg_len - 1) / seg_len : 1;
    const int64_t n_units = n_tiles * n_seg;
    if (n_units >= (int64_t)1 << 31 || seg_len > (int64_t)1 << 30) return SSM_ERR_UNSUPPORTED;
    if (ctas > n_units) ctas = n_units;
    if (ctas < 1) ctas = 1;
    g->lay = lay;
    g->n_tiles = n_tiles;
    g->tiles_per_group = (Dg + v.ch_per_tile - 1) / v.ch_per_tile;
    g->seg_len = seg_len;
    g->n_seg = n_seg;
    g->n_units = n_units;
    g->ctas = ctas;
    g->flags_off = 64;
    g->carry_off = (g->flags_off + (size_t)n_tiles * 4 + 255) / 256 * 256;
    g->ws_bytes = g->carry_off + (size_t)n_tiles * v.ch_per_tile * d.dstate * 4;
    return SSM_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn tensor_map_encoder() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load(std::memory_order_acquire);
    if (!f) {
        void* sym = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &sym, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            f = reinterpret_cast<EncodeTiledFn>(sym);
            fn.store(f, std::memory_order_release);
        }
    }
    return f;
}

// A (rows x cols) row-major tensor seen as 2-D boxes of box_cols steps x box_rows rows.
inline bool encode_rows(CUtensorMap* m, const void* base, int esz, uint64_t cols, uint64_t rows, uint32_t box_rows,
                        CUtensorMapSwizzle swz, uint32_t box_cols = kTB) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc || cols == 0 || rows == 0) return false;
    const cuuint64_t gdim[2] = {cols, rows};
    const cuuint64_t gstride[1] = {cols * (uint64_t)esz};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
               const_cast<void*>(base), gdim, gstride, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The caller's tensors of one forward call.
struct FwdArgs {
    const void* u;
    const void* delta;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const void* z;
    const float* delta_bias;
    int softplus;
    const float* h0;
    void* out;
    float* last_state;
    float* ckpt = nullptr;   // states entering every 8-step window (register kernel only)
};

// Launch the scan kernel of geometry `g` on workspace `ws` (laid out as FwdGeom says).
// The tensor-map (16-byte) variant when every row the maps describe is 16-byte
// aligned (L % 16 == 0 and aligned bases), else the guarded element-copy variant
// of the same layout.
inline int fwd_launch(const ssm_dims_t& d, const FwdGeom& g, const FwdArgs& a, unsigned char* ws,
                      unsigned spin_limit, cudaStream_t stream) {
    const int esz = d.io_dtype == SSM_BF16 ? 2 : 4;
    const int64_t P = d.dim / d.nheads;
    const int ct = g.lay.v.ch_per_tile;
    int delta_rows = ct;
    if (head_mode(d)) {
        delta_rows = (int)((ct - 1) / P + 2);
        if (delta_rows > ct) delta_rows = ct;
    }
    bool vec = d.seqlen > 0 && (d.seqlen % 16 == 0) && aligned16(a.u) && aligned16(a.delta) && aligned16(a.B) &&
               aligned16(a.C) && aligned16(a.out) && (!a.z || aligned16(a.z));
    TensorMaps tm;
    std::memset(&tm, 0, sizeof(tm));
    if (vec) {
        // boxes of one block (tb steps); B and C rows of 64 bytes take the 64-byte swizzle, of 128 the 128-byte one
        const uint32_t tb = (uint32_t)g.lay.v.tb;
        const CUtensorMapSwizzle bc_swz = tb * esz == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
        const uint64_t L = (uint64_t)d.seqlen;
        vec = encode_rows(&tm.u, a.u, esz, L, (uint64_t)(d.batch * d.dim), ct, CU_TENSOR_MAP_SWIZZLE_NONE, tb) &&
              encode_rows(&tm.delta, a.delta, esz, L, (uint64_t)(d.batch * d.nheads), delta_rows,
                          CU_TENSOR_MAP_SWIZZLE_NONE, tb) &&
              (!a.z ||
               encode_rows(&tm.z, a.z, esz, L, (uint64_t)(d.batch * d.dim), ct, CU_TENSOR_MAP_SWIZZLE_NONE, tb)) &&
              encode_rows(&tm.B, a.B, esz, L, (uint64_t)(d.batch * d.ngroups * d.dstate), (uint32_t)d.dstate,
                          bc_swz, tb) &&
              encode_rows(&tm.C, a.C, esz, L, (uint64_t)(d.batch * d.ngroups * d.dstate), (uint32_t)d.dstate,
                          bc_swz, tb);
        // a shape the tensor maps cannot describe takes the element-copy path
    }
    // with stored states: the register kernel's mode-2 variant of the same layout (the
    // tensor-memory kernel stores none)
    if (a.ckpt && g.lay.mode != 0) return SSM_ERR_UNSUPPORTED;
    Variant v;
    if (!pick_variant(d.io_dtype, d.dstate, head_mode(d), vec, g.lay.w, g.lay.spl, g.lay.kt, a.ckpt ? 2 : g.lay.mode,
                      &v))
        return SSM_ERR_UNSUPPORTED;
    FwdParams prm;
    prm.u = a.u; prm.delta = a.delta; prm.A = a.A; prm.B = a.B; prm.C = a.C; prm.D = a.D; prm.z = a.z;
    prm.bias = a.delta_bias; prm.h0 = a.h0; prm.out = a.out; prm.last_state = a.last_state;
    prm.ws = reinterpret_cast<WsHeader*>(ws);
    prm.flags = reinterpret_cast<unsigned*>(ws + g.flags_off);
    prm.carry = reinterpret_cast<float*>(ws + g.carry_off);
    prm.batch = d.batch; prm.dim = d.dim; prm.seqlen = d.seqlen; prm.nheads = d.nheads; prm.ngroups = d.ngroups;
    prm.softplus = a.softplus ? 1 : 0;
    prm.tiles_per_group = (int)g.tiles_per_group;
    prm.n_tiles = (int)g.n_tiles;
    prm.n_seg = (int)g.n_seg;
    prm.seg_len = (int)g.seg_len;
    prm.n_units = (unsigned)g.n_units;
    prm.n_ctas = (unsigned)g.ctas;
    prm.spin_limit = spin_limit;
    prm.delta_rows = delta_rows;
    prm.ckpt = a.ckpt;
    prm.ckpt_wins = (d.seqlen + 7) / 8;
    if (v.smem > 48 * 1024 &&
        cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, v.smem) != cudaSuccess)
        return SSM_ERR_CUDA;
    v.fn<<<(unsigned)g.ctas, v.threads, v.smem, stream>>>(prm, tm);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // namespace ssm
